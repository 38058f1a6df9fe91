"""Pins of the oracle's multi-frame canvas (oracle.positions_frames): several
<image> frames per prompt on an s x s grid.

The pages print the canvas for one 448x448 thumbnail only (HF card
mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI, "How the VLM rides the text-only
engine": the 8x8 table, and 9 = max(H, W) + 1 for the text after it); the MNN
card ("Validation") says sliced and multi-image prompts were checked too,
without values.  So the multi-frame values are a reading and their parity
with the pages is unpinned; what pins the oracle here:
  * one frame at s = 8 is the canvas rule (oracle.positions, itself pinned to
    the pages' table), on the golden O = 6 prompt and on every origin 0..100;
  * a closed form written independently of the oracle's running counter
    (frame i is the one-frame table anchored at O_i - i * A, text after it at
    p - (i + 1) * A, A = s^2 - s + 2) on well-spaced frames for several s;
  * two hand-worked prompts at s = 2, one with a frame cut short by the next
    marker;
  * invariants: every frame's rows tile its s x s grid, text after a frame
    resumes one past the frame's largest coordinate, T never decreases, and
    the returned (start, amount) places every later text token at p - amount.
"""
import numpy as np
import pytest

import oracle
from tests.helpers import golden_rows
from vlm_decoder_positional_b200 import inputs

MARK = inputs.IMAGE_TOKEN_ID


def frame_len(s):
    return s * s + 3


def shift(s):
    return s * s - s + 2


def closed_form(length, origins, s):
    """Planes of a prompt whose frames start at `origins`, at least
    frame_len(s) apart: frame i is the one-frame table at its own origin with
    every plane lowered by i * A; text after it sits at p - (i + 1) * A."""
    A = shift(s)
    out = np.zeros((3, length), dtype=np.int64)
    for p in range(length):
        i = max((j for j, o in enumerate(origins) if o <= p), default=-1)
        if i < 0:
            out[:, p] = p
            continue
        d = p - origins[i]
        c = origins[i] - i * A
        if d == 0:
            out[:, p] = (c, c - 1, c - 1)
        elif d <= s * s:
            k = d - 1
            out[:, p] = (c, c + k // s, c + k % s)
        elif d == s * s + 1:
            out[:, p] = (c, c + s, c + s)
        elif d == s * s + 2:
            out[:, p] = (c, c, c)
        else:
            out[:, p] = p - (i + 1) * A
    return out


def one(ids):
    return np.asarray(ids, np.int32), np.array([0, len(ids)], np.int32)


def test_one_frame_at_s8_is_the_golden_canvas_table():
    rows = golden_rows("canvas_O6_80.txt")
    rng = np.random.default_rng(0)
    ids, cu = one(inputs.prompt_ids(rng, 80, 6))
    pos, start, amount = oracle.positions_frames(ids, cu, MARK, 8)
    want = np.array([[int(v) for v in r[1:4]] for r in rows]).T
    np.testing.assert_array_equal(pos, want)
    assert (int(start[0]), int(amount[0])) == (73, 58)


def test_one_frame_at_s8_equals_the_canvas_rule_for_every_origin():
    rng = np.random.default_rng(1)
    prompts = [inputs.prompt_ids(rng, 201, o) for o in range(-1, 101)]
    ids, cu = inputs.pack(prompts)
    want = oracle.positions(ids, cu, MARK)
    got = oracle.positions_frames(ids, cu, MARK, 8)
    for w, g in zip(want, got):
        np.testing.assert_array_equal(g, w)


@pytest.mark.parametrize("s", [1, 2, 3, 8, 16])
def test_spaced_frames_match_the_closed_form(s):
    rng = np.random.default_rng(10 + s)
    F = frame_len(s)
    for count in (1, 2, 5):
        length = count * F + 300
        origins = inputs.spaced_origins(rng, count, 0, length - 1, F)
        ids, cu = one(inputs.prompt_ids_frames(rng, length, origins, s))
        pos, start, amount = oracle.positions_frames(ids, cu, MARK, s)
        np.testing.assert_array_equal(pos, closed_form(length, origins, s))
        assert int(start[0]) == origins[-1] + F
        assert int(amount[0]) == count * shift(s)


def test_hand_worked_two_frames_on_a_2x2_grid():
    # s = 2: a frame is <image>, 4 rows, </image>, "\n" (7 tokens) and the
    # text after it resumes at anchor + 3.  Text at 0, 1; frame at 2 (anchor
    # 2); text at 9, 10 -> 5, 6; frame at 11 (anchor 7); text at 18, 19 -> 10, 11.
    ids = [5, 6, MARK, 1, 1, 1, 1, 2, 3, 7, 8, MARK, 1, 1, 1, 1, 2, 3, 9, 9]
    pos, start, amount = oracle.positions_frames(*one(ids), MARK, 2)
    want = [(0, 0, 0), (1, 1, 1),
            (2, 1, 1), (2, 2, 2), (2, 2, 3), (2, 3, 2), (2, 3, 3), (2, 4, 4), (2, 2, 2),
            (5, 5, 5), (6, 6, 6),
            (7, 6, 6), (7, 7, 7), (7, 7, 8), (7, 8, 7), (7, 8, 8), (7, 9, 9), (7, 7, 7),
            (10, 10, 10), (11, 11, 11)]
    np.testing.assert_array_equal(pos.T, want)
    assert (int(start[0]), int(amount[0])) == (18, 8)  # 18 - 8 = 10


def test_hand_worked_frame_cut_short_by_the_next_marker():
    # s = 2: the frame at 2 has three tokens when the marker at 5 opens the
    # next; the counter still stands at 2 + 3 = 5 after it, so the second
    # frame's anchor is 5 and the text after it (index 12) resumes at 8.
    ids = [1, 1, MARK, 1, 1, MARK, 1, 1, 1, 1, 2, 3, 4]
    pos, start, amount = oracle.positions_frames(*one(ids), MARK, 2)
    want = [(0, 0, 0), (1, 1, 1), (2, 1, 1), (2, 2, 2), (2, 2, 3),
            (5, 4, 4), (5, 5, 5), (5, 5, 6), (5, 6, 5), (5, 6, 6), (5, 7, 7), (5, 5, 5),
            (8, 8, 8)]
    np.testing.assert_array_equal(pos.T, want)
    assert (int(start[0]), int(amount[0])) == (12, 4)


@pytest.mark.parametrize("s", [2, 8, 16])
def test_rows_tile_the_grid_and_text_resumes_past_the_frame(s):
    rng = np.random.default_rng(20 + s)
    F = frame_len(s)
    length = 4 * F + 200
    origins = inputs.spaced_origins(rng, 4, 0, length - F - 1, F + 1)
    ids, cu = one(inputs.prompt_ids_frames(rng, length, origins, s))
    pos, _, _ = oracle.positions_frames(ids, cu, MARK, s)
    for o in origins:
        t = pos[0, o]
        rows = pos[:, o + 1:o + 1 + s * s]
        assert (rows[0] == t).all()
        cells = set(zip((rows[1] - t).tolist(), (rows[2] - t).tolist()))
        assert cells == {(r, c) for r in range(s) for c in range(s)}
        assert tuple(pos[:, o]) == (t, t - 1, t - 1)
        assert tuple(pos[:, o + s * s + 1]) == (t, t + s, t + s)
        frame_max = pos[:, o:o + F].max()
        assert frame_max == t + s
        assert tuple(pos[:, o + F]) == (frame_max + 1,) * 3  # 9 = max(H, W) + 1 at s = 8


def test_t_never_decreases_even_with_crowded_markers():
    rng = np.random.default_rng(30)
    for s in (1, 2, 3, 8):
        ids = inputs.text_ids(rng, 3000)
        ids[rng.choice(3000, size=200, replace=False)] = MARK
        pos, _, _ = oracle.positions_frames(*one(ids), MARK, s)
        assert (np.diff(pos[0]) >= 0).all()
        assert pos[0, 0] == 0


def test_state_places_later_text_at_p_minus_amount():
    # appending text to a prompt: the new tokens' planes are p - amount under
    # the state the shorter prompt returned
    rng = np.random.default_rng(40)
    for s in (2, 8, 16):
        F = frame_len(s)
        origins = inputs.spaced_origins(rng, 3, 0, 3 * F + 100, F)
        longer = inputs.prompt_ids_frames(rng, origins[-1] + F + 400, origins, s)
        cut = origins[-1] + F + 37
        _, start, amount = oracle.positions_frames(*one(longer[:cut]), MARK, s)
        pos, _, _ = oracle.positions_frames(*one(longer), MARK, s)
        p = np.arange(int(start[0]), longer.shape[0])
        for r in range(3):
            np.testing.assert_array_equal(pos[r, p], p - int(amount[0]))


def test_text_only_and_packed_batches():
    rng = np.random.default_rng(50)
    prompts, per = [], []
    for i in range(12):
        length = int(rng.integers(0, 700))
        count = int(rng.integers(0, 4))
        s = 8
        origins = (inputs.spaced_origins(rng, count, 0, max(0, length - 1), frame_len(s))
                   if count and length > count * frame_len(s) else [])
        prompts.append(inputs.prompt_ids_frames(rng, length, origins, s))
    ids, cu = inputs.pack(prompts)
    pos, start, amount = oracle.positions_frames(ids, cu, MARK, 8)
    for b, pr in enumerate(prompts):
        p1, s1, a1 = oracle.positions_frames(*one(pr), MARK, 8)
        np.testing.assert_array_equal(pos[:, cu[b]:cu[b + 1]], p1)
        assert (start[b], amount[b]) == (s1[0], a1[0])
        if not (pr == MARK).any():
            np.testing.assert_array_equal(p1, np.tile(np.arange(pr.shape[0]), (3, 1)))
            assert (int(s1[0]), int(a1[0])) == (oracle.TEXT_ONLY_START, 0)


def test_second_frame_separates_the_rules():
    # the canvas rule treats a later marker as an ordinary token; the
    # multi-frame reading opens a frame there: they agree up to it, differ after
    rng = np.random.default_rng(60)
    ids, cu = one(inputs.prompt_ids_frames(rng, 400, [10, 150], 8))
    a, _, _ = oracle.positions(ids, cu, MARK)
    b, _, _ = oracle.positions_frames(ids, cu, MARK, 8)
    np.testing.assert_array_equal(a[:, :150], b[:, :150])
    assert (a[:, 150:] != b[:, 150:]).any(axis=0).all()


def test_rejects_bad_grid_sides():
    ids, cu = one([1, 2, 3])
    for s in (0, -1, 129):
        with pytest.raises(oracle.OracleError):
            oracle.positions_frames(ids, cu, MARK, s)
