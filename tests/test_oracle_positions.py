"""Pins for the oracle's position planes (CPU only).

Each test ties the oracle to something other than itself: the pages' worked
values (golden files), the structure of the 8x8 grid, the text-only special
case, the red arms that the pages report as failing, and a brute-force
comparison with a segment-by-segment construction of the canvas.
"""
import numpy as np
import pytest

import oracle
from tests.helpers import golden_rows
from vlm_decoder_positional_b200 import inputs

MARK = inputs.IMAGE_TOKEN_ID
TEXT_ONLY_START = 2 ** 30


def one_prompt(length, origin, seed=7, row_ids="v_plus_k"):
    rng = np.random.default_rng(seed)
    ids = inputs.prompt_ids(rng, length, origin, row_ids)
    return ids, np.array([0, length], dtype=np.int32)


def test_golden_o6_table_matches_config_1():
    wl = inputs.make_config(1, with_qk=False)
    pos, start, amount = oracle.positions(wl.ids, wl.cu_seqlens, MARK)
    want = np.array([[int(v) for v in r] for r in golden_rows("canvas_O6_80.txt")])
    assert want.shape == (80, 4) and (want[:, 0] == np.arange(80)).all()
    np.testing.assert_array_equal(pos.T, want[:, 1:])
    assert (int(start[0]), int(amount[0])) == (73, 58)


@pytest.mark.parametrize("row", golden_rows("shift_worked.txt"))
def test_worked_shift_values(row):
    O, want_start, want_amount, first_after = (int(v) for v in row)
    ids, cu = one_prompt(O + 120, O)
    pos, start, amount = oracle.positions(ids, cu, MARK)
    assert int(start[0]) == want_start and int(amount[0]) == want_amount
    assert pos[:, want_start].tolist() == [first_after] * 3
    # the first text token after the frame sits at O + 9 (9 = max(H, W) + 1)
    assert first_after == O + 9


@pytest.mark.parametrize("O", [0, 1, 6, 17, 40, 3000])
def test_rows_tile_the_8x8_grid_row_major(O):
    ids, cu = one_prompt(O + 80, O)
    pos, _, _ = oracle.positions(ids, cu, MARK)
    rows = pos[:, O + 1:O + 65]
    assert (rows[0] == O).all()
    cells = list(zip((rows[1] - O).tolist(), (rows[2] - O).tolist()))
    assert cells == [(r, c) for r in range(8) for c in range(8)]


@pytest.mark.parametrize("O", [0, 5, 33])
def test_frame_ranges_and_monotone_tail(O):
    n = O + 300
    ids, cu = one_prompt(n, O)
    pos, start, amount = oracle.positions(ids, cu, MARK)
    frame = pos[:, O:O + 67]
    assert (frame[0] == O).all()
    assert frame[1:].min() == O - 1 and frame[1:].max() == O + 8
    tail = pos[:, int(start[0]):]
    assert (tail[0] == tail[1]).all() and (tail[1] == tail[2]).all()
    assert (np.diff(tail[0]) == 1).all()
    assert (pos[0] <= np.arange(n)).all()


def test_text_only_is_one_dimensional():
    ids, cu = one_prompt(500, -1)
    assert not (ids == MARK).any()
    pos, start, amount = oracle.positions(ids, cu, MARK)
    assert int(start[0]) == TEXT_ONLY_START and int(amount[0]) == 0
    for r in range(3):
        np.testing.assert_array_equal(pos[r], np.arange(500))


def canvas_by_segments(ids, marker):
    """Independent construction: text advances a running counter on all three
    planes; the first <image> lays the 67-token frame on a canvas anchored at
    the counter; text after the frame resumes one past the largest coordinate
    the canvas used (the pages' 9 = max(H, W) + 1)."""
    out, nxt, i, seen = [], 0, 0, False
    n = len(ids)
    while i < n:
        if ids[i] == marker and not seen:
            seen = True
            o = nxt
            frame = ([(o, o - 1, o - 1)]
                     + [(o, o + r, o + c) for r in range(8) for c in range(8)]
                     + [(o, o + 8, o + 8), (o, o, o)])
            take = min(len(frame), n - i)
            out += frame[:take]
            i += take
            nxt = max(max(v) for v in frame) + 1
        else:
            out.append((nxt, nxt, nxt))
            nxt += 1
            i += 1
    return np.array(out, dtype=np.int64).T.reshape(3, n)


def test_brute_force_every_origin_and_position():
    rng = np.random.default_rng(3)
    prompts, origins = [], list(range(0, 101))
    for O in origins:
        prompts.append(inputs.prompt_ids(rng, 201, O))
    ids, cu = inputs.pack(prompts)
    pos, start, amount = oracle.positions(ids, cu, MARK)
    for b, O in enumerate(origins):
        seg = ids[cu[b]:cu[b + 1]]
        want = canvas_by_segments(seg.tolist(), MARK)
        np.testing.assert_array_equal(pos[:, cu[b]:cu[b + 1]], want, err_msg=f"O={O}")
        assert (int(start[b]), int(amount[b])) == (O + 67, 58)


def test_first_marker_wins_and_later_markers_are_text():
    ids, cu = one_prompt(400, 10)
    ids[200] = MARK
    pos, start, amount = oracle.positions(ids, cu, MARK)
    assert int(start[0]) == 77
    assert pos[:, 200].tolist() == [200 - 58] * 3
    want = canvas_by_segments(ids.tolist(), MARK)
    np.testing.assert_array_equal(pos, want)


def test_truncated_frame_and_origin_zero():
    ids, cu = one_prompt(40, 0)
    pos, start, amount = oracle.positions(ids, cu, MARK)
    assert pos[:, 0].tolist() == [0, -1, -1]
    assert (int(start[0]), int(amount[0])) == (67, 58)
    np.testing.assert_array_equal(pos, canvas_by_segments(ids.tolist(), MARK))


def test_pad_row_ids_give_the_same_planes():
    a, cu = one_prompt(150, 12, row_ids="v_plus_k")
    b, _ = one_prompt(150, 12, row_ids="pad")
    assert (a != b).any()
    np.testing.assert_array_equal(oracle.positions(a, cu, MARK)[0],
                                  oracle.positions(b, cu, MARK)[0])


def test_packed_batch_with_empty_sequences_is_per_sequence():
    rng = np.random.default_rng(11)
    lens, origins = [0, 90, 0, 130, 1, 70], [-1, 3, -1, -1, -1, 0]
    prompts = [inputs.prompt_ids(rng, n, o) for n, o in zip(lens, origins)]
    ids, cu = inputs.pack(prompts)
    pos, start, amount = oracle.positions(ids, cu, MARK)
    for b, p in enumerate(prompts):
        pb, sb, ab = oracle.positions(p, np.array([0, len(p)], np.int32), MARK)
        np.testing.assert_array_equal(pos[:, cu[b]:cu[b + 1]], pb)
        assert (start[b], amount[b]) == (sb[0], ab[0])


def test_malformed_cu_seqlens_rejected():
    ids = np.zeros(10, np.int32)
    for cu in ([0, 5, 4, 10], [1, 10], [0, 9]):
        with pytest.raises(oracle.OracleError):
            oracle.positions(ids, np.array(cu, np.int32), MARK)


@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_red_arms_fail_on_every_image_prompt(cfg):
    # The pages' negative controls, the amount + 1 arm and the 1-D planes arm,
    # must give different planes; on text-only prompts every arm agrees.
    wl = inputs.make_config(cfg, with_qk=False)
    green = oracle.positions(wl.ids, wl.cu_seqlens, MARK)[0]
    plus1 = oracle.positions(wl.ids, wl.cu_seqlens, MARK, rule="amount+1")[0]
    flat = oracle.positions(wl.ids, wl.cu_seqlens, MARK, rule="planes_1d")[0]
    cu = wl.cu_seqlens
    for b in range(wl.num_seqs):
        s = slice(cu[b], cu[b + 1])
        O = int(wl.frame_origin[b])
        if O < 0:
            assert (green[:, s] == plus1[:, s]).all() and (green[:, s] == flat[:, s]).all()
            continue
        assert (green[:, s] != flat[:, s]).any()
        assert (green[:, s] != plus1[:, s]).any()
        # only the text before the frame still matches under amount + 1: the
        # graph derives the origin from (start, amount), so the frame moves too
        pre = slice(cu[b], cu[b] + max(O - 1, 0))
        assert (green[:, pre] == plus1[:, pre]).all()
        rest = slice(cu[b] + max(O - 1, 0), cu[b + 1])
        assert (green[:, rest] != plus1[:, rest]).any(axis=0).all()


def test_step_form_reproduces_the_prompt_planes():
    # cmr_positions_step receives only (p, start, amount); it must give the
    # same planes as the prompt rule at every index of an image prompt and of
    # a text-only prompt, and p - amount for every token after the frame.
    rng = np.random.default_rng(5)
    prompts = [inputs.prompt_ids(rng, 300, 6), inputs.prompt_ids(rng, 300, 17),
               inputs.prompt_ids(rng, 300, -1), inputs.prompt_ids(rng, 300, 0)]
    ids, cu = inputs.pack(prompts)
    pos, start, amount = oracle.positions(ids, cu, MARK)
    for b in range(len(prompts)):
        n = 300
        p = np.arange(n, dtype=np.int32)
        step = oracle.positions_step(p, np.full(n, start[b]), np.full(n, amount[b]))
        np.testing.assert_array_equal(step, pos[:, cu[b]:cu[b + 1]])
    # generated tokens (p beyond the prompt) sit at p - 58 on all three planes
    gen = np.arange(300, 400, dtype=np.int32)
    step = oracle.positions_step(gen, np.full(100, start[0]), np.full(100, amount[0]))
    assert (step == gen - 58).all()


def test_decode_config_positions():
    wl = inputs.make_config(4, with_qk=False)
    _, start, amount = oracle.positions(wl.ids, wl.cu_seqlens, MARK)
    assert (amount == 58).all() and (start == wl.frame_origin + 67).all()
    step = oracle.positions_step(wl.cache_len, start, amount)
    assert (step == wl.cache_len - 58).all()


# ---------------------------------------------------------------------------
# chunked prefill, later turns and the rule variants
# ---------------------------------------------------------------------------

def run_in_chunks(ids, cuts, rule="canvas"):
    """Feed one prompt to the chunked form in pieces, carrying the state."""
    start = np.array([oracle.TEXT_ONLY_START], np.int32)
    amount = np.array([0], np.int32)
    out = []
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        pos, start, amount = oracle.positions_chunk(ids[lo:hi], np.array([0, hi - lo], np.int32),
                                                    MARK, rule, np.array([lo], np.int32),
                                                    start, amount)
        out.append(pos)
    return np.concatenate(out, axis=1), int(start[0]), int(amount[0])


@pytest.mark.parametrize("O", [-1, 0, 6, 17, 40, 100])
@pytest.mark.parametrize("chunk", [1, 16, 23, 67, 1000])
def test_chunked_prefill_reproduces_the_whole_prompt(O, chunk):
    # The port notes' S = 16 prefill answers as the one-token order: splitting
    # a prompt anywhere (inside the frame too) must not change a plane.
    ids, cu = one_prompt(300, O)
    whole, start, amount = oracle.positions(ids, cu, MARK)
    cuts = list(range(0, 300, chunk)) + [300]
    got, s, a = run_in_chunks(ids, cuts)
    np.testing.assert_array_equal(got, whole)
    assert (s, a) == (int(start[0]), int(amount[0]))


def test_second_turn_continues_the_kept_state():
    # A second question on the same image: turn 2's ids are appended to turn 1's
    # conversation and prefilled from the kept state (port notes, "Prefill in
    # chunks and a second turn"); the planes equal those of the whole conversation.
    rng = np.random.default_rng(21)
    turn1 = inputs.prompt_ids(rng, 88, 6)
    answer = inputs.text_ids(rng, 33)
    turn2 = inputs.text_ids(rng, 20)
    conv = np.concatenate([turn1, answer, turn2])
    whole, _, _ = oracle.positions(conv, np.array([0, conv.size], np.int32), MARK)
    got, s, a = run_in_chunks(conv, [0, 88, 121, conv.size])
    np.testing.assert_array_equal(got, whole)
    assert (s, a) == (73, 58)
    assert whole[:, -1].tolist() == [conv.size - 1 - 58] * 3


def test_chunked_batch_matches_per_sequence_chunks():
    rng = np.random.default_rng(22)
    n_seq = 7
    prompts = [inputs.prompt_ids(rng, 200, o) for o in (3, -1, 0, 50, 120, 190, -1)]
    offsets = np.array([0, 0, 17, 40, 100, 150, 199], np.int32)
    states = []
    for p, off in zip(prompts, offsets):
        _, s, a = oracle.positions_chunk(p[:off], np.array([0, off], np.int32), MARK)
        states.append((s[0], a[0]))
    tails = [p[off:] for p, off in zip(prompts, offsets)]
    ids, cu = inputs.pack(tails)
    st = np.array([s for s, _ in states], np.int32)
    am = np.array([a for _, a in states], np.int32)
    pos, s_out, a_out = oracle.positions_chunk(ids, cu, MARK, "canvas", offsets, st, am)
    for b in range(n_seq):
        whole, ws, wa = oracle.positions(prompts[b], np.array([0, 200], np.int32), MARK)
        np.testing.assert_array_equal(pos[:, cu[b]:cu[b + 1]], whole[:, offsets[b]:])
        assert (s_out[b], a_out[b]) == (ws[0], wa[0])


def test_qwen_vl_rule_shift_values():
    # CoreAIKit section of the port notes: the canvas shifts from where the pads
    # begin + 66 by 58; Qwen-VL's rule would give + 64 and 56.
    for O in (6, 17):
        ids, cu = one_prompt(O + 120, O)
        pads_begin = O + 1
        _, s, a = oracle.positions_chunk(ids, cu, MARK, "canvas")
        assert (int(s[0]), int(a[0])) == (pads_begin + 66, 58)
        pos, s, a = oracle.positions_chunk(ids, cu, MARK, "qwen_vl")
        assert (int(s[0]), int(a[0])) == (pads_begin + 64, 56)
        # </image> and "\n" now count as text after the frame, which resumes at O + 9
        assert pos[:, O + 65].tolist() == [O + 9] * 3
        assert pos[:, O + 66].tolist() == [O + 10] * 3
        canvas, _, _ = oracle.positions(ids, cu, MARK)
        np.testing.assert_array_equal(pos[:, :O + 65], canvas[:, :O + 65])


def test_planes_1d_rule_is_plain_positions():
    ids, cu = one_prompt(150, 10)
    pos, s, a = oracle.positions_chunk(ids, cu, MARK, "planes_1d", np.array([1000], np.int32))
    assert (int(s[0]), int(a[0])) == (2 ** 30, 0)
    for r in range(3):
        np.testing.assert_array_equal(pos[r], 1000 + np.arange(150))


def test_chunk_form_at_offset_zero_is_the_prompt_form():
    wl = inputs.make_config(2, with_qk=False)
    a = oracle.positions(wl.ids, wl.cu_seqlens, MARK)
    b = oracle.positions_chunk(wl.ids, wl.cu_seqlens, MARK)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
