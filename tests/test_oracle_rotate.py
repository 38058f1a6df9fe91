"""Pins for the oracle's frequency map, rotation and bf16 rounding (CPU only).

The rotation is checked against an independent textbook formulation (a complex
multiplication by e^{i*angle}), closed forms for single frequencies, and the
group properties of plane rotations.  The bf16 rounding is checked against
torch's float32 -> bf16 conversion where no double rounding can occur, and by
hand-worked ties, subnormals and overflow.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import golden_rows

THETA, SECTIONS, ROT = 1e7, (11, 11, 10), 64


def rand_bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)
    return x.view(torch.int16).numpy().view(np.uint16)


def golden_map():
    rows = golden_rows("freq_planes_11_11_10.txt")
    letter = {"T": 0, "H": 1, "W": 2}
    assert [int(r[0]) for r in rows] == list(range(32))
    return np.array([letter[r[1]] for r in rows])


def test_frequency_map_matches_golden_and_counts():
    plane = oracle.freq_planes(ROT, SECTIONS)
    np.testing.assert_array_equal(plane, golden_map())
    assert np.bincount(plane, minlength=3).tolist() == [11, 11, 10]


@pytest.mark.parametrize("rot,sec", [(64, (12, 11, 10)), (64, (0, 20, 12)), (64, (8, 12, 12)),
                                     (64, (-1, 22, 11))])
def test_frequency_map_rejects_sections_it_cannot_realise(rot, sec):
    with pytest.raises(oracle.OracleError):
        oracle.freq_planes(rot, sec)


def test_frequency_map_other_sections():
    # {T, H, W} = {16, 8, 8} over 32 frequencies: the interleave covers j < 24
    plane = oracle.freq_planes(64, (16, 8, 8))
    assert np.bincount(plane, minlength=3).tolist() == [16, 8, 8]
    assert (plane[24:] == 0).all() and plane[1] == 1 and plane[2] == 2


def textbook_rope(x, angle_per_freq):
    """(x_d + i x_{d+half}) * exp(i angle_d) for d < half (rotate-half pairing)."""
    half = angle_per_freq.shape[-1]
    z = (x[..., :half] + 1j * x[..., half:2 * half]) * np.exp(1j * angle_per_freq)
    y = x.copy()
    y[..., :half] = z.real
    y[..., half:2 * half] = z.imag
    return y


def inv_freq_closed_form(rot):
    # theta^(-2j/rot) written as a power of ten: theta = 1e7
    return 10.0 ** (-7.0 * 2.0 * np.arange(rot // 2) / rot)


def test_text_only_rotation_is_textbook_1d_rope():
    n, h, d = 50, 3, 256
    x = rand_bf16((1, n, h, d), 1)
    p = np.arange(n, dtype=np.int32) * 661 - 300   # includes negatives and > 3e4
    pos = np.stack([p, p, p])
    _, f64 = oracle.rotate_bf16(x, pos, THETA, SECTIONS, ROT, return_f64=True)
    xd = oracle.bf16_to_f64(x)
    ang = p[:, None].astype(np.float64) * inv_freq_closed_form(ROT)[None, :]
    want = textbook_rope(xd, ang[None, :, None, :])
    np.testing.assert_allclose(f64[..., :ROT], want[..., :ROT], rtol=0, atol=1e-9)


def test_mrope_uses_the_plane_of_each_frequency():
    n, h, d = 40, 2, 128
    rng = np.random.default_rng(2)
    pos = rng.integers(-5, 40000, size=(3, n)).astype(np.int32)
    x = np.random.default_rng(4).standard_normal((1, n, h, d))
    got = oracle.rotate_f64(x, pos, THETA, SECTIONS, ROT)
    plane = golden_map()
    ang = pos[plane, :].T.astype(np.float64) * inv_freq_closed_form(ROT)[None, :]
    want = textbook_rope(x, ang[None, :, None, :])
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-9)


def test_single_frequency_closed_forms():
    # unit vector on pair j at position p: output = (cos(p w_j), sin(p w_j))
    n = 3
    pos = np.tile(np.array([1, 1000, 32767], dtype=np.int32), (3, 1))
    for j, w in [(0, 1.0), (16, 1.0 / np.sqrt(1e7)), (31, 1e7 ** (-62.0 / 64.0))]:
        x = np.zeros((1, n, 1, 64))
        x[..., j] = 1.0
        y = oracle.rotate_f64(x, pos, THETA, SECTIONS, ROT)
        a = pos[0].astype(np.float64) * w
        np.testing.assert_allclose(y[0, :, 0, j], np.cos(a), atol=1e-12)
        np.testing.assert_allclose(y[0, :, 0, j + 32], np.sin(a), atol=1e-12)


def test_position_zero_is_identity_and_tail_dims_untouched():
    x = rand_bf16((2, 16, 4, 256), 3, scale=50.0)
    pos = np.zeros((3, 16), np.int32)
    np.testing.assert_array_equal(oracle.rotate_bf16(x, pos), x)
    pos = np.random.default_rng(0).integers(0, 9000, size=(3, 16)).astype(np.int32)
    y = oracle.rotate_bf16(x, pos)
    np.testing.assert_array_equal(y[..., 64:], x[..., 64:])
    assert (y[..., :64] != x[..., :64]).any()


def test_rotation_preserves_pair_norms_and_inverts():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((2, 30, 3, 96)) * 10
    pos = rng.integers(-100, 33000, size=(3, 30)).astype(np.int32)
    y = oracle.rotate_f64(x, pos, THETA, SECTIONS, ROT)
    n_in = x[..., :32] ** 2 + x[..., 32:64] ** 2
    n_out = y[..., :32] ** 2 + y[..., 32:64] ** 2
    np.testing.assert_allclose(n_out, n_in, rtol=1e-12)
    back = oracle.rotate_f64(y, -pos, THETA, SECTIONS, ROT)
    np.testing.assert_allclose(back, x, rtol=0, atol=1e-10)
    np.testing.assert_array_equal(y[..., 64:], x[..., 64:])


def test_rotation_composes_additively():
    rng = np.random.default_rng(10)
    x = rng.standard_normal((1, 20, 2, 64))
    a = rng.integers(-2000, 2000, size=(3, 20)).astype(np.int32)
    b = rng.integers(-2000, 2000, size=(3, 20)).astype(np.int32)
    ab = oracle.rotate_f64(oracle.rotate_f64(x, a), b)
    np.testing.assert_allclose(ab, oracle.rotate_f64(x, a + b), atol=1e-11)


def test_layers_and_heads_share_positions():
    x = rand_bf16((3, 8, 5, 64), 12)
    pos = np.random.default_rng(1).integers(0, 5000, size=(3, 8)).astype(np.int32)
    full = oracle.rotate_bf16(x, pos)
    for l in range(3):
        for h in range(5):
            one = oracle.rotate_bf16(x[l:l + 1, :, h:h + 1], pos)
            np.testing.assert_array_equal(full[l:l + 1, :, h:h + 1], one)


def test_bf16_decode_known_patterns():
    bits = np.array([0x3F80, 0xC000, 0x0001, 0x7F7F, 0x8000, 0x4049], np.uint16)
    want = [1.0, -2.0, 2.0 ** -133, (2 - 2 ** -7) * 2.0 ** 127, -0.0, 3.140625]
    got = oracle.bf16_to_f64(bits)
    assert got.tolist() == want
    assert np.signbit(got[4])


def test_bf16_rounding_matches_torch_on_float32_values():
    g = torch.Generator().manual_seed(0)
    f = torch.cat([torch.randn(4000, generator=g) * s for s in (1e-3, 1.0, 100.0, 1e30)])
    f = torch.cat([f, torch.tensor([1.00390625, 1.01171875, -1.00390625, 0.0, -0.0])])
    want = f.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.f64_to_bf16(f.double().numpy())
    np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("x,bits", [
    (1.0 + 2.0 ** -8, 0x3F80),                    # tie -> even (down)
    (1.0 + 3 * 2.0 ** -8, 0x3F82),                # tie -> even (up)
    (1.0 + 2.0 ** -8 + 2.0 ** -40, 0x3F81),       # just above the tie: rounds up
    (-(1.0 + 2.0 ** -8 + 2.0 ** -40), 0xBF81),    # (a float32 detour would give 1.0)
    (2.0 ** -134, 0x0000),                         # half the least subnormal: tie -> 0
    (3 * 2.0 ** -134, 0x0002),                     # 1.5 subnormal units: tie -> even
    (2.0 ** -126 * (1 - 2.0 ** -9), 0x0080),       # rounds up into the normal range
    ((2 - 2.0 ** -8 + 2.0 ** -30) * 2.0 ** 127, 0x7F80),  # above max + half ulp -> inf
    ((2 - 2.0 ** -8) * 2.0 ** 127, 0x7F80),        # the tie at max rounds to 2^128 = inf
    ((2 - 2.0 ** -8 - 2.0 ** -30) * 2.0 ** 127, 0x7F7F),  # below the tie -> max
    (-0.0, 0x8000),
])
def test_bf16_direct_rounding_cases(x, bits):
    assert int(oracle.f64_to_bf16(np.array([x]))[0]) == bits


def test_bf16_output_is_correctly_rounded_f64():
    x = rand_bf16((1, 64, 2, 64), 5, scale=300.0)
    pos = np.random.default_rng(8).integers(0, 30000, size=(3, 64)).astype(np.int32)
    y, f64 = oracle.rotate_bf16(x, pos, return_f64=True)
    np.testing.assert_array_equal(y[..., :64], oracle.f64_to_bf16(f64[..., :64]))


def test_cache_form_places_rotated_rows_at_each_tokens_index():
    # the cache form composes the pinned pieces: planes of the decode form at
    # the token's index, the pinned rotation, and a placement at [l, slot, h, p]
    L, n, hk, D = 2, 9, 2, 128
    q = rand_bf16((L, n, 3, D), 30)
    k = rand_bf16((L, n, hk, D), 31)
    v = rand_bf16((L, n, hk, D), 32)
    cu = np.array([0, 4, 4, 9], np.int32)               # an empty middle sequence
    off = np.array([70, 0, 3], np.int32)
    start = np.array([73, 1 << 30, 10], np.int32)
    amount = np.array([58, 0, 1], np.int32)
    slot = np.array([2, 0, 1], np.int32)
    kc0 = np.full((L, 3, hk, 8, D), 0x7F7F, np.uint16)
    vc0 = np.full((L, 3, hk, 8, D), 0x7F7F, np.uint16)
    qo, kc, vc, status = oracle.rotate_qk_cache(q, k, v, start, amount, kc0, vc0, cu, off, slot)
    assert status == 2                                  # sequence 0 sits at 70..73 > ctx 8
    p = np.array([70, 71, 72, 73, 3, 4, 5, 6, 7])
    b = np.array([0, 0, 0, 0, 2, 2, 2, 2, 2])
    pos = oracle.positions_step(p, start[b], amount[b])
    np.testing.assert_array_equal(qo, oracle.rotate_bf16(q, pos))
    kr = oracle.rotate_bf16(k, pos)
    written = np.zeros(kc0.shape[:4], bool)
    for t in range(4, 9):
        np.testing.assert_array_equal(kc[:, 1, :, p[t]], kr[:, t])
        np.testing.assert_array_equal(vc[:, 1, :, p[t]], v[:, t])
        written[:, 1, :, p[t]] = True
    assert (kc[~written] == 0x7F7F).all() and (vc[~written] == 0x7F7F).all()
