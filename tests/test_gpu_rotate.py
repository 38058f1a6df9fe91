"""GPU parity of the fused cos/sin + rotate kernel, through the C ABI.

Rotated dims: within 2 bf16 ulps or 1e-2 of the oracle's correctly rounded
fp64 result.  Dims past rot_dim: bit-exact (never written).  Every element is
compared; the 64 x 4096 and 6 x 32 x 8192 workloads are covered element by
element by test_gpu_accuracy.py (pos form) and test_gpu_full_parity.py (the
other forms)."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import assert_bf16_close, ulp_stats
from vlm_decoder_positional_b200 import cmr, inputs

pytestmark = pytest.mark.gpu


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def planes_for(wl, dev):
    ids = torch.from_numpy(wl.ids).to(dev)
    cu = torch.from_numpy(wl.cu_seqlens).to(dev)
    pos, start, amount = cmr.positions(ids, cu, wl.image_token_id)
    if wl.cache_len is not None:
        pos = cmr.positions_step(torch.from_numpy(wl.cache_len).to(dev), start, amount)
    return pos


def check_full(q, k, pos, theta=1e7, sections=(11, 11, 10), rot_dim=64, what=""):
    """Rotate on the GPU and compare every element with the oracle."""
    q_in = bits(q) if q is not None else None
    k_in = bits(k) if k is not None else None
    cmr.rotate_qk(q, k, pos, theta, sections, rot_dim)
    torch.cuda.synchronize()
    p = pos.cpu().numpy()
    worst = (0, 0.0)
    for name, t_in, t in (("q", q_in, q), ("k", k_in, k)):
        if t is None:
            continue
        t_in4 = t_in.reshape((1,) + t_in.shape) if t_in.ndim == 3 else t_in
        want = oracle.rotate_bf16(t_in4, p, theta, sections, rot_dim).reshape(t_in.shape)
        got = bits(t)
        np.testing.assert_array_equal(got[..., rot_dim:], t_in[..., rot_dim:])
        assert_bf16_close(got[..., :rot_dim], want[..., :rot_dim], f"{what} {name}")
        u, d = ulp_stats(got, want)
        worst = (max(worst[0], u), max(worst[1], d))
    return worst


@pytest.mark.parametrize("cfg", [1, 2, 4])
def test_rotate_full_compare_small_workloads(cuda_device, cfg):
    wl = inputs.make_config(cfg, device=cuda_device)
    pos = planes_for(wl, cuda_device)
    check_full(wl.q, wl.k, pos, what=wl.name)


@pytest.mark.parametrize("n", [1, 2, 7, 8, 9, 63, 64, 65, 1001])
@pytest.mark.parametrize("layers", [1, 2, 3, 5, 6, 7, 9])
def test_rotate_ragged_tokens_and_layer_counts(cuda_device, n, layers):
    g = torch.Generator(device=cuda_device).manual_seed(n * 31 + layers)
    q = torch.randn((layers, n, 8, 256), generator=g, device=cuda_device).to(torch.bfloat16)
    k = torch.randn((layers, n, 2, 256), generator=g, device=cuda_device).to(torch.bfloat16)
    pos = torch.randint(-70, 40000, (3, n), generator=g, device=cuda_device, dtype=torch.int32)
    check_full(q, k, pos, what=f"n={n} L={layers}")


@pytest.mark.parametrize("hq,hk,head_dim,rot_dim,sections", [
    (16, 4, 256, 64, (11, 11, 10)),
    (1, 0, 256, 64, (11, 11, 10)),
    (0, 3, 128, 64, (16, 8, 8)),
    (8, 2, 256, 16, (3, 3, 2)),
    (8, 2, 256, 32, (6, 5, 5)),
    (8, 2, 128, 128, (22, 21, 21)),
    (4, 4, 256, 256, (44, 42, 42)),
    (2, 1, 64, 48, (8, 8, 8)),
    (64, 64, 256, 64, (11, 11, 10)),
])
def test_rotate_other_shapes(cuda_device, hq, hk, head_dim, rot_dim, sections):
    g = torch.Generator(device=cuda_device).manual_seed(hq * 100 + hk + rot_dim)
    n, L = 77, 2
    q = (torch.randn((L, n, hq, head_dim), generator=g, device=cuda_device).to(torch.bfloat16)
         if hq else None)
    k = (torch.randn((L, n, hk, head_dim), generator=g, device=cuda_device).to(torch.bfloat16)
         if hk else None)
    pos = torch.randint(0, 30000, (3, n), generator=g, device=cuda_device, dtype=torch.int32)
    check_full(q, k, pos, 1e7, sections, rot_dim, what=f"{hq},{hk},{head_dim},{rot_dim}")


@pytest.mark.parametrize("theta", [1e4, 1e6, 5e8])
def test_rotate_other_theta_and_extreme_positions(cuda_device, theta):
    g = torch.Generator(device=cuda_device).manual_seed(17)
    n = 300
    q = (torch.randn((1, n, 8, 256), generator=g, device=cuda_device) * 30).to(torch.bfloat16)
    k = (torch.randn((1, n, 2, 256), generator=g, device=cuda_device) * 30).to(torch.bfloat16)
    pos = torch.randint(-(2 ** 30), 2 ** 30, (3, n), generator=g, device=cuda_device,
                        dtype=torch.int32)
    pos[:, :3] = torch.tensor([0, 2 ** 31 - 1, -(2 ** 31)], dtype=torch.int32)
    check_full(q, k, pos, theta, what=f"theta={theta}")


def test_text_only_planes_equal_plain_rope(cuda_device):
    # all three planes equal p: the GPU result must match the oracle, which
    # the CPU pins tie to textbook 1-D rotate-half RoPE
    n = 4096
    g = torch.Generator(device=cuda_device).manual_seed(3)
    q = torch.randn((1, n, 8, 256), generator=g, device=cuda_device).to(torch.bfloat16)
    k = torch.randn((1, n, 2, 256), generator=g, device=cuda_device).to(torch.bfloat16)
    p = torch.arange(n, dtype=torch.int32, device=cuda_device)
    check_full(q, k, torch.stack([p, p, p]), what="text-only")


def test_position_zero_leaves_bits_unchanged(cuda_device):
    g = torch.Generator(device=cuda_device).manual_seed(4)
    q = (torch.randn((2, 50, 8, 256), generator=g, device=cuda_device) * 100).to(torch.bfloat16)
    k = (torch.randn((2, 50, 2, 256), generator=g, device=cuda_device) * 100).to(torch.bfloat16)
    q0, k0 = q.clone(), k.clone()
    cmr.rotate_qk(q, k, torch.zeros((3, 50), dtype=torch.int32, device=cuda_device))
    torch.cuda.synchronize()
    assert torch.equal(q.view(torch.int16), q0.view(torch.int16))
    assert torch.equal(k.view(torch.int16), k0.view(torch.int16))


def test_three_dim_views_and_stream_argument(cuda_device):
    n = 333
    g = torch.Generator(device=cuda_device).manual_seed(5)
    q = torch.randn((n, 8, 256), generator=g, device=cuda_device).to(torch.bfloat16)
    k = torch.randn((n, 2, 256), generator=g, device=cuda_device).to(torch.bfloat16)
    pos = torch.randint(0, 9000, (3, n), generator=g, device=cuda_device, dtype=torch.int32)
    q_in, k_in = bits(q), bits(k)
    s = torch.cuda.Stream(cuda_device)
    s.wait_stream(torch.cuda.current_stream(cuda_device))
    cmr.rotate_qk(q, k, pos, stream=s)
    s.synchronize()
    p = pos.cpu().numpy()
    assert_bf16_close(bits(q)[None], oracle.rotate_bf16(q_in[None], p), "q")
    assert_bf16_close(bits(k)[None], oracle.rotate_bf16(k_in[None], p), "k")


def test_misaligned_and_host_pointers_are_rejected(cuda_device):
    q = torch.zeros((1, 4, 8, 256), dtype=torch.bfloat16, device=cuda_device)
    k = torch.zeros((1, 4, 2, 256), dtype=torch.bfloat16, device=cuda_device)
    pos = torch.zeros((3, 4), dtype=torch.int32, device=cuda_device)
    sec = cmr.ctypes.c_int32 * 3
    L = cmr.lib()
    rc = L.cmr_rotate_qk(q.data_ptr() + 2, k.data_ptr(), pos.data_ptr(), 4, 1, 8, 2, 256, 1e7,
                         sec(11, 11, 10), 64, None, None)
    assert rc == cmr.CMR_EINVAL
    host = np.zeros(4 * 8 * 256, np.uint16)
    rc = L.cmr_rotate_qk(host.ctypes.data, k.data_ptr(), pos.data_ptr(), 4, 1, 8, 2, 256, 1e7,
                         sec(11, 11, 10), 64, None, None)
    assert rc == cmr.CMR_EINVAL


# ---- the TMA-staged kernel (rot_dim 64, from 1024 tiles of 8 tokens) ----

STAGED_MIN_TOKENS = 1024 * 8


@pytest.mark.parametrize("n", [STAGED_MIN_TOKENS, STAGED_MIN_TOKENS + 1, STAGED_MIN_TOKENS + 7,
                               10001])
@pytest.mark.parametrize("layers", [1, 2, 3, 4, 5, 9])
def test_rotate_staged_ragged_tiles_and_ring_wrap(cuda_device, n, layers):
    # tiles of 8 tokens with a ragged last tile; 1 and 2 layers use a ring of
    # that many stages; 4, 5 and 9 layers wrap the 3-stage ring
    assert cmr.rotate_qk_kernel(n, layers, 8, 2) == "rotate_qk_staged_kernel"
    g = torch.Generator(device=cuda_device).manual_seed(n + 100 * layers)
    q = torch.randn((layers, n, 8, 256), generator=g, device=cuda_device).to(torch.bfloat16)
    k = torch.randn((layers, n, 2, 256), generator=g, device=cuda_device).to(torch.bfloat16)
    pos = torch.randint(-70, 400000, (3, n), generator=g, device=cuda_device, dtype=torch.int32)
    check_full(q, k, pos, what=f"staged n={n} L={layers}")


@pytest.mark.parametrize("hq,hk,head_dim", [(16, 4, 256), (1, 0, 256), (0, 3, 128), (8, 2, 64),
                                            (8, 2, 72), (3, 1, 256)])
def test_rotate_staged_other_heads_and_head_dims(cuda_device, hq, hk, head_dim):
    g = torch.Generator(device=cuda_device).manual_seed(hq * 1000 + hk * 10 + head_dim)
    n, L = 9001, 2
    assert cmr.rotate_qk_kernel(n, L, hq, hk, head_dim) == "rotate_qk_staged_kernel"
    q = (torch.randn((L, n, hq, head_dim), generator=g, device=cuda_device).to(torch.bfloat16)
         if hq else None)
    k = (torch.randn((L, n, hk, head_dim), generator=g, device=cuda_device).to(torch.bfloat16)
         if hk else None)
    pos = torch.randint(0, 30000, (3, n), generator=g, device=cuda_device, dtype=torch.int32)
    check_full(q, k, pos, what=f"staged {hq},{hk},{head_dim}")


def test_staged_and_register_kernels_agree_bit_for_bit(cuda_device):
    # the whole batch takes the staged kernel; the same rows rotated 512
    # tokens at a time take the register kernel: identical bits
    n, L = 20000, 6
    g = torch.Generator(device=cuda_device).manual_seed(11)
    q = inputs.random_qk((L, n, 8, 256), 5, cuda_device)
    k = inputs.random_qk((L, n, 2, 256), 6, cuda_device)
    pos = torch.randint(-(2 ** 20), 2 ** 20, (3, n), generator=g, device=cuda_device,
                        dtype=torch.int32)
    q2, k2 = q.clone(), k.clone()
    assert cmr.rotate_qk_kernel(n, L, 8, 2) == "rotate_qk_staged_kernel"
    assert cmr.rotate_qk_kernel(512, L, 8, 2) == "rotate_qk_kernel"
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    cmr.rotate_qk(q, k, pos, device_status=status)
    for a in range(0, n, 512):
        b = min(n, a + 512)
        qc, kc = q2[:, a:b].contiguous(), k2[:, a:b].contiguous()
        cmr.rotate_qk(qc, kc, pos[:, a:b].contiguous(), device_status=status)
        q2[:, a:b], k2[:, a:b] = qc, kc
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(q.view(torch.int16), q2.view(torch.int16))
    assert torch.equal(k.view(torch.int16), k2.view(torch.int16))


def test_staged_shift_form_matches_pos_form(cuda_device):
    # planes derived in the staged kernel from (start, amount) equal the pos
    # form's result, bit for bit, on a prefill batch large enough to stage
    wl = inputs.make_config(3, device=cuda_device)
    ids = torch.from_numpy(wl.ids).to(cuda_device)
    cu = torch.from_numpy(wl.cu_seqlens).to(cuda_device)
    pos, start, amount = cmr.positions(ids, cu, wl.image_token_id)
    assert cmr.rotate_qk_kernel(wl.n_tokens, wl.num_layers, wl.hq, wl.hk) == \
        "rotate_qk_staged_kernel"
    q2, k2 = wl.q.clone(), wl.k.clone()
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    cmr.rotate_qk(wl.q, wl.k, pos, device_status=status)
    cmr.rotate_qk_shift(q2, k2, start, amount, cu_seqlens=cu, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(wl.q.view(torch.int16), q2.view(torch.int16))
    assert torch.equal(wl.k.view(torch.int16), k2.view(torch.int16))


@pytest.mark.parametrize("theta", [1e4, 5e8])
def test_rotate_staged_other_theta_and_extreme_positions(cuda_device, theta):
    g = torch.Generator(device=cuda_device).manual_seed(23)
    n = 9000
    assert cmr.rotate_qk_kernel(n, 1, 8, 2) == "rotate_qk_staged_kernel"
    q = (torch.randn((1, n, 8, 256), generator=g, device=cuda_device) * 30).to(torch.bfloat16)
    k = (torch.randn((1, n, 2, 256), generator=g, device=cuda_device) * 30).to(torch.bfloat16)
    pos = torch.randint(-(2 ** 30), 2 ** 30, (3, n), generator=g, device=cuda_device,
                        dtype=torch.int32)
    pos[:, :3] = torch.tensor([0, 2 ** 31 - 1, -(2 ** 31)], dtype=torch.int32)
    check_full(q, k, pos, theta, what=f"staged theta={theta}")
