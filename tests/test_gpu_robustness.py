"""Guard bands around every buffer (no stray writes) and a seeded fuzz over
shapes and parameters against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import assert_bf16_close
from vlm_decoder_positional_b200 import cmr, inputs

pytestmark = pytest.mark.gpu
GUARD = 4096  # elements of canary on each side


def guarded(n, dtype, dev, fill):
    """A tensor of n elements inside a larger buffer whose margins hold `fill`."""
    buf = torch.full((n + 2 * GUARD,), fill, dtype=dtype, device=dev)
    return buf, buf[GUARD:GUARD + n]


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def test_no_writes_outside_any_buffer(cuda_device):
    dev = cuda_device
    wl = inputs.make_config(2, device=dev)
    n, b, L = wl.n_tokens, wl.num_seqs, 2
    ids_buf, ids = guarded(n, torch.int32, dev, -7)
    cu_buf, cu = guarded(b + 1, torch.int32, dev, -7)
    pos_buf, pos = guarded(3 * n, torch.int32, dev, -7)
    st_buf, st = guarded(b, torch.int32, dev, -7)
    am_buf, am = guarded(b, torch.int32, dev, -7)
    ids.copy_(torch.from_numpy(wl.ids))
    cu.copy_(torch.from_numpy(wl.cu_seqlens))
    canary = torch.tensor(-3.0, dtype=torch.bfloat16).view(torch.int16).item()
    q_buf, q = guarded(L * n * 8 * 256, torch.int16, dev, canary)
    k_buf, k = guarded(L * n * 2 * 256, torch.int16, dev, canary)
    g = torch.Generator(device=dev).manual_seed(0)
    q.copy_(torch.randn(q.numel(), generator=g, device=dev).to(torch.bfloat16).view(torch.int16))
    k.copy_(torch.randn(k.numel(), generator=g, device=dev).to(torch.bfloat16).view(torch.int16))
    qv = q.view(torch.bfloat16).view(L, n, 8, 256)
    kv = k.view(torch.bfloat16).view(L, n, 2, 256)
    cmr.positions(ids, cu, out=(pos.view(3, n), st, am))
    cmr.rotate_qk(qv, kv, pos.view(3, n))
    cmr.rotate_qk_shift(qv, kv, st, am, cu_seqlens=cu)
    torch.cuda.synchronize()
    for buf in (ids_buf, cu_buf, pos_buf, st_buf, am_buf):
        assert (buf[:GUARD] == -7).all() and (buf[-GUARD:] == -7).all()
    for buf in (q_buf, k_buf):
        assert (buf[:GUARD] == canary).all() and (buf[-GUARD:] == canary).all()


@pytest.mark.parametrize("seed", range(24))
def test_fuzz_shapes_and_parameters(cuda_device, seed):
    rng = np.random.default_rng(1000 + seed)
    dev = cuda_device
    rot_dim = int(rng.choice([16, 32, 48, 64, 96, 128]))
    head_dim = int(rot_dim + 8 * rng.integers(0, 20))
    F = rot_dim // 2
    s_h = int(rng.integers(0, (F + 1) // 3 + 1))
    s_w = int(rng.integers(0, (F + 0) // 3 + 1))
    if 3 * (s_h - 1) + 1 >= F:
        s_h = 0
    if 3 * (s_w - 1) + 2 >= F:
        s_w = 0
    sections = (F - s_h - s_w, s_h, s_w)
    hq, hk = int(rng.integers(0, 12)), int(rng.integers(0, 5))
    if hq + hk == 0:
        hq = 1
    L, n = int(rng.integers(1, 5)), int(rng.integers(1, 700))
    theta = float(10 ** rng.uniform(3, 8))
    pos = torch.from_numpy(rng.integers(-50000, 50000, size=(3, n)).astype(np.int32)).to(dev)
    g = torch.Generator(device=dev).manual_seed(seed)
    mk = lambda h: ((torch.randn((L, n, h, head_dim), generator=g, device=dev)
                     * float(10 ** rng.uniform(-2, 2))).to(torch.bfloat16) if h else None)
    q, k = mk(hq), mk(hk)
    q_in = bits(q) if hq else None
    k_in = bits(k) if hk else None
    cmr.rotate_qk(q, k, pos, theta, sections, rot_dim)
    torch.cuda.synchronize()
    p = pos.cpu().numpy()
    for name, t, t_in in (("q", q, q_in), ("k", k, k_in)):
        if t is None:
            continue
        got = bits(t)
        np.testing.assert_array_equal(got[..., rot_dim:], t_in[..., rot_dim:])
        want = oracle.rotate_bf16(t_in, p, theta, sections, rot_dim)
        assert_bf16_close(got, want, f"seed {seed} {name} rot {rot_dim} D {head_dim} {sections}")


@pytest.mark.parametrize("layers", [1, 4])
def test_staged_kernels_write_nothing_outside_any_buffer(cuda_device, layers):
    # 8,195 tokens: 1,025 tiles, the last holding 3 tokens, so the TMA boxes of
    # the last tile reach past the batch; the staged rotate, the staged shift
    # form and the staged cache form must write nothing there
    dev = cuda_device
    wl = inputs.make_batch([4100, 4095], [6, 4000], num_layers=layers, with_qk=False)
    n, b, L = wl.n_tokens, wl.num_seqs, layers
    assert n == 8195 and cmr.rotate_qk_kernel(n, L, 8, 2) == "rotate_qk_staged_kernel"
    assert cmr.rotate_qk_cache_kernel(n, L, 8, 2) == "rotate_qk_cache_staged_kernel"
    canary = torch.tensor(-3.0, dtype=torch.bfloat16).view(torch.int16).item()
    bufs = {}
    views = {}
    for name, shape in (("q", (L, n, 8, 256)), ("k", (L, n, 2, 256)), ("v", (L, n, 2, 256)),
                        ("kc", (L, b, 2, 4100, 256)), ("vc", (L, b, 2, 4100, 256))):
        buf, t = guarded(int(np.prod(shape)), torch.int16, dev, canary)
        bufs[name] = buf
        views[name] = t.view(torch.bfloat16).view(shape)
    g = torch.Generator(device=dev).manual_seed(layers)
    for name in ("q", "k", "v"):
        views[name].copy_(torch.randn(views[name].shape, generator=g, device=dev))
    pos_buf, pos = guarded(3 * n, torch.int32, dev, -7)
    st_buf, st = guarded(b, torch.int32, dev, -7)
    am_buf, am = guarded(b, torch.int32, dev, -7)
    cu = torch.from_numpy(wl.cu_seqlens).to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    cmr.positions(torch.from_numpy(wl.ids).to(dev), cu, out=(pos.view(3, n), st, am))
    cmr.rotate_qk(views["q"], views["k"], pos.view(3, n), device_status=status)
    cmr.rotate_qk_shift(views["q"], views["k"], st, am, cu_seqlens=cu, device_status=status)
    cmr.rotate_qk_cache(views["q"], views["k"], views["v"], st, am, views["kc"], views["vc"],
                        cu_seqlens=cu, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for buf in (pos_buf, st_buf, am_buf):
        assert (buf[:GUARD] == -7).all() and (buf[-GUARD:] == -7).all()
    for name, buf in bufs.items():
        assert (buf[:GUARD] == canary).all() and (buf[-GUARD:] == canary).all(), name


@pytest.mark.parametrize("seed", range(8))
def test_fuzz_staged_shapes(cuda_device, seed):
    # rot_dim 64 at staged sizes with random heads, head_dim, layers, theta
    # and sections: the TMA-staged kernel against the oracle
    rng = np.random.default_rng(2000 + seed)
    dev = cuda_device
    head_dim = int(64 + 8 * rng.integers(0, 25))
    s_h = int(rng.integers(0, 11))
    s_w = int(rng.integers(0, 11))
    sections = (32 - s_h - s_w, s_h, s_w)
    hq, hk = int(rng.integers(0, 13)), int(rng.integers(0, 5))
    if hq + hk == 0:
        hk = 1
    L, n = int(rng.integers(1, 5)), int(rng.integers(8192, 11000))
    assert cmr.rotate_qk_kernel(n, L, hq, hk, head_dim) == "rotate_qk_staged_kernel"
    theta = float(10 ** rng.uniform(3, 8))
    pos = torch.from_numpy(rng.integers(-50000, 50000, size=(3, n)).astype(np.int32)).to(dev)
    g = torch.Generator(device=dev).manual_seed(seed)
    mk = lambda h: ((torch.randn((L, n, h, head_dim), generator=g, device=dev)
                     * float(10 ** rng.uniform(-2, 2))).to(torch.bfloat16) if h else None)
    q, k = mk(hq), mk(hk)
    q_in = bits(q) if hq else None
    k_in = bits(k) if hk else None
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    cmr.rotate_qk(q, k, pos, theta, sections, 64, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    p = pos.cpu().numpy()
    for name, t, t_in in (("q", q, q_in), ("k", k, k_in)):
        if t is None:
            continue
        got = bits(t)
        np.testing.assert_array_equal(got[..., 64:], t_in[..., 64:])
        want = oracle.rotate_bf16(t_in, p, theta, sections, 64)
        assert_bf16_close(got, want, f"seed {seed} {name} D {head_dim} {sections} L {L}")
