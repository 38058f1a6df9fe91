"""GPU parity of the fused rotate + KV-cache write, through the C ABI:
Q rotated in place, rotated K rows and V rows placed at each token's index."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import assert_bf16_close
from vlm_decoder_positional_b200 import cmr, inputs

pytestmark = pytest.mark.gpu
SENTINEL = 0x7F7F


def t32(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(dev)


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def sentinel_cache(shape, dev):
    return torch.full(shape, SENTINEL, dtype=torch.int16, device=dev).view(torch.bfloat16)


def rand(shape, g, dev):
    return torch.randn(shape, generator=g, device=dev).to(torch.bfloat16)


def run_and_compare(q, k, v, start, amount, kc, vc, cu=None, off=None, slot=None, status_want=0):
    dev = q.device
    q_in, k_in, v_in = bits(q), bits(k), bits(v)
    kc_in, vc_in = bits(kc), bits(vc)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    cmr.rotate_qk_cache(q, k, v, start, amount, kc, vc, cu_seqlens=cu, pos_offset=off,
                        cache_slot=slot, device_status=status)
    torch.cuda.synchronize()
    np_ = lambda t: None if t is None else t.cpu().numpy()
    qo, kco, vco, st = oracle.rotate_qk_cache(q_in, k_in, v_in, np_(start), np_(amount), kc_in,
                                              vc_in, np_(cu), np_(off), np_(slot))
    assert int(status.item()) == st == status_want
    assert_bf16_close(bits(q), qo, "q")
    # K / V are only read
    np.testing.assert_array_equal(bits(k), k_in)
    np.testing.assert_array_equal(bits(v), v_in)
    got_kc, got_vc = bits(kc), bits(vc)
    np.testing.assert_array_equal(got_vc, vco)             # V rows are copies
    written = kco != kc_in
    np.testing.assert_array_equal(got_kc[~written], kco[~written])
    assert_bf16_close(got_kc[written], kco[written], "k_cache")


def test_prefill_varlen_into_permuted_slots(cuda_device):
    dev = cuda_device
    wl = inputs.make_config(2, device=dev)
    _, s, a = cmr.positions(t32(wl.ids, dev), t32(wl.cu_seqlens, dev))
    g = torch.Generator(device=dev).manual_seed(1)
    n = wl.n_tokens
    v = rand((1, n, 2, 256), g, dev)
    S, ctx = 20, 520
    kc = sentinel_cache((1, S, 2, ctx, 256), dev)
    vc = sentinel_cache((1, S, 2, ctx, 256), dev)
    slot = t32(np.random.default_rng(3).permutation(S)[:wl.num_seqs], dev)
    run_and_compare(wl.q, wl.k, v, s, a, kc, vc, cu=t32(wl.cu_seqlens, dev), slot=slot)


def test_decode_appends_at_each_sequences_length(cuda_device):
    dev = cuda_device
    rng = np.random.default_rng(4)
    B, ctx = 64, 4096                        # the engine's context limit
    prior = rng.integers(73, ctx, size=B)
    origins = np.array([rng.integers(0, p_ - 67 + 1) for p_ in prior])
    wl = inputs.make_batch(prior, origins, with_qk=False, device=dev)
    _, s, a = cmr.positions(t32(wl.ids, dev), t32(wl.cu_seqlens, dev))
    g = torch.Generator(device=dev).manual_seed(5)
    L = 2
    q, k, v = rand((L, B, 8, 256), g, dev), rand((L, B, 2, 256), g, dev), rand((L, B, 2, 256), g, dev)
    kc = sentinel_cache((L, B, 2, ctx, 256), dev)
    vc = sentinel_cache((L, B, 2, ctx, 256), dev)
    run_and_compare(q, k, v, s, a, kc, vc, off=t32(prior, dev))


def test_out_of_range_tokens_write_nothing_and_flag(cuda_device):
    dev = cuda_device
    g = torch.Generator(device=dev).manual_seed(6)
    B = 5
    q, k, v = rand((2, B, 4, 128), g, dev), rand((2, B, 3, 128), g, dev), rand((2, B, 3, 128), g, dev)
    kc = sentinel_cache((2, 3, 3, 16, 128), dev)
    vc = sentinel_cache((2, 3, 3, 16, 128), dev)
    start = t32([1 << 30] * B, dev)
    amount = t32([0] * B, dev)
    off = t32([0, 15, 16, 3, -1], dev)       # 16 and -1 fall outside ctx 16
    slot = t32([0, 1, 2, 5, 1], dev)         # slot 5 falls outside S 3
    run_and_compare(q, k, v, start, amount, kc, vc, off=off, slot=slot,
                    status_want=cmr.CMR_DEVICE_CACHE_RANGE)


def test_q_only_needs_no_cache(cuda_device):
    dev = cuda_device
    g = torch.Generator(device=dev).manual_seed(7)
    q = rand((1, 40, 8, 256), g, dev)
    q_in = bits(q)
    start, amount = t32([73], dev), t32([58], dev)
    cmr.rotate_qk_cache(q, None, None, start, amount, None, None, cu_seqlens=t32([0, 40], dev),
                        pos_offset=t32([50], dev))
    torch.cuda.synchronize()
    p = oracle.positions_step(np.arange(50, 90), np.full(40, 73), np.full(40, 58))
    assert_bf16_close(bits(q), oracle.rotate_bf16(q_in, p), "q")


def test_cache_path_matches_shift_path_bit_for_bit(cuda_device):
    # Q after the cache form equals Q after cmr_rotate_qk_shift, and the cached
    # K rows equal K rotated in place by cmr_rotate_qk_shift.
    dev = cuda_device
    wl = inputs.make_config(3, device=dev)
    cu = t32(wl.cu_seqlens, dev)
    _, s, a = cmr.positions(t32(wl.ids, dev), cu)
    v = wl.k.clone()
    kc = sentinel_cache((1, 64, 2, 4096, 256), dev)
    vc = sentinel_cache((1, 64, 2, 4096, 256), dev)
    q2, k2 = wl.q.clone(), wl.k.clone()
    cmr.rotate_qk_cache(wl.q, wl.k, v, s, a, kc, vc, cu_seqlens=cu)
    cmr.rotate_qk_shift(q2, k2, s, a, cu_seqlens=cu)
    torch.cuda.synchronize()
    assert torch.equal(wl.q.view(torch.int16), q2.view(torch.int16))
    # prompt b's tokens fill cache rows [b, :, 0:4096] in order
    kc_tokens = kc.view(1, 64, 2, 4096, 256).permute(0, 1, 3, 2, 4).reshape(1, 64 * 4096, 2, 256)
    assert torch.equal(kc_tokens.view(torch.int16), k2.view(torch.int16))
    vc_tokens = vc.permute(0, 1, 3, 2, 4).reshape(1, 64 * 4096, 2, 256)
    assert torch.equal(vc_tokens.view(torch.int16), v.view(torch.int16))


# ---- the TMA-staged cache kernel (rot_dim 64, from 1024 tiles of 8 tokens) ----

@pytest.mark.parametrize("layers", [1, 2, 4])
def test_staged_prefill_into_permuted_slots_with_out_of_range_tokens(cuda_device, layers):
    # 16,400 tokens in 4 prompts (a ragged last tile), slots permuted inside a
    # 5-sequence cache whose context (4,100) leaves the last 11 tokens of the
    # 4,111-token prompt outside: those write no K/V and set the status bit
    dev = cuda_device
    wl = inputs.make_batch([4100, 4096, 4111, 4093], [6, 17, 3000, 4080], num_layers=layers,
                           with_qk=False)
    n = wl.n_tokens
    assert cmr.rotate_qk_cache_kernel(n, layers, 8, 2) == "rotate_qk_cache_staged_kernel"
    cu = t32(wl.cu_seqlens, dev)
    _, s, a = cmr.positions(t32(wl.ids, dev), cu)
    q = inputs.random_qk((layers, n, 8, 256), 31, dev)
    k = inputs.random_qk((layers, n, 2, 256), 32, dev)
    v = inputs.random_qk((layers, n, 2, 256), 33, dev)
    kc = sentinel_cache((layers, 5, 2, 4100, 256), dev)
    vc = sentinel_cache((layers, 5, 2, 4100, 256), dev)
    run_and_compare(q, k, v, s, a, kc, vc, cu=cu, slot=t32([2, 0, 4, 1], dev),
                    status_want=cmr.CMR_DEVICE_CACHE_RANGE)


def test_staged_kernels_are_the_ones_that_run(cuda_device):
    # the kernel names the library reports are the kernels the profiler sees
    from torch.profiler import ProfilerActivity, profile
    dev = cuda_device
    wl = inputs.make_batch([4100, 4100], [6, 17], num_layers=2, with_qk=False)
    n = wl.n_tokens
    cu = t32(wl.cu_seqlens, dev)
    pos, s, a = cmr.positions(t32(wl.ids, dev), cu)
    q = inputs.random_qk((2, n, 8, 256), 41, dev)
    k = inputs.random_qk((2, n, 2, 256), 42, dev)
    v = inputs.random_qk((2, n, 2, 256), 43, dev)
    kc = sentinel_cache((2, 2, 2, 4100, 256), dev)
    vc = sentinel_cache((2, 2, 2, 4100, 256), dev)
    cmr.rotate_qk_cache(q, k, v, s, a, kc, vc, cu_seqlens=cu)   # first launch outside capture
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        cmr.rotate_qk(q, k, pos)
        cmr.rotate_qk_cache(q, k, v, s, a, kc, vc, cu_seqlens=cu)
        q1, k1 = q[:1, :512].contiguous(), k[:1, :512].contiguous()
        cmr.rotate_qk(q1, k1, pos[:, :512].contiguous())
        torch.cuda.synchronize()
    names = " ".join(e.name for e in prof.events())
    for kernel in (cmr.rotate_qk_kernel(n, 2, 8, 2), cmr.rotate_qk_cache_kernel(n, 2, 8, 2),
                   cmr.rotate_qk_kernel(512, 1, 8, 2)):
        assert kernel + "<" in names or kernel + "(" in names, (kernel, names[:2000])
    assert "rotate_qk_staged_kernel" in names and "rotate_qk_cache_staged_kernel" in names


CACHE_FIRST_CALL_IN_CAPTURE = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
from vlm_decoder_positional_b200 import cmr, inputs
dev = torch.device("cuda", 0)
wl = inputs.make_batch([4100, 4100], [6, 17], num_layers=3, with_qk=False)
n = wl.n_tokens
assert cmr.rotate_qk_cache_kernel(n, 3, 8, 2) == "rotate_qk_cache_staged_kernel"
cu = torch.from_numpy(wl.cu_seqlens).to(dev)
s = torch.tensor([73, 84], dtype=torch.int32, device=dev)
a = torch.tensor([58, 58], dtype=torch.int32, device=dev)
q0 = inputs.random_qk((3, n, 8, 256), 51, dev)
k = inputs.random_qk((3, n, 2, 256), 52, dev)
v = inputs.random_qk((3, n, 2, 256), 53, dev)
def fresh():
    kc = torch.zeros((3, 2, 2, 4100, 256), dtype=torch.bfloat16, device=dev)
    return q0.clone(), kc, torch.zeros_like(kc)
q1, kc1, vc1 = fresh()
torch.cuda.synchronize()
g = torch.cuda.CUDAGraph()
with torch.cuda.graph(g):   # the process's first library call: the staged kernel would
    cmr.rotate_qk_cache(q1, k, v, s, a, kc1, vc1, cu_seqlens=cu)   # need an attribute call
g.replay()
q2, kc2, vc2 = fresh()
cmr.rotate_qk_cache(q2, k, v, s, a, kc2, vc2, cu_seqlens=cu)       # eager: staged kernel
torch.cuda.synchronize()
for x, y in ((q1, q2), (kc1, kc2), (vc1, vc2)):
    assert torch.equal(x.view(torch.int16), y.view(torch.int16))
print("ok")
"""


def test_cache_form_first_call_inside_graph_capture(cuda_device, tmp_path):
    # a fresh process whose first library call is a staged-size cache form
    # being captured: the launch falls back to the register kernel (the staged
    # one needs a shared-memory opt-in first), and its replay equals the eager
    # staged kernel's result bit for bit
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    script = tmp_path / "cache_first_call.py"
    script.write_text(CACHE_FIRST_CALL_IN_CAPTURE)
    out = subprocess.run([sys.executable, str(script), root], capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0 and out.stdout.strip().endswith("ok"), out.stderr[-2000:]
