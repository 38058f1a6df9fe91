"""Every element of the two large workloads (64 x 4096 tokens with x100
outliers; 6 layers x 32 x 8192 tokens) against the oracle, in the launch
configuration the bench times, for the forms that the accuracy record does
not cover: the rotation with planes derived in the kernel (shift form), and
the rotation + KV-cache write on the 64 x 4096 shape (Q, and every cache row:
written rows against the oracle's rotated K and V, unwritten rows untouched).
The oracle runs on a thread pool over token ranges."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import BarStats, oracle_rotate_threads
from vlm_decoder_positional_b200 import cmr, inputs

pytestmark = pytest.mark.gpu
ROT = 64
SENTINEL = 0x7F7F


def t32(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(dev)


def bits(t, dims=None):
    t = t if dims is None else t[..., :dims]
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("cfg", [3, 5])
def test_shift_form_every_element(cuda_device, cfg):
    dev = cuda_device
    wl = inputs.make_config(cfg, device=dev)
    ids, cu = t32(wl.ids, dev), t32(wl.cu_seqlens, dev)
    _, start, amount = cmr.positions(ids, cu)
    assert cmr.rotate_qk_kernel(wl.n_tokens, wl.num_layers, wl.hq, wl.hk) == \
        "rotate_qk_staged_kernel"
    q_in, k_in = bits(wl.q, ROT), bits(wl.k, ROT)
    q_tail, k_tail = wl.q[..., ROT:].clone(), wl.k[..., ROT:].clone()
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    cmr.rotate_qk_shift(wl.q, wl.k, start, amount, cu_seqlens=cu, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(wl.q[..., ROT:].view(torch.int16), q_tail.view(torch.int16))
    assert torch.equal(wl.k[..., ROT:].view(torch.int16), k_tail.view(torch.int16))
    del q_tail, k_tail
    # the oracle's planes for every token, from the ids alone
    p, s_o, a_o = oracle.positions(wl.ids, wl.cu_seqlens)
    np.testing.assert_array_equal(start.cpu().numpy(), s_o)
    np.testing.assert_array_equal(amount.cpu().numpy(), a_o)
    BarStats(f"{wl.name} shift q").add(bits(wl.q, ROT), oracle_rotate_threads(q_in, p)).check()
    BarStats(f"{wl.name} shift k").add(bits(wl.k, ROT), oracle_rotate_threads(k_in, p)).check()


def test_cache_form_every_element_64x4096(cuda_device):
    dev = cuda_device
    wl = inputs.make_config(3, device=dev)
    n, b = wl.n_tokens, wl.num_seqs
    ids, cu = t32(wl.ids, dev), t32(wl.cu_seqlens, dev)
    _, start, amount = cmr.positions(ids, cu)
    assert cmr.rotate_qk_cache_kernel(n, 1, 8, 2) == "rotate_qk_cache_staged_kernel"
    v = inputs.random_qk((1, n, 2, 256), wl.seed + 3, dev)
    ctx = int(np.diff(wl.cu_seqlens).max()) + 8  # the last 8 positions stay unwritten
    kc = torch.full((1, b, 2, ctx, 256), SENTINEL, dtype=torch.int16, device=dev)
    vc = torch.full_like(kc, SENTINEL)
    kc, vc = kc.view(torch.bfloat16), vc.view(torch.bfloat16)
    slot = np.random.default_rng(7).permutation(b).astype(np.int32)
    q_in, k_in, v_in = bits(wl.q, ROT), bits(wl.k), bits(v)
    q_tail = wl.q[..., ROT:].clone()
    k_before, v_before = wl.k.clone(), v.clone()
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    cmr.rotate_qk_cache(wl.q, wl.k, v, start, amount, kc, vc, cu_seqlens=cu,
                        cache_slot=t32(slot, dev), device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(wl.q[..., ROT:].view(torch.int16), q_tail.view(torch.int16))
    assert torch.equal(wl.k.view(torch.int16), k_before.view(torch.int16))  # K, V read only
    assert torch.equal(v.view(torch.int16), v_before.view(torch.int16))
    p, _, _ = oracle.positions(wl.ids, wl.cu_seqlens)
    BarStats("cache q").add(bits(wl.q, ROT), oracle_rotate_threads(q_in, p)).check()
    # every K row rotated by the oracle (its untouched dims kept), V rows copied
    k_rot = oracle_rotate_threads(k_in, p)
    tok = np.arange(n)
    seq = np.repeat(np.arange(b), np.diff(wl.cu_seqlens))
    local = tok - wl.cu_seqlens[seq]
    got_kc, got_vc = bits(kc), bits(vc)
    rows_k = got_kc[0][slot[seq], :, local, :]          # [n, 2, 256]
    rows_v = got_vc[0][slot[seq], :, local, :]
    BarStats("k_cache rotated dims").add(rows_k[..., :ROT], k_rot[0][..., :ROT]).check()
    np.testing.assert_array_equal(rows_k[..., ROT:], k_in[0][..., ROT:])
    np.testing.assert_array_equal(rows_v, v_in[0])
    # every other cache row keeps the sentinel
    written = np.zeros((b, ctx), dtype=bool)
    written[slot[seq], local] = True
    assert (got_kc[0].transpose(0, 2, 1, 3)[~written] == SENTINEL).all()
    assert (got_vc[0].transpose(0, 2, 1, 3)[~written] == SENTINEL).all()
