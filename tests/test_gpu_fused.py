"""The one-call path (cmr_positions_rotate_qk: the positions kernels, then the
rotation launched to overlap them) gives the bits of the two separate calls,
and every element of the two large workloads matches the oracle.  It is also
checked inside a CUDA graph, where the overlap becomes a programmatic edge."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import BarStats, oracle_rotate_threads
from vlm_decoder_positional_b200 import cmr, inputs

pytestmark = pytest.mark.gpu
ROT = 64


def t32(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(dev)


def bits(t, dims=None):
    t = t if dims is None else t[..., :dims]
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("cfg", [1, 2, 3, 5])
def test_one_call_equals_two_calls(cuda_device, cfg):
    dev = cuda_device
    wl = inputs.make_config(cfg, device=dev)
    ids, cu = t32(wl.ids, dev), t32(wl.cu_seqlens, dev)
    q2, k2 = wl.q.clone(), wl.k.clone()
    large = cfg in (3, 5)
    q_in = bits(wl.q, ROT) if large else None
    k_in = bits(wl.k, ROT) if large else None
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    pos, start, amount = cmr.positions_rotate_qk(ids, cu, wl.q, wl.k, device_status=status)
    torch.cuda.synchronize()
    assert cmr.last_rotate_kernel() == cmr.rotate_qk_kernel(wl.n_tokens, wl.num_layers, wl.hq,
                                                            wl.hk)
    pos2, start2, amount2 = cmr.positions(ids, cu)
    cmr.rotate_qk(q2, k2, pos2, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(pos, pos2) and torch.equal(start, start2) and torch.equal(amount, amount2)
    assert torch.equal(wl.q.view(torch.int16), q2.view(torch.int16))
    assert torch.equal(wl.k.view(torch.int16), k2.view(torch.int16))
    del q2, k2
    p, s_o, a_o = oracle.positions(wl.ids, wl.cu_seqlens)
    np.testing.assert_array_equal(pos.cpu().numpy(), p)
    np.testing.assert_array_equal(start.cpu().numpy(), s_o)
    np.testing.assert_array_equal(amount.cpu().numpy(), a_o)
    if large:  # every element of the rotated dims against the oracle
        BarStats(f"{wl.name} one-call q").add(bits(wl.q, ROT),
                                              oracle_rotate_threads(q_in, p)).check()
        BarStats(f"{wl.name} one-call k").add(bits(wl.k, ROT),
                                              oracle_rotate_threads(k_in, p)).check()


@pytest.mark.parametrize("shape,kernel", [((4, 1500, 2), "rotate_qk_kernel"),
                                          ((3, 9000, 6), "rotate_qk_staged_kernel")])
def test_one_call_replayed_from_a_cuda_graph(cuda_device, shape, kernel):
    # the register kernel (750 tiles of 8 tokens) and the staged kernel; three
    # replays on fresh inputs
    dev = cuda_device
    b, length, layers = shape
    wl = inputs.make_batch([length] * b, [5 + 100 * i for i in range(b)], num_layers=layers,
                           with_qk=False)
    n = wl.n_tokens
    assert cmr.rotate_qk_kernel(n, layers, 8, 2) == kernel
    ids, cu = t32(wl.ids, dev), t32(wl.cu_seqlens, dev)
    q = torch.empty((layers, n, 8, 256), dtype=torch.bfloat16, device=dev)
    k = torch.empty((layers, n, 2, 256), dtype=torch.bfloat16, device=dev)
    pos = torch.empty((3, n), dtype=torch.int32, device=dev)
    st = torch.empty(b, dtype=torch.int32, device=dev)
    am = torch.empty(b, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    cmr.positions_rotate_qk(ids, cu, q, k, out=(pos, st, am), device_status=status)  # warm-up
    torch.cuda.synchronize()
    assert cmr.last_rotate_kernel() == kernel
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cmr.positions_rotate_qk(ids, cu, q, k, out=(pos, st, am), device_status=status)
    want_pos, _, _ = oracle.positions(wl.ids, wl.cu_seqlens)
    for rep in range(3):
        q.copy_(inputs.random_qk(tuple(q.shape), 100 + rep, dev))
        k.copy_(inputs.random_qk(tuple(k.shape), 200 + rep, dev))
        pos.fill_(-1)
        q_in, k_in = bits(q), bits(k)
        g.replay()
        torch.cuda.synchronize()
        np.testing.assert_array_equal(pos.cpu().numpy(), want_pos)
        BarStats("graph q").add(bits(q), oracle_rotate_threads(q_in, want_pos)).check()
        BarStats("graph k").add(bits(k), oracle_rotate_threads(k_in, want_pos)).check()
    assert int(status.item()) == 0


def test_one_call_with_empty_prompts_and_without_layers(cuda_device):
    # empty prompts get their state from the origin scan alone; with no
    # layers to rotate the planes kernel writes pos
    dev = cuda_device
    rng = np.random.default_rng(9)
    prompts = [np.zeros(0, np.int32), inputs.prompt_ids(rng, 5000, 17), np.zeros(0, np.int32),
               inputs.prompt_ids(rng, 4000, -1), inputs.prompt_ids(rng, 3000, 2990)]
    ids_np, cu_np = inputs.pack(prompts)
    ids, cu = t32(ids_np, dev), t32(cu_np, dev)
    n = ids_np.shape[0]
    want = oracle.positions(ids_np, cu_np)
    for layers in (0, 1, 3):
        q = inputs.random_qk((layers, n, 8, 256), 40 + layers, dev) if layers else \
            torch.empty((0, n, 8, 256), dtype=torch.bfloat16, device=dev)
        k = inputs.random_qk((layers, n, 2, 256), 50 + layers, dev) if layers else \
            torch.empty((0, n, 2, 256), dtype=torch.bfloat16, device=dev)
        q_in = bits(q)
        got = cmr.positions_rotate_qk(ids, cu, q, k)
        torch.cuda.synchronize()
        for g, w in zip(got, want):
            np.testing.assert_array_equal(g.cpu().numpy(), w)
        if layers:
            BarStats(f"q L={layers}").add(bits(q), oracle_rotate_threads(q_in, want[0])).check()
