"""cmr_positions_rotate_qk_host, the whole path on a batch held in pinned host
memory (the kernels read and write it over PCIe): bit for bit the results of
cmr_positions_rotate_qk on the same batch in device memory, and the planes
and rotated rows of the oracle; device and pageable buffers are refused."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import BarStats, oracle_rotate_threads
from vlm_decoder_positional_b200 import cmr, inputs

pytestmark = pytest.mark.gpu


def pinned(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)) if isinstance(a, np.ndarray) else a.cpu()
    if dtype is not None:
        t = t.to(dtype)
    return t.contiguous().pin_memory()


def bits(t):
    return t.contiguous().cpu().view(torch.int16)


def test_other_rot_dims_and_head_counts(cuda_device):
    # the row-coalesced kernel at rot_dim 16 .. 256 (2 .. 32 lanes per row),
    # and the register kernel for a rot_dim it does not take (48)
    dev = cuda_device
    rng = np.random.default_rng(12)
    ids, cu = inputs.pack([inputs.prompt_ids(rng, n, o) for n, o in ((300, 20), (77, -1),
                                                                   (500, 400))])
    n = ids.shape[0]
    for rot_dim, sections, hq, hk, D, kernel in (
            (16, (4, 2, 2), 3, 1, 64, "rotate_qk_rows_kernel"),
            (32, (6, 5, 5), 2, 2, 128, "rotate_qk_rows_kernel"),
            (128, (22, 21, 21), 4, 1, 128, "rotate_qk_rows_kernel"),
            (256, (44, 42, 42), 1, 1, 256, "rotate_qk_rows_kernel"),
            (48, (8, 8, 8), 2, 1, 64, "rotate_qk_kernel")):
        q = pinned(inputs.random_qk((2, n, hq, D), rot_dim, "cpu"))
        k = pinned(inputs.random_qk((2, n, hk, D), rot_dim + 1, "cpu"))
        q_d, k_d = q.to(dev), k.to(dev)
        want = cmr.positions_rotate_qk(torch.from_numpy(ids).to(dev), torch.from_numpy(cu).to(dev),
                                       q_d, k_d, sections=sections, rot_dim=rot_dim)
        got = cmr.positions_rotate_qk_host(pinned(ids), pinned(cu), q, k, sections=sections,
                                           rot_dim=rot_dim, device=dev)
        assert cmr.last_rotate_kernel() == kernel
        torch.cuda.synchronize(dev)
        for g, w in zip(got, want):
            assert torch.equal(g, w.cpu())
        assert torch.equal(bits(q), bits(q_d)) and torch.equal(bits(k), bits(k_d)), rot_dim


@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_host_batch_equals_the_device_path_bit_for_bit(cuda_device, cfg):
    dev = cuda_device
    wl = inputs.make_config(cfg, device=dev)
    ids_h, cu_h = pinned(wl.ids), pinned(wl.cu_seqlens)
    q_h, k_h = pinned(wl.q), pinned(wl.k)
    q_d, k_d = wl.q.clone(), wl.k.clone()
    want = cmr.positions_rotate_qk(torch.from_numpy(wl.ids).to(dev),
                                   torch.from_numpy(wl.cu_seqlens).to(dev), q_d, k_d)
    got = cmr.positions_rotate_qk_host(ids_h, cu_h, q_h, k_h, device=dev)
    assert cmr.last_rotate_kernel() == "rotate_qk_rows_kernel"
    torch.cuda.synchronize(dev)
    for g, w in zip(got, want):
        assert g.is_pinned()
        assert torch.equal(g, w.cpu())
    assert torch.equal(bits(q_h), bits(q_d)) and torch.equal(bits(k_h), bits(k_d))


def test_host_batch_against_the_oracle(cuda_device):
    dev = cuda_device
    wl = inputs.make_config(2, device="cpu")
    q_in = wl.q.view(torch.int16).numpy().view(np.uint16).copy()
    k_in = wl.k.view(torch.int16).numpy().view(np.uint16).copy()
    q_h, k_h = pinned(wl.q), pinned(wl.k)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    pos, start, amount = cmr.positions_rotate_qk_host(pinned(wl.ids), pinned(wl.cu_seqlens),
                                                      q_h, k_h, device=dev,
                                                      device_status=status)
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0
    want = oracle.positions(wl.ids, wl.cu_seqlens, inputs.IMAGE_TOKEN_ID)
    for g, w in zip((pos, start, amount), want):
        np.testing.assert_array_equal(g.numpy(), w)
    p = want[0]
    BarStats("q (host batch)").add(q_h.view(torch.int16).numpy().view(np.uint16),
                                    oracle_rotate_threads(q_in, p)).check()
    BarStats("k (host batch)").add(k_h.view(torch.int16).numpy().view(np.uint16),
                                    oracle_rotate_threads(k_in, p)).check()


def test_empty_prompts_and_no_layers(cuda_device):
    dev = cuda_device
    rng = np.random.default_rng(9)
    prompts = [np.zeros(0, np.int32), inputs.prompt_ids(rng, 120, 3), np.zeros(0, np.int32),
               inputs.prompt_ids(rng, 9, -1)]
    ids, cu = inputs.pack(prompts)
    n = ids.shape[0]
    want = oracle.positions(ids, cu, inputs.IMAGE_TOKEN_ID)
    q = pinned(torch.zeros((0, n, 8, 256), dtype=torch.bfloat16))
    k = pinned(torch.zeros((0, n, 2, 256), dtype=torch.bfloat16))
    got = cmr.positions_rotate_qk_host(pinned(ids), pinned(cu), q, k, device=dev)
    torch.cuda.synchronize(dev)
    for g, w in zip(got, want):
        np.testing.assert_array_equal(g.numpy(), w)
    q = pinned(inputs.random_qk((1, n, 8, 256), 3, "cpu"))
    k = pinned(inputs.random_qk((1, n, 2, 256), 4, "cpu"))
    q_d, k_d = q.to(dev), k.to(dev)
    cmr.positions_rotate_qk(torch.from_numpy(ids).to(dev), torch.from_numpy(cu).to(dev), q_d, k_d)
    got = cmr.positions_rotate_qk_host(pinned(ids), pinned(cu), q, k, device=dev)
    torch.cuda.synchronize(dev)
    for g, w in zip(got, want):
        np.testing.assert_array_equal(g.numpy(), w)
    assert torch.equal(bits(q), bits(q_d)) and torch.equal(bits(k), bits(k_d))


def test_device_and_pageable_buffers_are_refused(cuda_device):
    dev = cuda_device
    wl = inputs.make_config(1, device="cpu")
    n, b = wl.n_tokens, wl.num_seqs
    sec = (__import__("ctypes").c_int32 * 3)(11, 11, 10)
    host = dict(ids=pinned(wl.ids), cu=pinned(wl.cu_seqlens), q=pinned(wl.q), k=pinned(wl.k),
                pos=pinned(torch.empty((3, n), dtype=torch.int32)),
                st=pinned(torch.empty(b, dtype=torch.int32)),
                am=pinned(torch.empty(b, dtype=torch.int32)))
    for name in host:
        for other in (host[name].to(dev), host[name].clone()):  # device, then pageable
            a = dict(host)
            a[name] = other
            with torch.cuda.device(dev):
                st = cmr.lib().cmr_positions_rotate_qk_host(
                    a["ids"].data_ptr(), a["cu"].data_ptr(), b, n, inputs.IMAGE_TOKEN_ID,
                    a["pos"].data_ptr(), a["st"].data_ptr(), a["am"].data_ptr(),
                    a["q"].data_ptr(), a["k"].data_ptr(), 1, 8, 2, 256, 1e7, sec, 64, None, None)
            assert st == cmr.CMR_EINVAL, (name, cmr.lib().cmr_last_error_message())
    with pytest.raises(ValueError):
        cmr.positions_rotate_qk_host(torch.from_numpy(wl.ids), pinned(wl.cu_seqlens),
                                     host["q"], host["k"], device=dev)


def test_malformed_cu_seqlens_sets_a_host_status_word(cuda_device):
    # the status word may itself live in mapped host memory
    dev = cuda_device
    n = 100
    ids = pinned(np.zeros(n, np.int32))
    q = pinned(inputs.random_qk((1, n, 8, 256), 5, "cpu"))
    k = pinned(inputs.random_qk((1, n, 2, 256), 6, "cpu"))
    sec = (__import__("ctypes").c_int32 * 3)(11, 11, 10)
    for bad in ([0, 60, 50, 100], [0, 50, 120], [5, 50, 100]):
        cu = pinned(np.array(bad, np.int32))
        b = len(bad) - 1
        pos = pinned(torch.empty((3, n), dtype=torch.int32))
        st = pinned(torch.empty(b, dtype=torch.int32))
        am = pinned(torch.empty(b, dtype=torch.int32))
        status = pinned(torch.zeros(1, dtype=torch.int32))
        with torch.cuda.device(dev):
            rc = cmr.lib().cmr_positions_rotate_qk_host(
                ids.data_ptr(), cu.data_ptr(), b, n, inputs.IMAGE_TOKEN_ID, pos.data_ptr(),
                st.data_ptr(), am.data_ptr(), q.data_ptr(), k.data_ptr(), 1, 8, 2, 256, 1e7, sec,
                64, status.data_ptr(), None)
        assert rc == cmr.CMR_OK, cmr.lib().cmr_last_error_message()
        torch.cuda.synchronize(dev)
        assert int(status[0]) & cmr.CMR_DEVICE_BAD_CU_SEQLENS, bad
