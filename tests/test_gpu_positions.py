"""GPU parity of the position planes: bit-exact against the oracle, through the
C ABI, on the five workloads, the red arms and the edge cases."""
import numpy as np
import pytest
import torch

import oracle
from vlm_decoder_positional_b200 import cmr, inputs

pytestmark = pytest.mark.gpu
MARK = inputs.IMAGE_TOKEN_ID


def gpu_positions(ids, cu, dev, marker=MARK):
    ids_t = torch.from_numpy(np.ascontiguousarray(ids, np.int32)).to(dev)
    cu_t = torch.from_numpy(np.ascontiguousarray(cu, np.int32)).to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    pos, start, amount = cmr.positions(ids_t, cu_t, marker, device_status=status)
    torch.cuda.synchronize(dev)
    return pos.cpu().numpy(), start.cpu().numpy(), amount.cpu().numpy(), int(status.item())


def check_batch(ids, cu, dev, marker=MARK):
    got = gpu_positions(ids, cu, dev, marker)
    want = oracle.positions(ids, cu, marker)
    assert got[3] == 0
    np.testing.assert_array_equal(got[0], want[0])
    np.testing.assert_array_equal(got[1], want[1])
    np.testing.assert_array_equal(got[2], want[2])
    return got


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_positions_bit_exact_on_every_workload(cuda_device, cfg):
    wl = inputs.make_config(cfg, with_qk=False)
    pos, start, amount, _ = check_batch(wl.ids, wl.cu_seqlens, cuda_device)
    # the red arms must differ from what the GPU produced on image prompts
    for rule in ("amount+1", "planes_1d"):
        red = oracle.positions(wl.ids, wl.cu_seqlens, MARK, rule=rule)[0]
        for b in range(wl.num_seqs):
            if wl.frame_origin[b] >= 0:
                s = slice(wl.cu_seqlens[b], wl.cu_seqlens[b + 1])
                assert (red[:, s] != pos[:, s]).any(), (rule, b)


def test_decode_step_bit_exact(cuda_device):
    wl = inputs.make_config(4, with_qk=False)
    _, start, amount, _ = check_batch(wl.ids, wl.cu_seqlens, cuda_device)
    dev = cuda_device
    got = cmr.positions_step(torch.from_numpy(wl.cache_len).to(dev),
                             torch.from_numpy(start).to(dev), torch.from_numpy(amount).to(dev))
    want = oracle.positions_step(wl.cache_len, start, amount)
    np.testing.assert_array_equal(got.cpu().numpy(), want)
    assert (want == wl.cache_len - 58).all()


def test_step_form_on_every_index_and_arbitrary_shifts(cuda_device):
    rng = np.random.default_rng(1)
    n = 200_000
    p = rng.integers(-5, 1 << 20, size=n).astype(np.int32)
    start = rng.integers(0, 1 << 20, size=n).astype(np.int32)
    amount = rng.integers(-100, 1000, size=n).astype(np.int32)
    start[::7] = 1 << 30
    amount[::7] = 0
    # around real frames: every offset of the frame for a few origins
    o = np.repeat(np.array([0, 6, 17, 5000]), 80)
    off = np.tile(np.arange(-3, 77), 4)
    p = np.concatenate([p, (o + off).astype(np.int32)])
    start = np.concatenate([start, (o + 67).astype(np.int32)])
    amount = np.concatenate([amount, np.full(o.size, 58, np.int32)])
    dev = cuda_device
    got = cmr.positions_step(torch.from_numpy(p).to(dev), torch.from_numpy(start).to(dev),
                             torch.from_numpy(amount).to(dev))
    np.testing.assert_array_equal(got.cpu().numpy(), oracle.positions_step(p, start, amount))


def test_edge_cases(cuda_device):
    rng = np.random.default_rng(2)
    cases = [
        ([1], [0]), ([1], [-1]), ([67], [0]), ([66], [0]), ([68], [0]), ([0], [-1]),
        ([0, 0, 5, 0], [-1, -1, 2, -1]), ([300], [299]), ([300], [233]), ([300], [234]),
        ([3, 4, 5, 1000, 2, 70], [0, 1, -1, 998, 0, 3]),
    ]
    for lens, origins in cases:
        prompts = [inputs.prompt_ids(rng, n, o) for n, o in zip(lens, origins)]
        ids, cu = inputs.pack(prompts)
        check_batch(ids, cu, cuda_device)


def test_long_single_prompt_spans_many_ctas(cuda_device):
    rng = np.random.default_rng(3)
    for origin in (-1, 0, 2047, 2048, 150_001, 299_990):
        ids = inputs.prompt_ids(rng, 300_000, origin)
        check_batch(ids, np.array([0, 300_000], np.int32), cuda_device)


def test_many_short_prompts_and_repeated_markers(cuda_device):
    rng = np.random.default_rng(4)
    lens = rng.integers(0, 90, size=5000)
    origins = np.where(rng.random(5000) < 0.6, rng.integers(0, 30, size=5000), -1)
    prompts = [inputs.prompt_ids(rng, int(n), int(o)) for n, o in zip(lens, origins)]
    for p in prompts[::9]:
        if len(p) > 10:
            p[rng.integers(0, len(p), size=3)] = MARK   # extra markers
    ids, cu = inputs.pack(prompts)
    check_batch(ids, cu, cuda_device)


def test_pad_row_ids_and_other_marker_ids(cuda_device):
    rng = np.random.default_rng(5)
    prompts = [inputs.prompt_ids(rng, 200, 10, row_ids="pad"), inputs.prompt_ids(rng, 200, 0)]
    ids, cu = inputs.pack(prompts)
    check_batch(ids, cu, cuda_device)
    check_batch(ids, cu, cuda_device, marker=198)   # "\n" as the marker id: a different O


def test_malformed_cu_seqlens_sets_status_without_faulting(cuda_device):
    ids = np.zeros(100, np.int32)
    for cu in ([0, 60, 50, 100], [0, 50, 120], [5, 50, 100], [0, 50, 90]):
        _, _, _, status = gpu_positions(ids, np.array(cu, np.int32), cuda_device)
        assert status & cmr.CMR_DEVICE_BAD_CU_SEQLENS


def test_host_pointer_is_rejected(cuda_device):
    ids = np.zeros(16, np.int32)
    cu = torch.tensor([0, 16], dtype=torch.int32, device=cuda_device)
    out = torch.empty((3, 16), dtype=torch.int32, device=cuda_device)
    st = torch.empty(1, dtype=torch.int32, device=cuda_device)
    rc = cmr.lib().cmr_positions(ids.ctypes.data, cu.data_ptr(), 1, 16, MARK, out.data_ptr(),
                                 st.data_ptr(), st.data_ptr(), None, None)
    assert rc == cmr.CMR_EINVAL
    assert b"not device memory" in cmr.lib().cmr_last_error_message()
