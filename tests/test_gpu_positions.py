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


BLOCK = 16_384  # ids per block of the origin scan


@pytest.mark.parametrize("length", [120_000, 200_000, 300_000, 1_000_000])
def test_cluster_scan_block_and_rank_boundaries(cuda_device, length):
    # prompts this long average more than four blocks of ids, so each one is
    # scanned by a cluster of 2, 4, 8 or 16 CTAs dealing the blocks round-robin;
    # markers sit on both sides of every block edge the prompt has (so on
    # every rank and round), first and last, or nowhere
    rng = np.random.default_rng(10 + length // 1000)
    blocks = (length + BLOCK - 1) // BLOCK
    origins = {-1, 0, 1, length - 1, length - 67, length // 2}
    for j in range(1, blocks):
        origins.update({j * BLOCK - 1, j * BLOCK, j * BLOCK + BLOCK // 2})
    origins = sorted(o for o in origins if -1 <= o < length)
    if length >= 300_000:  # a sample of the edges keeps the batch small
        origins = origins[:: 3 if length < 1_000_000 else 5] + [-1]
    prompts = [inputs.prompt_ids(rng, length, o) for o in origins]
    # a later marker does not hide an earlier one: extra markers after O
    for p, o in zip(prompts, origins):
        if 0 <= o < length - 100:
            p[rng.integers(o + 68, length, size=5)] = MARK
    # batches of up to 4 prompts: few enough for the largest cluster size
    # the length takes (2 at 120k tokens ... 16 at 1M)
    for i in range(0, len(prompts), 4):
        ids, cu = inputs.pack(prompts[i:i + 4])
        check_batch(ids, cu, cuda_device)


def test_cluster_scan_with_short_and_empty_prompts_in_the_batch(cuda_device):
    # a long average (clusters of 8) with short and empty prompts among the
    # long ones: the ranks past a short prompt's end scan nothing
    rng = np.random.default_rng(20)
    lens = [300_000, 0, 5, 70, 300_000, 1, 200_000, 0]
    origins = [200_000, -1, 2, 0, -1, 0, 16_384 * 7 + 3, -1]
    prompts = [inputs.prompt_ids(rng, n, o) for n, o in zip(lens, origins)]
    ids, cu = inputs.pack(prompts)
    check_batch(ids, cu, cuda_device)


def test_cluster_scan_in_chunks_and_the_one_call_path(cuda_device):
    # the continuation form over long chunks (clusters), with sequences whose
    # frame is already known (no scan) beside ones still text-only, and the
    # one-call path's origin scan on long prompts
    dev = cuda_device
    rng = np.random.default_rng(30)
    n = 150_000
    prompts = [inputs.prompt_ids(rng, n, o) for o in (-1, 70_000, -1, 131_072)]
    ids_np, cu_np = inputs.pack(prompts)
    offset = np.array([0, 1000, 5000, 0], np.int32)
    in_start = np.array([1 << 30, 1 << 30, 4000, 1 << 30], np.int32)
    in_amount = np.array([0, 0, 3942, 0], np.int32)
    want = oracle.positions_chunk(ids_np, cu_np, MARK, pos_offset=offset, in_start=in_start,
                                  in_amount=in_amount)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(dev)
    got = cmr.positions_chunk(t(ids_np), t(cu_np), pos_offset=t(offset),
                              state=(t(in_start), t(in_amount)))
    for g, w in zip(got, want):
        np.testing.assert_array_equal(g.cpu().numpy(), w)
    q = inputs.random_qk((1, ids_np.shape[0], 2, 256), 31, dev)
    k = inputs.random_qk((1, ids_np.shape[0], 1, 256), 32, dev)
    pos, start, amount = cmr.positions_rotate_qk(t(ids_np), t(cu_np), q, k)
    want = oracle.positions(ids_np, cu_np, MARK)
    for g, w in zip((pos, start, amount), want):
        np.testing.assert_array_equal(g.cpu().numpy(), w)


CAPTURE_FIRST = r"""
import sys
import numpy as np, torch
sys.path.insert(0, sys.argv[1])
import oracle
from vlm_decoder_positional_b200 import cmr, inputs
dev = torch.device("cuda", 0)
rng = np.random.default_rng(40)
n = int(sys.argv[2])
ids_np, cu_np = inputs.pack([inputs.prompt_ids(rng, n, o) for o in (-1, n - 50_000)])
ids, cu = torch.from_numpy(ids_np).to(dev), torch.from_numpy(cu_np).to(dev)
pos = torch.empty((3, ids.numel()), dtype=torch.int32, device=dev)
st = torch.empty(2, dtype=torch.int32, device=dev)
am = torch.empty(2, dtype=torch.int32, device=dev)
g = torch.cuda.CUDAGraph()
with torch.cuda.graph(g):  # the library's first launch in this process
    cmr.positions(ids, cu, out=(pos, st, am))
g.replay()
torch.cuda.synchronize()
want = oracle.positions(ids_np, cu_np, inputs.IMAGE_TOKEN_ID)
for a, b in zip((pos, st, am), want):
    np.testing.assert_array_equal(a.cpu().numpy(), b)
print("ok")
"""


@pytest.mark.parametrize("length", [300_000, 1_000_000])
def test_cluster_scan_first_launched_inside_a_graph_capture(cuda_device, length):
    # the occupancy query that picks the cluster form runs during the capture;
    # at 1M tokens the 16-CTA opt-in is not set there, and the portable size runs
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "-c", CAPTURE_FIRST, root, str(length)],
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.strip().endswith("ok")


def test_large_batch_in_long_slices(cuda_device):
    # 256 prompts x 65,536 tokens: enough CTAs for three waves even with the
    # planes kernel's long (8,192-token) slices.  Text-only prompts, markers
    # on both sides of every slice edge and at the prompts' ends, and random
    # origins; every plane bit-exact
    rng = np.random.default_rng(1234)
    n, F = 65536, 67
    prompts = []
    for i in range(256):
        kind = i % 4
        if kind == 0:
            prompts.append(inputs.text_ids(rng, n))
            continue
        if kind == 1:
            edge = 8192 * int(rng.integers(1, 8))
            origin = edge - 1 if i % 8 == 1 else edge          # either side of a slice edge
        elif kind == 2:
            origin = n - 1 - int(rng.integers(0, F + 2))        # a frame cut off by the end
        else:
            origin = int(rng.integers(0, n))
        prompts.append(inputs.prompt_ids_frames(rng, n, [origin], 8))
    ids, cu = inputs.pack(prompts)
    check_batch(ids, cu, cuda_device)


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
