"""GPU parity of the multi-frame canvas (cmr_positions_frames) with the
oracle, bit for bit: grid sides 1 .. 128, several frames per prompt (spaced,
crowded, cut short, truncated), text-only and empty prompts, prompts spanning
many slices, reduced and stale workspaces, a CUDA-graph replay, unaligned buffers, the rotation with the
planes it writes, and decode after the last frame."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import BarStats, oracle_rotate_threads
from vlm_decoder_positional_b200 import cmr, inputs

pytestmark = pytest.mark.gpu
MARK = inputs.IMAGE_TOKEN_ID


def t32(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(dev)


def run_both(ids, cu, dev, s, workspace=None, status_want=0):
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    pos, start, amount = cmr.positions_frames(t32(ids, dev), t32(cu, dev), s,
                                              workspace=workspace, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == status_want
    want = oracle.positions_frames(ids, cu, MARK, s)
    for name, g, w in zip(("pos", "start", "amount"), (pos, start, amount), want):
        np.testing.assert_array_equal(g.cpu().numpy(), w, err_msg=f"{name} s={s}")
    return pos, start, amount


def random_batch(rng, s, n_prompts, max_len, crowded=False):
    F = s * s + 3
    prompts = []
    for _ in range(n_prompts):
        length = int(rng.integers(0, max_len + 1))
        kind = rng.integers(0, 4)
        if kind == 0 or length == 0:
            origins = []                                           # text-only
        elif kind == 1 and length > F:
            count = int(rng.integers(1, max(2, min(8, length // F))))
            origins = inputs.spaced_origins(rng, count, 0, length - 1, F)   # spaced frames
        else:
            count = int(rng.integers(1, 6))                            # cut short / overlapping
            origins = sorted(rng.integers(0, length, size=count).tolist())
        ids = inputs.prompt_ids_frames(rng, length, origins, s)
        if crowded and length:
            ids[rng.integers(0, length, size=max(1, length // 50))] = MARK
        prompts.append(ids)
    return inputs.pack(prompts)


@pytest.mark.parametrize("s", [1, 2, 3, 8, 16])
def test_random_batches_match_the_oracle(cuda_device, s):
    rng = np.random.default_rng(100 + s)
    for crowded in (False, True):
        ids, cu = random_batch(rng, s, 40, 6000, crowded)
        run_both(ids, cu, cuda_device, s)


@pytest.mark.parametrize("s", [5, 7, 100, 128])
def test_other_grid_sides_up_to_the_largest(cuda_device, s):
    # grid rows k / s for sides that are not powers of two, up to s = 128
    # (frames of 16,387 tokens), whole and cut short
    rng = np.random.default_rng(800 + s)
    ids, cu = random_batch(rng, s, 12, 3 * (s * s + 3) + 500)
    run_both(ids, cu, cuda_device, s)


def test_one_frame_at_s8_equals_cmr_positions(cuda_device):
    dev = cuda_device
    for cfg in (1, 2, 3):
        wl = inputs.make_config(cfg, with_qk=False)
        pos, start, amount = run_both(wl.ids, wl.cu_seqlens, dev, 8)
        p2, s2, a2 = cmr.positions(t32(wl.ids, dev), t32(wl.cu_seqlens, dev))
        assert torch.equal(pos, p2) and torch.equal(start, s2) and torch.equal(amount, a2)


@pytest.mark.parametrize("s", [8, 16])
def test_long_prompts_over_many_slices(cuda_device, s):
    # 300k-token prompts (147 slices each): one with frames all along, one
    # text-only, one whose only frame sits near the end, one with crowded markers
    rng = np.random.default_rng(200 + s)
    F = s * s + 3
    n = 300_000
    frames = inputs.prompt_ids_frames(rng, n, inputs.spaced_origins(rng, 400, 0, n - 1, F + 5), s)
    text = inputs.text_ids(rng, n)
    late = inputs.prompt_ids_frames(rng, n, [n - F // 2], s)
    crowded = inputs.text_ids(rng, n)
    crowded[rng.integers(0, n, size=3000)] = MARK
    ids, cu = inputs.pack([frames, text, late, crowded])
    run_both(ids, cu, cuda_device, s)


def test_small_workspaces_give_the_same_planes(cuda_device):
    dev = cuda_device
    rng = np.random.default_rng(300)
    ids, cu = random_batch(rng, 8, 12, 20000)
    b = cu.shape[0] - 1
    full = cmr.positions_frames_workspace_bytes(b, ids.shape[0])
    assert full > 16 * b
    for nbytes in (16 * b, 16 * b + 15, 32 * b, full - 16, full, full + 4096):
        ws = torch.full((nbytes,), 0x5A, dtype=torch.uint8, device=dev)  # stale contents
        run_both(ids, cu, dev, 8, workspace=ws)
        run_both(ids, cu, dev, 8, workspace=ws)  # and what the previous call left
    with pytest.raises(cmr.CmrError):
        cmr.positions_frames(t32(ids, dev), t32(cu, dev), 8,
                             workspace=torch.empty(16 * b - 1, dtype=torch.uint8, device=dev))


def test_empty_prompts_and_malformed_cu_seqlens(cuda_device):
    dev = cuda_device
    rng = np.random.default_rng(400)
    prompts = [np.zeros(0, np.int32), inputs.prompt_ids_frames(rng, 500, [3, 100], 8),
               np.zeros(0, np.int32), inputs.text_ids(rng, 7), np.zeros(0, np.int32)]
    ids, cu = inputs.pack(prompts)
    run_both(ids, cu, dev, 8)
    for bad in ([0, 60, 50, 100], [0, 50, 120], [5, 50, 100]):
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        cmr.positions_frames(t32(np.zeros(100, np.int32), dev), t32(bad, dev), 8,
                             device_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) & cmr.CMR_DEVICE_BAD_CU_SEQLENS


def test_graph_replay_and_the_rotation_with_frame_planes(cuda_device):
    dev = cuda_device
    rng = np.random.default_rng(500)
    ids_np, cu_np = random_batch(rng, 8, 16, 4000)
    ids, cu = t32(ids_np, dev), t32(cu_np, dev)
    n, b = ids_np.shape[0], cu_np.shape[0] - 1
    pos = torch.empty((3, n), dtype=torch.int32, device=dev)
    st = torch.empty(b, dtype=torch.int32, device=dev)
    am = torch.empty(b, dtype=torch.int32, device=dev)
    ws = torch.empty(cmr.positions_frames_workspace_bytes(b, n), dtype=torch.uint8, device=dev)
    cmr.positions_frames(ids, cu, 8, out=(pos, st, am), workspace=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cmr.positions_frames(ids, cu, 8, out=(pos, st, am), workspace=ws)
    want, want_s, want_a = oracle.positions_frames(ids_np, cu_np, MARK, 8)
    for _ in range(2):
        pos.fill_(-9)
        g.replay()
        torch.cuda.synchronize()
        np.testing.assert_array_equal(pos.cpu().numpy(), want)
        np.testing.assert_array_equal(st.cpu().numpy(), want_s)
        np.testing.assert_array_equal(am.cpu().numpy(), want_a)
    q = inputs.random_qk((2, n, 8, 256), 7, dev)
    k = inputs.random_qk((2, n, 2, 256), 8, dev)
    q_in = q[..., :64].contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    cmr.rotate_qk(q, k, pos)
    torch.cuda.synchronize()
    got = q[..., :64].contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    BarStats("q with frame planes").add(got, oracle_rotate_threads(q_in, want)).check()


def test_unaligned_buffers_and_odd_token_counts(cuda_device):
    # ids and the planes at addresses that are not 16-byte aligned, and token
    # counts that leave the plane rows unaligned: element-wise paths
    dev = cuda_device
    rng = np.random.default_rng(600)
    for n_extra in (0, 1, 2, 3):
        ids_np, cu_np = random_batch(rng, 8, 9, 5000)
        if n_extra:
            ids_np = np.concatenate([ids_np, inputs.text_ids(rng, n_extra)])
            cu_np = cu_np.copy()
            cu_np[-1] += n_extra
        n, b = ids_np.shape[0], cu_np.shape[0] - 1
        want = oracle.positions_frames(ids_np, cu_np, MARK, 8)
        for shift in (0, 1, 3):
            ids_buf = torch.zeros(n + 4, dtype=torch.int32, device=dev)
            ids_buf[shift:shift + n] = t32(ids_np, dev)
            pos_buf = torch.full((3 * n + 4,), -5, dtype=torch.int32, device=dev)
            pos = pos_buf[shift:shift + 3 * n].view(3, n)
            st = torch.empty(b, dtype=torch.int32, device=dev)
            am = torch.empty(b, dtype=torch.int32, device=dev)
            cmr.positions_frames(ids_buf[shift:shift + n], t32(cu_np, dev), 8, out=(pos, st, am))
            torch.cuda.synchronize()
            np.testing.assert_array_equal(pos.cpu().numpy(), want[0])
            np.testing.assert_array_equal(st.cpu().numpy(), want[1])
            assert (pos_buf[:shift] == -5).all() and (pos_buf[shift + 3 * n:] == -5).all()


def test_decode_continues_after_the_last_frame(cuda_device):
    # the state of a multi-frame prompt drives the decode forms: the planes of
    # each later token (cmr_positions_step, and the rotation deriving them in
    # the kernel) equal the oracle's on the prompt extended with text
    dev = cuda_device
    rng = np.random.default_rng(700)
    for s in (2, 8, 16):
        F = s * s + 3
        prompts, longer = [], []
        for i in range(6):
            count = int(rng.integers(0, 4))
            origins = inputs.spaced_origins(rng, count, 0, count * (F + 40), F + 1) if count else []
            full = inputs.prompt_ids_frames(rng, (origins[-1] if origins else 0) + F + 60,
                                            origins, s)
            cut = (origins[-1] + F if origins else 0) + int(rng.integers(0, 20))
            prompts.append(full[:cut])
            longer.append(full)
        ids_np, cu_np = inputs.pack(prompts)
        _, start, amount = cmr.positions_frames(t32(ids_np, dev), t32(cu_np, dev), s)
        cache_len = np.array([p.shape[0] for p in prompts], np.int32)
        got = cmr.positions_step(t32(cache_len, dev), start, amount).cpu().numpy()
        for b, full in enumerate(longer):
            want, _, _ = oracle.positions_frames(*(np.asarray(full, np.int32),
                                                   np.array([0, full.shape[0]], np.int32)),
                                                 MARK, s)
            np.testing.assert_array_equal(got[:, b], want[:, cache_len[b]])
        # the same planes, derived inside the rotation (one token per sequence)
        n = len(prompts)
        q = inputs.random_qk((1, n, 8, 256), 70 + s, dev)
        k = inputs.random_qk((1, n, 2, 256), 80 + s, dev)
        q2, k2 = q.clone(), k.clone()
        cmr.rotate_qk_shift(q, k, start, amount, pos_offset=t32(cache_len, dev))
        cmr.rotate_qk(q2, k2, t32(got, dev))
        torch.cuda.synchronize()
        assert torch.equal(q.view(torch.int16), q2.view(torch.int16))
        assert torch.equal(k.view(torch.int16), k2.view(torch.int16))
