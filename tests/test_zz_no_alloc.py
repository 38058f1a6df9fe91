"""cmr_positions_frames_noalloc, the entry point for callers that cannot
allocate device memory (code inside a CUDA-graph capture, serving loops that
forbid allocation on the hot path, plug-ins whose host owns every device
buffer): called through the C ABI, it must give the planes and state of
cmr_positions_frames with a caller's workspace, bit for bit, on two different
batches in a row (the second must not see the first's leftovers in the
shared built-in scratch).  Kept in a file collected last so that a run that
stops at the first failure has run every other test; it passes alone in a
fresh process too."""
import ctypes

import numpy as np
import pytest
import torch

from vlm_decoder_positional_b200 import cmr, inputs

pytestmark = pytest.mark.gpu


def t32(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(dev)


def batch(seed, s, n_prompts, max_len):
    rng = np.random.default_rng(seed)
    F = s * s + 3
    prompts = []
    for i in range(n_prompts):
        length = int(rng.integers(1, max_len))
        count = min(int(rng.integers(0, 6)), length // (F + 1))
        origins = inputs.spaced_origins(rng, count, 0, length - 1, F + 1) if count else []
        prompts.append(inputs.prompt_ids_frames(rng, length, origins, s))
    return inputs.pack(prompts)


def no_alloc_call(ids, cu, s, dev):
    """cmr_positions_frames_noalloc through ctypes; outputs preset to -7."""
    n, b = ids.numel(), cu.numel() - 1
    pos = torch.full((3, n), -7, dtype=torch.int32, device=dev)
    start = torch.full((b,), -7, dtype=torch.int32, device=dev)
    amount = torch.full((b,), -7, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        rc = cmr.lib().cmr_positions_frames_noalloc(
            ids.data_ptr(), cu.data_ptr(), b, n, cmr.IMAGE_TOKEN_ID, s, pos.data_ptr(),
            start.data_ptr(), amount.data_ptr(), status.data_ptr(),
            torch.cuda.current_stream(dev).cuda_stream)
    assert rc == cmr.CMR_OK, cmr.lib().cmr_last_error_message()
    return pos, start, amount, status


def test_no_alloc_entry_point_matches_the_workspace_one_in_a_row(cuda_device):
    dev = cuda_device
    # different batches in a row: long prompts at s = 8 (several slices
    # each), shorter ones at s = 16 (one slice each), and 9,000 prompts whose
    # two slices each would not fit the scratch (one slice each instead)
    for seed, s, n_prompts, max_len in ((1, 8, 24, 30000), (2, 16, 300, 3000),
                                        (3, 8, 9000, 9000)):
        ids_np, cu_np = batch(seed, s, n_prompts, max_len)
        ids, cu = t32(ids_np, dev), t32(cu_np, dev)
        got = no_alloc_call(ids, cu, s, dev)
        want = cmr.positions_frames(ids, cu, s)
        torch.cuda.synchronize()
        assert int(got[3].item()) == 0
        for g, w in zip(got[:3], want):
            assert torch.equal(g, w)


def test_no_alloc_entry_point_refuses_more_sequences_than_its_scratch_serves(cuda_device):
    dev = cuda_device
    n = 16385
    ids = torch.zeros(n, dtype=torch.int32, device=dev)
    cu = torch.arange(n + 1, dtype=torch.int32, device=dev)  # 16,385 one-token prompts
    pos = torch.empty((3, n), dtype=torch.int32, device=dev)
    st = torch.empty(n, dtype=torch.int32, device=dev)
    rc = cmr.lib().cmr_positions_frames_noalloc(ids.data_ptr(), cu.data_ptr(), n, n,
                                                 cmr.IMAGE_TOKEN_ID, 8, pos.data_ptr(),
                                                 st.data_ptr(), st.data_ptr(), None, None)
    assert rc == cmr.CMR_EINVAL
    assert b"16384" in cmr.lib().cmr_last_error_message()
