"""Accuracy record of the rotate kernels against the oracle on the five
workloads, every element of Q and K (all layers, heads and rotated dims,
compared with the oracle's correctly rounded fp64 result): none outside the
bar, at least 99.99 % bit-identical, and the untouched dims kept bit for bit.
The oracle runs on a thread pool over token ranges.  Set
CMR_ACCURACY_REPORT=<file> to also write the per-workload statistics (max
ulp, max |d|, share bit-identical) as JSON."""
import json
import os

import numpy as np
import pytest
import torch

from tests.helpers import BarStats, oracle_rotate_threads
from vlm_decoder_positional_b200 import cmr, inputs

pytestmark = pytest.mark.gpu
ROT = 64


def rotated_bits(t):
    """uint16 copy of the rotated dims of a bf16 tensor [L, N, H, D]."""
    return t[..., :ROT].contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def test_accuracy_record(cuda_device):
    dev = cuda_device
    record = {}
    for cfg in (1, 2, 3, 4, 5):
        wl = inputs.make_config(cfg, device=dev)
        pos, s, a = cmr.positions(torch.from_numpy(wl.ids).to(dev),
                                  torch.from_numpy(wl.cu_seqlens).to(dev))
        if wl.cache_len is not None:
            pos = cmr.positions_step(torch.from_numpy(wl.cache_len).to(dev), s, a)
        q_in, k_in = rotated_bits(wl.q), rotated_bits(wl.k)
        q_tail, k_tail = wl.q[..., ROT:].clone(), wl.k[..., ROT:].clone()
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        cmr.rotate_qk(wl.q, wl.k, pos, device_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(wl.q[..., ROT:].view(torch.int16), q_tail.view(torch.int16))
        assert torch.equal(wl.k[..., ROT:].view(torch.int16), k_tail.view(torch.int16))
        del q_tail, k_tail
        p = pos.cpu().numpy()
        rec = {"kernel": cmr.rotate_qk_kernel(wl.qk_tokens, wl.num_layers, wl.hq, wl.hk)}
        for name, x_in, x in (("q", q_in, wl.q), ("k", k_in, wl.k)):
            st = BarStats(f"{wl.name} {name}").add(rotated_bits(x),
                                                   oracle_rotate_threads(x_in, p))
            rec[name] = st.record()
            st.check()
            assert rec[name]["bit_identical"] >= 0.9999, (wl.name, name, rec[name])
        record[wl.name] = rec
        del wl, q_in, k_in
        torch.cuda.empty_cache()
    path = os.environ.get("CMR_ACCURACY_REPORT")
    if path:
        with open(path, "w") as f:
            json.dump(record, f, indent=1)
