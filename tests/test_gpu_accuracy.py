"""Accuracy record of the rotate kernel against the oracle on the five
workloads: every element within the bar, nearly all bit-identical to the
correctly rounded fp64 result.  Set CMR_ACCURACY_REPORT=<file> to also write
the per-workload statistics (max ulp, max |d|, share bit-identical) as JSON."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from tests.helpers import bf16_mismatches, bf16_ordinal, bf16_value
from vlm_decoder_positional_b200 import cmr, inputs

pytestmark = pytest.mark.gpu
SAMPLE = 20000  # tokens sampled from the two large workloads (all layers, all heads)


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def stats(got, want):
    ulp = np.abs(bf16_ordinal(got) - bf16_ordinal(want))
    d = np.abs(bf16_value(got) - bf16_value(want))
    return {"elements": int(ulp.size), "max_ulp": int(ulp.max()), "max_abs": float(d.max()),
            "bit_identical": float((ulp == 0).mean()), "over_1_ulp": int((ulp > 1).sum()),
            "max_abs_where_over_2_ulp": float(d[ulp > 2].max(initial=0.0)),
            "outside_bar": int(bf16_mismatches(got, want).sum())}


def test_accuracy_record(cuda_device):
    dev = cuda_device
    record = {}
    for cfg in (1, 2, 3, 4, 5):
        wl = inputs.make_config(cfg, device=dev)
        pos, s, a = cmr.positions(torch.from_numpy(wl.ids).to(dev),
                                  torch.from_numpy(wl.cu_seqlens).to(dev))
        if wl.cache_len is not None:
            pos = cmr.positions_step(torch.from_numpy(wl.cache_len).to(dev), s, a)
        n = wl.qk_tokens
        idx = (np.arange(n) if n <= SAMPLE
               else np.sort(np.random.default_rng(cfg).choice(n, SAMPLE, replace=False)))
        it = torch.from_numpy(idx).to(dev)
        q_in, k_in = bits(wl.q[:, it]), bits(wl.k[:, it])
        cmr.rotate_qk(wl.q, wl.k, pos)
        torch.cuda.synchronize()
        p = pos[:, it].cpu().numpy()
        rec = {}
        for name, x_in, x in (("q", q_in, wl.q), ("k", k_in, wl.k)):
            rec[name] = stats(bits(x[:, it])[..., :64], oracle.rotate_bf16(x_in, p)[..., :64])
            assert rec[name]["outside_bar"] == 0, (wl.name, name, rec[name])
            assert rec[name]["bit_identical"] >= 0.9999, (wl.name, name, rec[name])
        record[wl.name] = rec
        del wl
        torch.cuda.empty_cache()
    path = os.environ.get("CMR_ACCURACY_REPORT")
    if path:
        with open(path, "w") as f:
            json.dump(record, f, indent=1)
