"""The test helpers that split the oracle over threads and accumulate the
parity bar over chunks give the same answers as one plain call."""
import numpy as np

import oracle
from tests.helpers import (BarStats, bf16_mismatches, bf16_ordinal, oracle_rotate_threads)


def test_threaded_oracle_equals_one_call():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((3, 101, 4, 80)).astype(np.float32).view(np.uint32) >> 16)
    x = x.astype(np.uint16)
    pos = rng.integers(-5000, 5000, size=(3, 101)).astype(np.int32)
    want = oracle.rotate_bf16(x, pos, 1e6, (6, 5, 5), 32)
    for threads in (1, 2, 7, 200):
        got = oracle_rotate_threads(x, pos, 1e6, (6, 5, 5), 32, threads=threads)
        np.testing.assert_array_equal(got, want)


def test_chunked_statistics_match_the_plain_bar():
    rng = np.random.default_rng(6)
    want = rng.integers(0, 1 << 16, size=50000).astype(np.uint16)
    want &= np.uint16(0x7F7F)  # finite values only
    got = want.copy()
    step = rng.integers(-4, 5, size=want.size)
    got = np.clip(bf16_ordinal(want) + step, -0x7F7F, 0x7F7F)
    got = np.where(got < 0, 0x8000 | (-got), got).astype(np.uint16)
    s = BarStats().add(got, want, chunk=977)
    assert s.elements == want.size
    assert s.outside_bar == int(bf16_mismatches(got, want).sum())
    assert s.max_ulp == int(np.abs(bf16_ordinal(got) - bf16_ordinal(want)).max())
    assert s.identical == int((got == want).sum() + ((got == 0x8000) & (want == 0)).sum()
                              + ((got == 0) & (want == 0x8000)).sum())
