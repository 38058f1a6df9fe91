"""Test helpers: golden-file readers and the bf16 parity bar.

Parity bar for rotated Q/K (fixed before any kernel ran): an element passes when
its bf16 result is within 2 units in the last place of the oracle's
(correctly rounded) bf16 value, or when the two differ by at most 1e-2 in
absolute value.  Units in the last place are counted on the monotone integer
image of the bf16 bit pattern, so +0 and -0 are 0 apart.
"""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
MAX_ULP = 2
ABS_TOL = 1e-2


def golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def bf16_ordinal(bits):
    """Monotone map of bf16 bit patterns to integers (sign-magnitude -> two's)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.int32)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def bf16_value(bits):
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_mismatches(got_bits, want_bits, max_ulp=MAX_ULP, abs_tol=ABS_TOL):
    """Boolean mask of elements that fail the parity bar (NaN always fails)."""
    got_bits = np.asarray(got_bits, dtype=np.uint16)
    want_bits = np.asarray(want_bits, dtype=np.uint16)
    ulp = np.abs(bf16_ordinal(got_bits) - bf16_ordinal(want_bits))
    g, w = bf16_value(got_bits), bf16_value(want_bits)
    with np.errstate(invalid="ignore"):
        ok = (ulp <= max_ulp) | (np.abs(g - w) <= abs_tol)
    ok &= ~np.isnan(g) & ~np.isnan(w)
    return ~ok


def assert_bf16_close(got_bits, want_bits, what=""):
    bad = bf16_mismatches(got_bits, want_bits)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        g = np.asarray(got_bits)[bad][:5]
        w = np.asarray(want_bits)[bad][:5]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements outside the bar; first at "
            f"{idx.tolist()} got {bf16_value(g).tolist()} want {bf16_value(w).tolist()}")


def ulp_stats(got_bits, want_bits):
    ulp = np.abs(bf16_ordinal(got_bits) - bf16_ordinal(want_bits))
    d = np.abs(bf16_value(got_bits) - bf16_value(want_bits))
    return int(ulp.max(initial=0)), float(d.max(initial=0.0))
