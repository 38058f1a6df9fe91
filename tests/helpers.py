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


def host_threads():
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_rotate_threads(x_bits, pos, theta=1e7, sections=(11, 11, 10), rot_dim=64,
                          threads=None):
    """oracle.rotate_bf16 over contiguous token ranges on a thread pool (the
    oracle is C called through ctypes, which releases the GIL).  Each token's
    rotation depends only on its own planes, so the result equals one call
    over the whole array.  x_bits: uint16 [L, N, H, D]; pos: int32 [3, N]."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    x_bits = np.asarray(x_bits, dtype=np.uint16)
    pos = np.asarray(pos, dtype=np.int32)
    n = x_bits.shape[1]
    threads = min(threads or host_threads(), max(1, n))
    out = np.empty_like(x_bits)
    cuts = np.linspace(0, n, threads + 1).astype(np.int64)

    def run(i):
        lo, hi = int(cuts[i]), int(cuts[i + 1])
        if hi > lo:
            out[:, lo:hi] = oracle.rotate_bf16(x_bits[:, lo:hi], pos[:, lo:hi], theta, sections,
                                               rot_dim)

    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(run, range(threads)))
    return out


class BarStats:
    """Element statistics of a bf16 result against the oracle's, accumulated
    over chunks so that arrays of billions of elements never need a float64
    copy of the whole: elements, worst ulp distance, worst |difference|, share
    bit-identical, elements more than 1 ulp away, worst |difference| among
    those more than 2 ulps away, and elements outside the bar."""

    def __init__(self, what=""):
        self.what = what
        self.elements = 0
        self.max_ulp = 0
        self.max_abs = 0.0
        self.identical = 0
        self.over_1_ulp = 0
        self.max_abs_over_2_ulp = 0.0
        self.outside_bar = 0
        self.first_bad = None

    def add(self, got_bits, want_bits, chunk=1 << 24):
        g_all = np.asarray(got_bits, dtype=np.uint16).reshape(-1)
        w_all = np.asarray(want_bits, dtype=np.uint16).reshape(-1)
        assert g_all.shape == w_all.shape, (g_all.shape, w_all.shape)
        for lo in range(0, g_all.size, chunk):
            g, w = g_all[lo:lo + chunk], w_all[lo:lo + chunk]
            ulp = np.abs(bf16_ordinal(g) - bf16_ordinal(w))
            d = np.abs(bf16_value(g) - bf16_value(w))
            bad = bf16_mismatches(g, w)
            self.elements += int(g.size)
            self.max_ulp = max(self.max_ulp, int(ulp.max(initial=0)))
            self.max_abs = max(self.max_abs, float(np.nanmax(d, initial=0.0)))
            self.identical += int((ulp == 0).sum())
            self.over_1_ulp += int((ulp > 1).sum())
            self.max_abs_over_2_ulp = max(self.max_abs_over_2_ulp,
                                          float(d[ulp > 2].max(initial=0.0)))
            nbad = int(bad.sum())
            if nbad and self.first_bad is None:
                i = int(np.argmax(bad))
                self.first_bad = (lo + i, float(bf16_value(g[i])), float(bf16_value(w[i])))
            self.outside_bar += nbad
        return self

    def record(self):
        return {"elements": self.elements, "max_ulp": self.max_ulp, "max_abs": self.max_abs,
                "bit_identical": self.identical / max(self.elements, 1),
                "over_1_ulp": self.over_1_ulp,
                "max_abs_where_over_2_ulp": self.max_abs_over_2_ulp,
                "outside_bar": self.outside_bar}

    def check(self):
        if self.outside_bar:
            raise AssertionError(
                f"{self.what}: {self.outside_bar} of {self.elements} elements outside the bar; "
                f"first (flat index, got, want) = {self.first_bad}")
        return self
