"""The host pipeline's chunk plan (CPU): contiguous ranges of whole prompts
that cover the batch once, each within the token limit unless it is a single
longer prompt, and each as long as the limit allows (greedy)."""
import numpy as np
import pytest

from vlm_decoder_positional_b200 import pipeline


def check_plan(cu, limit):
    ch = pipeline.prompt_chunks(cu, limit)
    b = len(cu) - 1
    if b == 0:
        assert ch == []
        return ch
    assert ch[0][0] == 0 and ch[-1][1] == b
    assert all(s0 < s1 for s0, s1 in ch)
    assert all(a[1] == b_[0] for a, b_ in zip(ch, ch[1:]))
    for s0, s1 in ch:
        assert cu[s1] - cu[s0] <= limit or s1 - s0 == 1
        if s1 < b:  # one more prompt would break the limit
            assert cu[s1 + 1] - cu[s0] > limit
    return ch


def test_worked_plan():
    cu = np.array([0, 5, 5, 30, 31, 100, 101], np.int64)
    assert check_plan(cu, 30) == [(0, 3), (3, 4), (4, 5), (5, 6)]


def test_edge_plans():
    assert check_plan(np.array([0], np.int64), 10) == []
    assert check_plan(np.array([0, 0, 0, 0], np.int64), 1) == [(0, 3)]       # empty prompts
    assert check_plan(np.array([0, 1000], np.int64), 10) == [(0, 1)]         # one long prompt
    assert check_plan(np.array([0, 10, 20, 30], np.int64), 10) == [(0, 1), (1, 2), (2, 3)]


@pytest.mark.parametrize("seed", range(20))
def test_random_plans(seed):
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, 3000, size=int(rng.integers(1, 200)))
    lens[rng.random(lens.shape[0]) < 0.1] = 0
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    check_plan(cu, int(rng.integers(1, 20000)))
