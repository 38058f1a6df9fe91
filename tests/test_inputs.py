"""The seeded workload generator: shapes, frame layout and determinism (CPU)."""
import numpy as np
import pytest
import torch

from vlm_decoder_positional_b200 import inputs


@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_frames_are_laid_out_as_the_processor_does(cfg):
    wl = inputs.make_config(cfg, with_qk=False)
    cu = wl.cu_seqlens
    assert cu[0] == 0 and cu[-1] == wl.n_tokens and (np.diff(cu) >= 0).all()
    for b in range(wl.num_seqs):
        seq = wl.ids[cu[b]:cu[b + 1]]
        O = int(wl.frame_origin[b])
        marks = np.flatnonzero(seq == inputs.IMAGE_TOKEN_ID)
        if O < 0:
            assert marks.size == 0
            continue
        assert marks.tolist() == [O]
        fr = inputs.frame_ids()
        n = min(len(seq) - O, 67)
        np.testing.assert_array_equal(seq[O:O + n], fr[:n])
        assert (seq[:O] < inputs.VOCAB).all()


def test_config_shapes():
    c1 = inputs.make_config(1)
    assert c1.q.shape == (1, 80, 8, 256) and c1.k.shape == (1, 80, 2, 256)
    assert c1.q.dtype == torch.bfloat16 and int(c1.frame_origin[0]) == 6
    c2 = inputs.make_config(2, with_qk=False)
    lens = np.diff(c2.cu_seqlens)
    assert c2.num_seqs == 16 and lens.min() >= 96 and lens.max() <= 512
    o = c2.frame_origin
    assert np.isin(o, [6, 17]).sum() >= 8 and o.max() <= 40
    c3 = inputs.make_config(3, with_qk=False)
    assert c3.n_tokens == 64 * 4096 and (c3.frame_origin < 0).sum() == 16
    assert c3.frame_origin.max() <= 3000
    c4 = inputs.make_config(4, with_qk=False)
    assert c4.num_seqs == 1024 and (c4.cache_len == np.diff(c4.cu_seqlens)).all()
    assert c4.cache_len.min() >= 73 and c4.cache_len.max() <= 32768
    assert (c4.frame_origin + 67 <= c4.cache_len).all()
    c5 = inputs.make_config(5, with_qk=False)
    assert c5.n_tokens == 32 * 8192 and c5.frame_origin.max() <= 6000


def test_deterministic_and_outliers():
    a = inputs.random_qk((1, 64, 2, 256), 99, outlier_frac=0.05)
    b = inputs.random_qk((1, 64, 2, 256), 99, outlier_frac=0.05)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    big = (a.float().abs() > 20).float().mean().item()
    assert 0.02 < big < 0.08
    w1 = inputs.make_config(2, with_qk=False)
    w2 = inputs.make_config(2, with_qk=False)
    assert (w1.ids == w2.ids).all()


def test_text_ids_avoid_the_marker():
    rng = np.random.default_rng(0)
    ids = inputs.text_ids(rng, 2_000_000)
    assert not (ids == inputs.IMAGE_TOKEN_ID).any()
    assert ids.min() >= 0 and ids.max() < inputs.VOCAB
