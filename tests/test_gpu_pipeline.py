"""The host-buffer pipeline gives exactly the device path's results."""
import numpy as np
import pytest
import torch

from vlm_decoder_positional_b200 import cmr, inputs, pipeline

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg,chunk", [(2, 1000), (3, 3 * 4096), (5, 2 * 8192)])
def test_host_pipeline_matches_the_device_path(cuda_device, cfg, chunk):
    wl = inputs.make_config(cfg, device=cuda_device)
    dev = cuda_device
    ref_q, ref_k = wl.q.clone(), wl.k.clone()
    pos, s, a = cmr.positions(torch.from_numpy(wl.ids).to(dev), torch.from_numpy(wl.cu_seqlens).to(dev))
    cmr.rotate_qk(ref_q, ref_k, pos)
    q_h = wl.q.cpu().pin_memory()
    k_h = wl.k.cpu().pin_memory()
    ids_h = torch.from_numpy(wl.ids).pin_memory()
    pos_h = torch.empty((3, wl.n_tokens), dtype=torch.int32, pin_memory=True)
    st_h = torch.empty(wl.num_seqs, dtype=torch.int32, pin_memory=True)
    am_h = torch.empty(wl.num_seqs, dtype=torch.int32, pin_memory=True)
    lens = np.diff(wl.cu_seqlens)
    pl = pipeline.HostPipeline(dev, wl.num_layers, wl.hq, wl.hk, wl.head_dim,
                               max_chunk_tokens=max(chunk, int(lens.max())),
                               max_chunk_seqs=wl.num_seqs, depth=3)
    for _ in range(2):   # the second run reuses the ring (inputs rotated twice)
        pl.run(ids_h, wl.cu_seqlens, q_h, k_h, pos_h, st_h, am_h, chunk_tokens=chunk)
    torch.cuda.synchronize()
    cmr.rotate_qk(ref_q, ref_k, pos)
    torch.cuda.synchronize()
    assert torch.equal(pos_h, pos.cpu()) and torch.equal(st_h, s.cpu()) and torch.equal(am_h, a.cpu())
    assert torch.equal(q_h.view(torch.int16), ref_q.cpu().view(torch.int16))
    assert torch.equal(k_h.view(torch.int16), ref_k.cpu().view(torch.int16))


def test_copy_rotated_dims_moves_exactly_the_rotated_dims(cuda_device):
    g = torch.Generator().manual_seed(1)
    h = torch.randn((3, 50, 4, 256), generator=g).to(torch.bfloat16).pin_memory()
    d = torch.full((3, 50, 4, 256), 7.0, dtype=torch.bfloat16, device=cuda_device)
    cmr.copy_rotated_dims(d, h, 64)
    torch.cuda.synchronize()
    assert torch.equal(d[..., :64].cpu(), h[..., :64])
    assert (d[..., 64:] == 7.0).all()
    back = torch.zeros_like(h).pin_memory()
    cmr.copy_rotated_dims(back, d, 64)
    torch.cuda.synchronize()
    assert torch.equal(back[..., :64], h[..., :64]) and (back[..., 64:] == 0).all()
