"""GPU parity of the chunked positions form, its rules, and the rotate that
derives the planes in the kernel, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import assert_bf16_close
from vlm_decoder_positional_b200 import cmr, inputs

pytestmark = pytest.mark.gpu
MARK = inputs.IMAGE_TOKEN_ID


def t32(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(dev)


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def chunk_batches(wl, size):
    """Split every prompt of a workload into consecutive chunks of `size`
    tokens; step i holds the i-th chunk of every prompt (empty once done)."""
    lens = np.diff(wl.cu_seqlens)
    steps = int(np.ceil(lens.max() / size))
    for i in range(steps):
        lo = np.minimum(lens, i * size)
        hi = np.minimum(lens, (i + 1) * size)
        parts = [wl.ids[wl.cu_seqlens[b] + lo[b]: wl.cu_seqlens[b] + hi[b]]
                 for b in range(wl.num_seqs)]
        ids, cu = inputs.pack(parts)
        yield ids, cu, lo.astype(np.int32)


@pytest.mark.parametrize("cfg,size", [(1, 16), (2, 16), (2, 100), (3, 1000), (5, 4096)])
@pytest.mark.parametrize("rule", ["canvas", "qwen_vl", "planes_1d"])
def test_chunked_prefill_bit_exact(cuda_device, cfg, size, rule):
    wl = inputs.make_config(cfg, with_qk=False)
    dev = cuda_device
    b = wl.num_seqs
    g_state = (t32(np.full(b, 1 << 30), dev), t32(np.zeros(b), dev))
    o_state = (np.full(b, 1 << 30, np.int32), np.zeros(b, np.int32))
    got_all, want_all = [], []
    for ids, cu, off in chunk_batches(wl, size):
        g_out = (torch.empty((3, ids.size), dtype=torch.int32, device=dev),
                 torch.empty(b, dtype=torch.int32, device=dev),
                 torch.empty(b, dtype=torch.int32, device=dev))
        pos, s, a = cmr.positions_chunk(t32(ids, dev), t32(cu, dev), t32(off, dev), g_state,
                                        rule, out=g_out)
        wpos, ws, wa = oracle.positions_chunk(ids, cu, MARK, rule, off, *o_state)
        np.testing.assert_array_equal(pos.cpu().numpy(), wpos)
        np.testing.assert_array_equal(s.cpu().numpy(), ws)
        np.testing.assert_array_equal(a.cpu().numpy(), wa)
        g_state, o_state = (s, a), (ws, wa)
        got_all.append(pos.cpu().numpy())
    if rule == "canvas":
        # the chunks together give the whole-prompt planes
        whole = oracle.positions(wl.ids, wl.cu_seqlens, MARK)[0]
        per_prompt = {b_: [] for b_ in range(b)}
        for (ids, cu, off), pos in zip(chunk_batches(wl, size), got_all):
            for b_ in range(b):
                per_prompt[b_].append(pos[:, cu[b_]:cu[b_ + 1]])
        for b_ in range(b):
            np.testing.assert_array_equal(np.concatenate(per_prompt[b_], axis=1),
                                          whole[:, wl.cu_seqlens[b_]:wl.cu_seqlens[b_ + 1]])


def test_rules_on_whole_prompts(cuda_device):
    for cfg in (2, 3):
        wl = inputs.make_config(cfg, with_qk=False)
        for rule in ("canvas", "qwen_vl", "planes_1d"):
            pos, s, a = cmr.positions_chunk(t32(wl.ids, cuda_device), t32(wl.cu_seqlens, cuda_device),
                                            rule=rule)
            wpos, ws, wa = oracle.positions_chunk(wl.ids, wl.cu_seqlens, MARK, rule)
            np.testing.assert_array_equal(pos.cpu().numpy(), wpos)
            np.testing.assert_array_equal(s.cpu().numpy(), ws)
            np.testing.assert_array_equal(a.cpu().numpy(), wa)


def test_overlapping_state_is_rejected(cuda_device):
    ids = t32(np.zeros(8), cuda_device)
    cu = t32([0, 8], cuda_device)
    st = t32([1 << 30], cuda_device)
    am = t32([0], cuda_device)
    with pytest.raises(cmr.CmrError):
        cmr.positions_chunk(ids, cu, state=(st, am),
                            out=(torch.empty((3, 8), dtype=torch.int32, device=cuda_device), st, am))


@pytest.mark.parametrize("cfg", [1, 2, 3, 5])
def test_shift_rotate_equals_pos_rotate_bit_for_bit(cuda_device, cfg):
    wl = inputs.make_config(cfg, device=cuda_device)
    dev = cuda_device
    ids, cu = t32(wl.ids, dev), t32(wl.cu_seqlens, dev)
    pos, s, a = cmr.positions(ids, cu)
    q2, k2 = wl.q.clone(), wl.k.clone()
    cmr.rotate_qk(wl.q, wl.k, pos)
    cmr.rotate_qk_shift(q2, k2, s, a, cu_seqlens=cu)
    torch.cuda.synchronize()
    assert torch.equal(wl.q.view(torch.int16), q2.view(torch.int16))
    assert torch.equal(wl.k.view(torch.int16), k2.view(torch.int16))


def test_decode_step_in_one_launch(cuda_device):
    wl = inputs.make_config(4, device=cuda_device)
    dev = cuda_device
    _, s, a = cmr.positions(t32(wl.ids, dev), t32(wl.cu_seqlens, dev))
    cache_len = t32(wl.cache_len, dev)
    q_in, k_in = bits(wl.q), bits(wl.k)
    q2, k2 = wl.q.clone(), wl.k.clone()
    cmr.rotate_qk_shift(wl.q, wl.k, s, a, pos_offset=cache_len)          # one launch
    cmr.rotate_qk(q2, k2, cmr.positions_step(cache_len, s, a))           # two launches
    torch.cuda.synchronize()
    assert torch.equal(wl.q.view(torch.int16), q2.view(torch.int16))
    p = oracle.positions_step(wl.cache_len, s.cpu().numpy(), a.cpu().numpy())
    assert_bf16_close(bits(wl.q), oracle.rotate_bf16(q_in, p), "decode q")
    assert_bf16_close(bits(wl.k), oracle.rotate_bf16(k_in, p), "decode k")


def test_shift_rotate_on_chunks_at_offsets(cuda_device):
    # the second chunk of every prompt of the varlen workload, rotated with the
    # state the first chunk left
    wl = inputs.make_config(2, device=cuda_device)
    dev = cuda_device
    first = [wl.ids[wl.cu_seqlens[b]: wl.cu_seqlens[b] + 60] for b in range(wl.num_seqs)]
    rest = [wl.ids[wl.cu_seqlens[b] + 60: wl.cu_seqlens[b + 1]] for b in range(wl.num_seqs)]
    ids1, cu1 = inputs.pack(first)
    ids2, cu2 = inputs.pack(rest)
    _, s, a = cmr.positions_chunk(t32(ids1, dev), t32(cu1, dev))
    off = t32(np.full(wl.num_seqs, 60), dev)
    n2 = ids2.size
    g = torch.Generator(device=dev).manual_seed(9)
    q = torch.randn((1, n2, 8, 256), generator=g, device=dev).to(torch.bfloat16)
    k = torch.randn((1, n2, 2, 256), generator=g, device=dev).to(torch.bfloat16)
    q_in, k_in = bits(q), bits(k)
    cmr.rotate_qk_shift(q, k, s, a, cu_seqlens=t32(cu2, dev), pos_offset=off)
    torch.cuda.synchronize()
    whole = oracle.positions(wl.ids, wl.cu_seqlens, MARK)[0]
    p = np.concatenate([whole[:, wl.cu_seqlens[b] + 60: wl.cu_seqlens[b + 1]]
                        for b in range(wl.num_seqs)], axis=1)
    assert_bf16_close(bits(q), oracle.rotate_bf16(q_in, p), "chunk q")
    assert_bf16_close(bits(k), oracle.rotate_bf16(k_in, p), "chunk k")


def test_shift_rotate_with_empty_prompts(cuda_device):
    rng = np.random.default_rng(6)
    lens, origins = [0, 5, 0, 0, 90, 1, 0], [-1, 1, -1, -1, 20, 0, -1]
    prompts = [inputs.prompt_ids(rng, n, o) for n, o in zip(lens, origins)]
    ids, cu = inputs.pack(prompts)
    dev = cuda_device
    pos, s, a = cmr.positions(t32(ids, dev), t32(cu, dev))
    n = ids.size
    g = torch.Generator(device=dev).manual_seed(2)
    q = torch.randn((3, n, 8, 256), generator=g, device=dev).to(torch.bfloat16)
    k = torch.randn((3, n, 2, 256), generator=g, device=dev).to(torch.bfloat16)
    q2, k2 = q.clone(), k.clone()
    cmr.rotate_qk(q, k, pos)
    cmr.rotate_qk_shift(q2, k2, s, a, cu_seqlens=t32(cu, dev))
    torch.cuda.synchronize()
    assert torch.equal(q.view(torch.int16), q2.view(torch.int16))
    assert torch.equal(k.view(torch.int16), k2.view(torch.int16))


def test_graph_capture_replays_bit_for_bit(cuda_device):
    # the library enqueues kernels only (no sync, no allocation), so a CUDA
    # graph of positions + rotate replays exactly what eager launches do
    dev = cuda_device
    wl = inputs.make_config(2, device=dev)
    ids, cu = t32(wl.ids, dev), t32(wl.cu_seqlens, dev)
    q0, k0 = wl.q.clone(), wl.k.clone()
    pos = torch.empty((3, wl.n_tokens), dtype=torch.int32, device=dev)
    st = torch.empty(wl.num_seqs, dtype=torch.int32, device=dev)
    am = torch.empty(wl.num_seqs, dtype=torch.int32, device=dev)
    q, k = q0.clone(), k0.clone()
    cmr.positions(ids, cu, out=(pos, st, am))
    cmr.rotate_qk(q, k, pos)
    torch.cuda.synchronize()
    eager = (pos.clone(), q.clone(), k.clone())
    q.copy_(q0)
    k.copy_(k0)
    pos.zero_()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cmr.positions(ids, cu, out=(pos, st, am))
        cmr.rotate_qk(q, k, pos)
    q.copy_(q0)
    k.copy_(k0)
    pos.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(pos, eager[0])
    assert torch.equal(q.view(torch.int16), eager[1].view(torch.int16))
    assert torch.equal(k.view(torch.int16), eager[2].view(torch.int16))


@pytest.mark.parametrize("hq,hk,head_dim,rot_dim,sections,L", [
    (16, 4, 256, 64, (11, 11, 10), 3), (0, 2, 256, 64, (11, 11, 10), 2),
    (8, 0, 128, 32, (6, 5, 5), 1), (4, 4, 256, 256, (44, 42, 42), 2),
])
def test_shift_and_cache_forms_on_other_shapes(cuda_device, hq, hk, head_dim, rot_dim, sections, L):
    dev = cuda_device
    rng = np.random.default_rng(hq * 7 + hk)
    lens = [37, 0, 120, 5, 200]
    prompts = [inputs.prompt_ids(rng, n, o) for n, o in zip(lens, [3, -1, 0, -1, 50])]
    ids, cu_np = inputs.pack(prompts)
    n = ids.size
    cu = t32(cu_np, dev)
    pos, s, a = cmr.positions(t32(ids, dev), cu)
    g = torch.Generator(device=dev).manual_seed(3)
    mk = lambda h: torch.randn((L, n, h, head_dim), generator=g, device=dev).to(torch.bfloat16) if h else None
    q, k, v = mk(hq), mk(hk), mk(hk)
    qa = q.clone() if hq else None
    ka = k.clone() if hk else None
    cmr.rotate_qk(qa, ka, pos, 1e7, sections, rot_dim)
    qb = q.clone() if hq else None
    kb = k.clone() if hk else None
    cmr.rotate_qk_shift(qb, kb, s, a, cu_seqlens=cu, theta=1e7, sections=sections, rot_dim=rot_dim)
    qc = q.clone() if hq else None
    kc = vc = None
    if hk:
        kc = torch.zeros((L, len(lens), hk, 256, head_dim), dtype=torch.bfloat16, device=dev)
        vc = torch.zeros_like(kc)
    cmr.rotate_qk_cache(qc, k, v, s, a, kc, vc, cu_seqlens=cu, theta=1e7, sections=sections,
                        rot_dim=rot_dim)
    torch.cuda.synchronize()
    if hq:
        assert torch.equal(qa.view(torch.int16), qb.view(torch.int16))
        assert torch.equal(qa.view(torch.int16), qc.view(torch.int16))
        p = pos.cpu().numpy()
        assert_bf16_close(bits(qa), oracle.rotate_bf16(bits(q), p, 1e7, sections, rot_dim), "q")
    if hk:
        assert torch.equal(ka.view(torch.int16), kb.view(torch.int16))
        for b_ in range(len(lens)):
            lo, hi = int(cu_np[b_]), int(cu_np[b_ + 1])
            got_k = kc[:, b_, :, :hi - lo].permute(0, 2, 1, 3)
            got_v = vc[:, b_, :, :hi - lo].permute(0, 2, 1, 3)
            assert torch.equal(got_k.contiguous().view(torch.int16), ka[:, lo:hi].view(torch.int16))
            assert torch.equal(got_v.contiguous().view(torch.int16), v[:, lo:hi].view(torch.int16))


@pytest.mark.parametrize("layers", [1, 3])
def test_staged_shift_rotate_on_chunks_at_offsets(cuda_device, layers):
    # second chunks of 4 prompts of 8,192 tokens, split so that two frames lie
    # in the first chunks and two (one cut off by the prompt's end) in the
    # second: 19,668 tokens, enough for the TMA-staged kernel.  The second
    # chunks' state comes from cmr_positions_chunk at their offsets; the rotate
    # derives every token's planes from it in the kernel.
    dev = cuda_device
    wl = inputs.make_batch([8192] * 4, [6, 2500, 5000, 8150], with_qk=False)
    cut = [2000, 2600, 4000, 4500]
    first = [wl.ids[wl.cu_seqlens[b]: wl.cu_seqlens[b] + cut[b]] for b in range(4)]
    rest = [wl.ids[wl.cu_seqlens[b] + cut[b]: wl.cu_seqlens[b + 1]] for b in range(4)]
    ids1, cu1 = inputs.pack(first)
    ids2, cu2 = inputs.pack(rest)
    _, s1, a1 = cmr.positions_chunk(t32(ids1, dev), t32(cu1, dev))
    off = t32(np.array(cut), dev)
    pos2, s, a = cmr.positions_chunk(t32(ids2, dev), t32(cu2, dev), pos_offset=off,
                                     state=(s1, a1))
    n2 = ids2.size
    assert cmr.rotate_qk_kernel(n2, layers, 8, 2) == "rotate_qk_staged_kernel"
    q = inputs.random_qk((layers, n2, 8, 256), 21, dev)
    k = inputs.random_qk((layers, n2, 2, 256), 22, dev)
    q_in, k_in = bits(q), bits(k)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    cmr.rotate_qk_shift(q, k, s, a, cu_seqlens=t32(cu2, dev), pos_offset=off,
                        device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    whole = oracle.positions(wl.ids, wl.cu_seqlens, MARK)[0]
    p = np.concatenate([whole[:, wl.cu_seqlens[b] + cut[b]: wl.cu_seqlens[b + 1]]
                        for b in range(4)], axis=1)
    np.testing.assert_array_equal(pos2.cpu().numpy(), p)
    assert_bf16_close(bits(q), oracle.rotate_bf16(q_in, p), "staged chunk q")
    assert_bf16_close(bits(k), oracle.rotate_bf16(k_in, p), "staged chunk k")


FIRST_CALL_IN_CAPTURE = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
from vlm_decoder_positional_b200 import cmr, inputs
dev = torch.device("cuda", 0)
L, n = 2, 20000
assert cmr.rotate_qk_kernel(n, L, 8, 2) == "rotate_qk_staged_kernel"
q0 = inputs.random_qk((L, n, 8, 256), 3, dev)
k0 = inputs.random_qk((L, n, 2, 256), 4, dev)
pos = torch.randint(0, 40000, (3, n), dtype=torch.int32, device=dev)
q, k = q0.clone(), k0.clone()
status = torch.zeros(1, dtype=torch.int32, device=dev)
torch.cuda.synchronize()
g = torch.cuda.CUDAGraph()
with torch.cuda.graph(g):          # the process's first library call
    cmr.rotate_qk(q, k, pos, device_status=status)
q.copy_(q0); k.copy_(k0)
g.replay()
torch.cuda.synchronize()
qe, ke = q0.clone(), k0.clone()
cmr.rotate_qk(qe, ke, pos, device_status=status)
torch.cuda.synchronize()
assert int(status.item()) == 0
assert torch.equal(q.view(torch.int16), qe.view(torch.int16))
assert torch.equal(k.view(torch.int16), ke.view(torch.int16))
print("ok")
"""


def test_first_call_of_a_process_inside_graph_capture(cuda_device, tmp_path):
    # a fresh process whose very first library call is a staged rotate being
    # captured into a CUDA graph: the launch path makes no call that a capture
    # forbids, and the replay equals an eager launch bit for bit
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    script = tmp_path / "first_call.py"
    script.write_text(FIRST_CALL_IN_CAPTURE)
    out = subprocess.run([sys.executable, str(script), root], capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0 and out.stdout.strip().endswith("ok"), out.stderr[-2000:]
