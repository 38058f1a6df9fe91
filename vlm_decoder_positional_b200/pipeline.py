"""Canvas M-RoPE on host-resident batches: copies overlapped with the kernels.

For callers whose ids and Q/K live in (pinned) host memory.  The batch is cut
into chunks of whole prompts (a prompt is never split, so each chunk's planes
need nothing from another chunk).  Each chunk goes host -> device on one stream,
through cmr_positions_rotate_qk (the positions kernels, then the rotation
overlapping them) on a second, and back on a third, over a
ring of `depth` device buffers, so the host-to-device copy of one chunk, the
kernels of the next and the device-to-host copy of a third run at the same
time (PCIe moves both directions at once).  Only the rotated dims of each head
row cross PCIe (cmr_copy_rotated_dims, a pitched copy): the rest of Q/K is
neither read nor written by the method.  Only copies, streams and events live
here; every step of the method runs in the library's kernels.
"""
from typing import List, Tuple

import numpy as np
import torch

from . import cmr


def prompt_chunks(cu_seqlens: np.ndarray, max_tokens: int) -> List[Tuple[int, int]]:
    """Contiguous prompt ranges [s0, s1) of at most max_tokens tokens each (a
    longer prompt forms a chunk of its own)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    b = len(cu) - 1
    out, s0 = [], 0
    while s0 < b:
        s1 = s0 + 1
        while s1 < b and cu[s1 + 1] - cu[s0] <= max_tokens:
            s1 += 1
        out.append((s0, s1))
        s0 = s1
    return out


class HostPipeline:
    """Reusable device buffers and streams for batches of a fixed shape family.

    q_host / k_host: pinned bf16 [L, N, hq, D] / [L, N, hk, D], rotated in
    place; ids_host / cu_host: int32 [N] / [B + 1]; pos_host: pinned int32
    [3, N]; start_host / amount_host: pinned int32 [B]."""

    def __init__(self, device, num_layers, hq, hk, head_dim, max_chunk_tokens, max_chunk_seqs,
                 depth=3):
        self.dev = torch.device(device)
        self.L, self.hq, self.hk, self.D = num_layers, hq, hk, head_dim
        self.max_tokens, self.max_seqs, self.depth = max_chunk_tokens, max_chunk_seqs, depth
        T, S = max_chunk_tokens, max_chunk_seqs
        kw = dict(device=self.dev)
        self.q = [torch.empty(num_layers * T * hq * head_dim, dtype=torch.bfloat16, **kw)
                  for _ in range(depth)]
        self.k = [torch.empty(num_layers * T * hk * head_dim, dtype=torch.bfloat16, **kw)
                  for _ in range(depth)]
        self.ids = [torch.empty(T, dtype=torch.int32, **kw) for _ in range(depth)]
        self.cu = [torch.empty(S + 1, dtype=torch.int32, **kw) for _ in range(depth)]
        self.cu_stage = [torch.empty(S + 1, dtype=torch.int32, pin_memory=True)
                         for _ in range(depth)]
        self.pos = [torch.empty(3 * T, dtype=torch.int32, **kw) for _ in range(depth)]
        self.start = [torch.empty(S, dtype=torch.int32, **kw) for _ in range(depth)]
        self.amount = [torch.empty(S, dtype=torch.int32, **kw) for _ in range(depth)]
        self.s_in = torch.cuda.Stream(self.dev)
        self.s_run = torch.cuda.Stream(self.dev)
        self.s_out = torch.cuda.Stream(self.dev)
        self.copied_in = [torch.cuda.Event() for _ in range(depth)]
        self.computed = [torch.cuda.Event() for _ in range(depth)]
        self.copied_out = [torch.cuda.Event() for _ in range(depth)]
        self.used = [False] * depth

    def run(self, ids_host, cu_host, q_host, k_host, pos_host, start_host, amount_host,
            theta=1e7, sections=(11, 11, 10), rot_dim=64,
            image_token_id=cmr.IMAGE_TOKEN_ID, chunk_tokens=None):
        """Planes and rotation of a whole host batch; returns when the results are
        enqueued (synchronise the device, or the three streams, before reading)."""
        L, hq, hk, D = self.L, self.hq, self.hk, self.D
        cu_np = np.asarray(cu_host.numpy() if isinstance(cu_host, torch.Tensor) else cu_host,
                           dtype=np.int64)
        n_all = int(cu_np[-1])
        chunks = prompt_chunks(cu_np, chunk_tokens or self.max_tokens)
        main = torch.cuda.current_stream(self.dev)
        for st in (self.s_in, self.s_run, self.s_out):
            st.wait_stream(main)
        for i, (s0, s1) in enumerate(chunks):
            r = i % self.depth
            t0, t1 = int(cu_np[s0]), int(cu_np[s1])
            n, b = t1 - t0, s1 - s0
            if n > self.max_tokens or b > self.max_seqs:
                raise ValueError("a prompt is longer than the pipeline's chunk buffers")
            q_d = self.q[r][:L * n * hq * D].view(L, n, hq, D)
            k_d = self.k[r][:L * n * hk * D].view(L, n, hk, D)
            pos_d = self.pos[r][:3 * n].view(3, n)
            if self.used[r]:
                # the host rewrites this slot's pinned staging buffer: its last
                # host-to-device copy must have finished
                self.copied_in[r].synchronize()
            self.cu_stage[r][:b + 1].copy_(torch.from_numpy((cu_np[s0:s1 + 1] - t0).astype(np.int32)))
            with torch.cuda.stream(self.s_in):
                if self.used[r]:
                    self.s_in.wait_event(self.copied_out[r])  # ring slot free again
                self.cu[r][:b + 1].copy_(self.cu_stage[r][:b + 1], non_blocking=True)
                self.ids[r][:n].copy_(ids_host[t0:t1], non_blocking=True)
                for l in range(L):  # only the rotated dims of each head row
                    cmr.copy_rotated_dims(q_d[l], q_host[l, t0:t1], rot_dim, self.s_in)
                    cmr.copy_rotated_dims(k_d[l], k_host[l, t0:t1], rot_dim, self.s_in)
                self.copied_in[r].record(self.s_in)
            with torch.cuda.stream(self.s_run):
                self.s_run.wait_event(self.copied_in[r])
                cmr.positions_rotate_qk(self.ids[r][:n], self.cu[r][:b + 1], q_d, k_d, theta,
                                        sections, rot_dim, image_token_id,
                                        out=(pos_d, self.start[r][:b], self.amount[r][:b]))
                self.computed[r].record(self.s_run)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.computed[r])
                for l in range(L):
                    cmr.copy_rotated_dims(q_host[l, t0:t1], q_d[l], rot_dim, self.s_out)
                    cmr.copy_rotated_dims(k_host[l, t0:t1], k_d[l], rot_dim, self.s_out)
                for plane in range(3):
                    pos_host[plane, t0:t1].copy_(pos_d[plane], non_blocking=True)
                start_host[s0:s1].copy_(self.start[r][:b], non_blocking=True)
                amount_host[s0:s1].copy_(self.amount[r][:b], non_blocking=True)
                self.copied_out[r].record(self.s_out)
            self.used[r] = True
        for st in (self.s_in, self.s_run, self.s_out):
            main.wait_stream(st)
        return n_all
