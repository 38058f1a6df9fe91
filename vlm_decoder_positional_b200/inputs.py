"""Seeded synthetic workloads for canvas M-RoPE.

This module builds inputs only: token ids with image frames laid out as the
processor lays them out, packed cu_seqlens, and bf16 Q/K drawn from N(0, 1).
It holds none of the method's arithmetic (no planes, no start/amount, no
rotation), so the CUDA path and the oracle can both consume what it makes.

Prompt layout (HF card mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI, "Prompt" and the
engine I/O table): ``<image>`` (248078) at the frame origin O, then 64 image
rows written as V + k (V = 248,094, k = 0..63), then ``</image>`` (248079) and
the template's "\\n" (198); text ids elsewhere.  Frames that run past the end
of a sequence are truncated.

The five named workloads mirror the shapes, sizes and value distributions of
the pages' use: one 448x448 image per prompt, the 6 full-attention layers of
the 24-layer hybrid decoder, 8 query heads and 2 KV heads of width 256.
"""
from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np
import torch

VOCAB = 248094          # text vocabulary; image rows are written as VOCAB + k
IMAGE_TOKEN_ID = 248078  # <image>
IMAGE_END_ID = 248079    # </image>
IMAGE_PAD_ID = 248056    # <|image_pad|>, the processor's placeholder for a row
NEWLINE_ID = 198         # "\n"
ROWS_PER_IMAGE = 64      # 448x448 thumbnail -> 64 merged rows

HQ, HK, HEAD_DIM = 8, 2, 256
ROT_DIM, THETA, SECTIONS = 64, 1e7, (11, 11, 10)
BASE_SEED = 20261013


@dataclass
class Workload:
    name: str
    ids: np.ndarray             # int32 [N]
    cu_seqlens: np.ndarray      # int32 [B + 1]
    frame_origin: np.ndarray    # int32 [B]: index of <image> in each prompt, -1 if none
    q: Optional[torch.Tensor]   # bf16 [L, T, HQ, D]
    k: Optional[torch.Tensor]   # bf16 [L, T, HK, D]
    num_layers: int = 1
    hq: int = HQ
    hk: int = HK
    head_dim: int = HEAD_DIM
    rot_dim: int = ROT_DIM
    theta: float = THETA
    sections: tuple = SECTIONS
    image_token_id: int = IMAGE_TOKEN_ID
    # decode workloads: the new token of prompt b sits at absolute index
    # cache_len[b] (the prompt's length); Q/K then hold one token per prompt.
    cache_len: Optional[np.ndarray] = None
    seed: int = 0
    meta: dict = field(default_factory=dict)

    @property
    def n_tokens(self) -> int:
        return int(self.ids.shape[0])

    @property
    def num_seqs(self) -> int:
        return int(self.cu_seqlens.shape[0]) - 1

    @property
    def qk_tokens(self) -> int:
        return int(self.q.shape[1]) if self.q is not None else 0


def text_ids(rng: np.random.Generator, n: int, avoid=(IMAGE_TOKEN_ID,)) -> np.ndarray:
    """Uniform text ids in [0, VOCAB), redrawn where they hit an id in ``avoid``."""
    ids = rng.integers(0, VOCAB, size=n, dtype=np.int64)
    bad = np.isin(ids, avoid)
    while bad.any():
        ids[bad] = rng.integers(0, VOCAB, size=int(bad.sum()), dtype=np.int64)
        bad = np.isin(ids, avoid)
    return ids.astype(np.int32)


def frame_ids(row_ids: str = "v_plus_k", grid_side: int = 8) -> np.ndarray:
    """The ids of one image frame: <image>, grid_side^2 rows, </image>, "\\n"
    (67 ids for the 448x448 thumbnail's 8x8 grid)."""
    n_rows = grid_side * grid_side
    if row_ids == "v_plus_k":
        rows = VOCAB + np.arange(n_rows)
    elif row_ids == "pad":
        rows = np.full(n_rows, IMAGE_PAD_ID)
    else:
        raise ValueError(row_ids)
    return np.concatenate([[IMAGE_TOKEN_ID], rows, [IMAGE_END_ID, NEWLINE_ID]]).astype(np.int32)


def prompt_ids(rng: np.random.Generator, length: int, origin: int,
               row_ids: str = "v_plus_k") -> np.ndarray:
    """One prompt of ``length`` ids; a frame starts at ``origin`` (none if < 0)."""
    ids = text_ids(rng, length)
    if origin >= 0:
        fr = frame_ids(row_ids)
        end = min(length, origin + fr.shape[0])
        if origin < length:
            ids[origin:end] = fr[: end - origin]
    return ids


def prompt_ids_frames(rng: np.random.Generator, length: int, origins: Sequence[int],
                      grid_side: int = 8) -> np.ndarray:
    """One prompt of ``length`` ids with a frame of grid_side^2 rows starting at
    each of ``origins`` (laid in order, each truncated by the end of the prompt
    and overwritten from the next origin on if they overlap)."""
    ids = text_ids(rng, length)
    fr = frame_ids("v_plus_k", grid_side)
    for o in sorted(origins):
        if 0 <= o < length:
            end = min(length, o + fr.shape[0])
            ids[o:end] = fr[: end - o]
    return ids


def spaced_origins(rng: np.random.Generator, count: int, lo: int, hi: int,
                   gap: int) -> list:
    """``count`` sorted origins in [lo, hi] at least ``gap`` apart (uniform
    over such sets: draw count points in [lo, hi - (count-1) gap], sort,
    spread)."""
    span = hi - (count - 1) * gap
    if span < lo:
        raise ValueError("no room for that many spaced origins")
    base = np.sort(rng.integers(lo, span + 1, size=count))
    return [int(b + i * gap) for i, b in enumerate(base)]


def pack(prompts: Sequence[np.ndarray]):
    lens = np.array([p.shape[0] for p in prompts], dtype=np.int64)
    cu = np.zeros(len(prompts) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lens)
    if cu[-1] > np.iinfo(np.int32).max:
        raise ValueError("packed batch exceeds int32 token indices")
    ids = np.concatenate(prompts).astype(np.int32) if prompts else np.zeros(0, np.int32)
    return ids, cu.astype(np.int32)


def random_qk(shape, seed: int, device="cpu", outlier_frac: float = 0.0,
              outlier_scale: float = 100.0) -> torch.Tensor:
    """bf16 N(0, 1) values (fp32 draws rounded to bf16, nearest-even), drawn one
    layer at a time; a Bernoulli(outlier_frac) mask scales values by
    outlier_scale before rounding."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    for l in range(shape[0]):
        x = torch.randn(shape[1:], generator=g, device=device, dtype=torch.float32)
        if outlier_frac > 0:
            m = torch.rand(shape[1:], generator=g, device=device) < outlier_frac
            x = torch.where(m, x * outlier_scale, x)
        out[l].copy_(x.to(torch.bfloat16))
        del x
    return out


def make_batch(lengths, origins, num_layers=1, hq=HQ, hk=HK, head_dim=HEAD_DIM,
               seed=BASE_SEED, device="cpu", outlier_frac=0.0, row_ids="v_plus_k",
               with_qk=True, name="custom", **params) -> Workload:
    """A packed prefill batch with one (possibly truncated) frame per prompt."""
    rng = np.random.default_rng(seed)
    prompts = [prompt_ids(rng, int(n), int(o), row_ids) for n, o in zip(lengths, origins)]
    ids, cu = pack(prompts)
    n = ids.shape[0]
    q = k = None
    if with_qk:
        q = random_qk((num_layers, n, hq, head_dim), seed + 1, device, outlier_frac)
        k = random_qk((num_layers, n, hk, head_dim), seed + 2, device, outlier_frac)
    origin = np.array([o if o < n_ else -1 for n_, o in zip(lengths, origins)], dtype=np.int32)
    return Workload(name=name, ids=ids, cu_seqlens=cu, frame_origin=origin, q=q, k=k,
                    num_layers=num_layers, hq=hq, hk=hk, head_dim=head_dim, seed=seed,
                    **params)


CONFIG_NAMES = {
    1: "c1_single_prompt_80",
    2: "c2_varlen_16x96-512",
    3: "c3_64x4096_outliers",
    4: "c4_decode_1024",
    5: "c5_6layers_32x8192",
    6: "c6_multiframe_256x65536",  # the multi-frame positions' workload (not a rotate config)
}


def make_config(index: int, device="cpu", with_qk=True, seed=None) -> Workload:
    """The five synthetic workloads (1-based index, seed = 20261013 + index), and
    6: the multi-frame positions' workload (make_frames_workload)."""
    seed = BASE_SEED + index if seed is None else seed
    rng = np.random.default_rng(seed)
    name = CONFIG_NAMES[index]
    if index == 1:
        # one 80-token prompt: frame at 6..72, text from 73
        return make_batch([80], [6], seed=seed, device=device, with_qk=with_qk, name=name)
    if index == 2:
        # 16 prompts, lengths U[96, 512]; half with O in {6, 17}, half with O ~ U[0, 40]
        lengths = rng.integers(96, 513, size=16)
        fixed = rng.choice(np.array([6, 17]), size=8)
        free = rng.integers(0, 41, size=8)
        origins = np.concatenate([fixed, free])[rng.permutation(16)]
        return make_batch(lengths, origins, seed=seed, device=device, with_qk=with_qk,
                          name=name)
    if index == 3:
        # 64 x 4096; 48 prompts with a frame at O ~ U[0, 3000], 16 text-only;
        # 5 % of Q/K values scaled x100 before rounding
        origins = rng.integers(0, 3001, size=64)
        text_only = rng.permutation(64)[:16]
        origins[text_only] = -1
        return make_batch([4096] * 64, origins, seed=seed, device=device, with_qk=with_qk,
                          outlier_frac=0.05, name=name)
    if index == 4:
        # decode: 1024 prompts of prior length U[73, 32768], each with a frame at
        # O ~ U[0, prior - 67]; one new token per prompt at index prior
        prior = rng.integers(73, 32769, size=1024)
        origins = np.array([rng.integers(0, p - 67 + 1) for p in prior])
        wl = make_batch(prior, origins, seed=seed, device=device, with_qk=False, name=name)
        wl.cache_len = prior.astype(np.int32)
        if with_qk:
            wl.q = random_qk((1, 1024, HQ, HEAD_DIM), seed + 1, device)
            wl.k = random_qk((1, 1024, HK, HEAD_DIM), seed + 2, device)
        return wl
    if index == 5:
        # 6 full-attention layers per launch; 32 x 8192, one frame each at O ~ U[0, 6000]
        origins = rng.integers(0, 6001, size=32)
        return make_batch([8192] * 32, origins, num_layers=6, seed=seed, device=device,
                          with_qk=with_qk, name=name)
    if index == 6:
        return make_frames_workload(seed=seed, device=device)  # positions only: no Q/K
    raise ValueError("config index must be 1..6")


def make_frames_workload(num_prompts=256, length=65536, frames=32, grid_side=8, seed=None,
                         device="cpu", with_qk=False, min_text=16) -> Workload:
    """Prompts that each hold several frames on a grid_side x grid_side grid (a
    thumbnail and its slices, or several images), with at least ``min_text``
    text tokens between frames: the workload of the multi-frame positions.
    The default, 256 prompts x 65,536 tokens with 32 frames each (16.8 M
    tokens, 268 MB of ids and planes), is larger than the L2.  Q/K are not
    drawn unless asked for (one layer)."""
    seed = BASE_SEED + 6 if seed is None else seed
    rng = np.random.default_rng(seed)
    F = grid_side * grid_side + 3
    prompts, first = [], []
    for _ in range(num_prompts):
        origins = spaced_origins(rng, frames, 0, length - F, F + min_text)
        prompts.append(prompt_ids_frames(rng, length, origins, grid_side))
        first.append(origins[0])
    ids, cu = pack(prompts)
    n = ids.shape[0]
    q = k = None
    if with_qk:
        q = random_qk((1, n, HQ, HEAD_DIM), seed + 1, device)
        k = random_qk((1, n, HK, HEAD_DIM), seed + 2, device)
    name = (f"c6_multiframe_{num_prompts}x{length}_{frames}frames_s{grid_side}"
            if (num_prompts, length, frames, grid_side) != (256, 65536, 32, 8)
            else CONFIG_NAMES[6])
    return Workload(name=name, ids=ids, cu_seqlens=cu,
                    frame_origin=np.array(first, dtype=np.int32), q=q, k=k, seed=seed,
                    meta={"grid_side": grid_side, "frames_per_prompt": frames})
