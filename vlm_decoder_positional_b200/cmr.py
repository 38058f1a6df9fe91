"""Python binding of libcmr (include/cmr.h): argument marshalling only.

Every step of the path runs in the library's CUDA kernels; this module checks
tensor dtypes/devices/shapes, allocates outputs with torch when the caller does
not pass them, and forwards raw pointers and the current CUDA stream.  There
is no fallback: if libcmr.so is missing or a call fails, it raises.
"""
import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcmr.so")

CMR_OK, CMR_EINVAL, CMR_ECUDA, CMR_EUNSUPPORTED = 0, 1, 2, 3
CMR_DEVICE_BAD_CU_SEQLENS = 1
CMR_DEVICE_CACHE_RANGE = 2
CMR_DEVICE_WAIT_TIMEOUT = 4
RULES = {"canvas": 0, "qwen_vl": 1, "planes_1d": 2}
TEXT_ONLY_START = 1 << 30

IMAGE_TOKEN_ID = 248078

# name -> (restype, argtypes); mirrors include/cmr.h
_i32p = ctypes.c_void_p
SIGNATURES = {
    "cmr_positions": (ctypes.c_int, [_i32p, _i32p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32,
                                     _i32p, _i32p, _i32p, _i32p, ctypes.c_void_p]),
    "cmr_positions_chunk": (ctypes.c_int, [_i32p, _i32p, ctypes.c_int32, ctypes.c_int64,
                                           ctypes.c_int32, ctypes.c_int32, _i32p, _i32p, _i32p,
                                           _i32p, _i32p, _i32p, _i32p, ctypes.c_void_p]),
    "cmr_positions_frames": (ctypes.c_int, [_i32p, _i32p, ctypes.c_int32, ctypes.c_int64,
                                            ctypes.c_int32, ctypes.c_int32, _i32p, _i32p, _i32p,
                                            ctypes.c_void_p, ctypes.c_size_t, _i32p,
                                            ctypes.c_void_p]),
    "cmr_positions_frames_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int32, ctypes.c_int64]),
    "cmr_positions_frames_noalloc": (ctypes.c_int, [_i32p, _i32p, ctypes.c_int32, ctypes.c_int64,
                                                    ctypes.c_int32, ctypes.c_int32, _i32p, _i32p,
                                                    _i32p, _i32p, ctypes.c_void_p]),
    "cmr_positions_step": (ctypes.c_int, [_i32p, _i32p, _i32p, ctypes.c_int32, _i32p,
                                          ctypes.c_void_p]),
    "cmr_rotate_qk_shift": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, _i32p,
                                           ctypes.c_int32, _i32p, _i32p, _i32p, ctypes.c_int64,
                                           ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.c_int32, ctypes.c_double,
                                           ctypes.POINTER(ctypes.c_int32), ctypes.c_int32,
                                           _i32p, ctypes.c_void_p]),
    "cmr_rotate_qk_cache": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                           _i32p, ctypes.c_int32, _i32p, _i32p, _i32p,
                                           ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.c_int32, ctypes.c_int32, ctypes.c_double,
                                           ctypes.POINTER(ctypes.c_int32), ctypes.c_int32,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                           ctypes.c_int32, _i32p, _i32p, ctypes.c_void_p]),
    "cmr_rotate_qk": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, _i32p, ctypes.c_int64,
                                     ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                     ctypes.c_int32, ctypes.c_double,
                                     ctypes.POINTER(ctypes.c_int32), ctypes.c_int32,
                                     _i32p, ctypes.c_void_p]),
    "cmr_positions_rotate_qk": (ctypes.c_int, [_i32p, _i32p, ctypes.c_int32, ctypes.c_int64,
                                               ctypes.c_int32, _i32p, _i32p, _i32p,
                                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                               ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                               ctypes.c_double, ctypes.POINTER(ctypes.c_int32),
                                               ctypes.c_int32, _i32p, ctypes.c_void_p]),
    "cmr_positions_rotate_qk_host": (ctypes.c_int, [_i32p, _i32p, ctypes.c_int32, ctypes.c_int64,
                                               ctypes.c_int32, _i32p, _i32p, _i32p,
                                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                               ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                               ctypes.c_double, ctypes.POINTER(ctypes.c_int32),
                                               ctypes.c_int32, _i32p, ctypes.c_void_p]),
    "cmr_rotate_qk_kernel": (ctypes.c_char_p, [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                               ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]),
    "cmr_rotate_qk_cache_kernel": (ctypes.c_char_p, [ctypes.c_int64, ctypes.c_int32,
                                                     ctypes.c_int32, ctypes.c_int32,
                                                     ctypes.c_int32, ctypes.c_int32]),
    "cmr_copy_rotated_dims": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                             ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                             ctypes.c_void_p]),
    "cmr_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "cmr_last_error_message": (ctypes.c_char_p, []),
    "cmr_last_rotate_kernel": (ctypes.c_char_p, []),
    "cmr_version": (ctypes.c_int32, []),
}

_lib = None


class CmrError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().cmr_last_error_message().decode()
        super().__init__(f"{where}: {lib().cmr_status_string(status).decode()} -- {msg}")


def lib() -> ctypes.CDLL:
    """The loaded libcmr.so with its signatures set; raises if it was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m vlm_decoder_positional_b200.build`"
                " (there is no CPU fallback)")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def version() -> int:
    return int(lib().cmr_version())


def _check(status: int, where: str):
    if status != CMR_OK:
        raise CmrError(status, where)


def _stream_ptr(device: torch.device, stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return int(s.cuda_stream)


def _want(t: torch.Tensor, name: str, dtype: torch.dtype, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _status_ptr(device_status: Optional[torch.Tensor], dev) -> Optional[int]:
    if device_status is None:
        return None
    _want(device_status, "device_status", torch.int32, dev)
    return device_status.data_ptr()


def positions(ids: torch.Tensor, cu_seqlens: torch.Tensor, image_token_id: int = IMAGE_TOKEN_ID,
              out: Optional[Tuple[torch.Tensor, torch.Tensor, torch.Tensor]] = None,
              device_status: Optional[torch.Tensor] = None,
              stream: Optional[torch.cuda.Stream] = None):
    """cmr_positions: (pos int32 [3, N], start int32 [B], amount int32 [B])."""
    _want(ids, "ids", torch.int32)
    _want(cu_seqlens, "cu_seqlens", torch.int32, ids.device)
    n, b = ids.numel(), cu_seqlens.numel() - 1
    if b < 0:
        raise ValueError("cu_seqlens needs num_seqs + 1 entries")
    if out is None:
        pos = torch.empty((3, n), dtype=torch.int32, device=ids.device)
        start = torch.empty(b, dtype=torch.int32, device=ids.device)
        amount = torch.empty(b, dtype=torch.int32, device=ids.device)
    else:
        pos, start, amount = out
        _want(pos, "pos", torch.int32, ids.device)
        _want(start, "start", torch.int32, ids.device)
        _want(amount, "amount", torch.int32, ids.device)
        if pos.shape != (3, n) or start.numel() != b or amount.numel() != b:
            raise ValueError("output shapes must be [3, N], [B], [B]")
    st_ptr = None
    if device_status is not None:
        _want(device_status, "device_status", torch.int32, ids.device)
        st_ptr = device_status.data_ptr()
    with torch.cuda.device(ids.device):
        _check(lib().cmr_positions(ids.data_ptr() if n else None, cu_seqlens.data_ptr(), b, n,
                                   int(image_token_id), pos.data_ptr() if n else None,
                                   start.data_ptr() if b else None,
                                   amount.data_ptr() if b else None, st_ptr,
                                   _stream_ptr(ids.device, stream)), "cmr_positions")
    return pos, start, amount


def positions_chunk(ids: torch.Tensor, cu_seqlens: torch.Tensor,
                    pos_offset: Optional[torch.Tensor] = None,
                    state: Optional[Tuple[torch.Tensor, torch.Tensor]] = None,
                    rule: str = "canvas", image_token_id: int = IMAGE_TOKEN_ID,
                    out: Optional[Tuple[torch.Tensor, torch.Tensor, torch.Tensor]] = None,
                    device_status: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None):
    """cmr_positions_chunk: planes of prompt chunks at absolute offsets, carrying
    each sequence's (start, amount) state.  Returns (pos [3, N], start [B],
    amount [B]) -- the state after the chunk."""
    _want(ids, "ids", torch.int32)
    dev = ids.device
    _want(cu_seqlens, "cu_seqlens", torch.int32, dev)
    n, b = ids.numel(), cu_seqlens.numel() - 1
    if b < 0:
        raise ValueError("cu_seqlens needs num_seqs + 1 entries")
    if rule not in RULES:
        raise ValueError(f"rule must be one of {sorted(RULES)}")
    per_seq = [(pos_offset, "pos_offset")]
    if state is not None:
        per_seq += [(state[0], "in_start"), (state[1], "in_amount")]
    for t, name in per_seq:
        if t is None:
            continue
        _want(t, name, torch.int32, dev)
        if t.numel() != b:
            raise ValueError(f"{name} needs num_seqs entries")
    off_ptr = pos_offset.data_ptr() if pos_offset is not None else None
    in_s = state[0].data_ptr() if state is not None else None
    in_a = state[1].data_ptr() if state is not None else None
    if out is None:
        pos = torch.empty((3, n), dtype=torch.int32, device=dev)
        start = torch.empty(b, dtype=torch.int32, device=dev)
        amount = torch.empty(b, dtype=torch.int32, device=dev)
    else:
        pos, start, amount = out
        for t, name in ((pos, "pos"), (start, "start"), (amount, "amount")):
            _want(t, name, torch.int32, dev)
        if pos.shape != (3, n) or start.numel() != b or amount.numel() != b:
            raise ValueError("output shapes must be [3, N], [B], [B]")
    st_ptr = None
    if device_status is not None:
        _want(device_status, "device_status", torch.int32, dev)
        st_ptr = device_status.data_ptr()
    with torch.cuda.device(dev):
        _check(lib().cmr_positions_chunk(ids.data_ptr() if n else None, cu_seqlens.data_ptr(), b,
                                         n, int(image_token_id), RULES[rule], off_ptr, in_s, in_a,
                                         pos.data_ptr() if n else None,
                                         start.data_ptr() if b else None,
                                         amount.data_ptr() if b else None, st_ptr,
                                         _stream_ptr(dev, stream)), "cmr_positions_chunk")
    return pos, start, amount


def positions_frames_workspace_bytes(num_seqs: int, n_tokens: int) -> int:
    """Workspace bytes cmr_positions_frames uses at full parallelism."""
    return int(lib().cmr_positions_frames_workspace_bytes(int(num_seqs), int(n_tokens)))


def positions_frames(ids: torch.Tensor, cu_seqlens: torch.Tensor, grid_side: int = 8,
                     image_token_id: int = IMAGE_TOKEN_ID,
                     out: Optional[Tuple[torch.Tensor, torch.Tensor, torch.Tensor]] = None,
                     workspace: Optional[torch.Tensor] = None,
                     device_status: Optional[torch.Tensor] = None,
                     stream: Optional[torch.cuda.Stream] = None):
    """cmr_positions_frames: planes of prompts in which every <image> marker
    opens a frame on a grid_side x grid_side grid.  workspace: a CUDA tensor of
    at least 16 bytes per sequence (allocated at full size when None).
    Returns (pos [3, N], start [B], amount [B])."""
    _want(ids, "ids", torch.int32)
    dev = ids.device
    _want(cu_seqlens, "cu_seqlens", torch.int32, dev)
    n, b = ids.numel(), cu_seqlens.numel() - 1
    if b < 0:
        raise ValueError("cu_seqlens needs num_seqs + 1 entries")
    if out is None:
        pos = torch.empty((3, n), dtype=torch.int32, device=dev)
        start = torch.empty(b, dtype=torch.int32, device=dev)
        amount = torch.empty(b, dtype=torch.int32, device=dev)
    else:
        pos, start, amount = out
        for t, name in ((pos, "pos"), (start, "start"), (amount, "amount")):
            _want(t, name, torch.int32, dev)
        if pos.shape != (3, n) or start.numel() != b or amount.numel() != b:
            raise ValueError("output shapes must be [3, N], [B], [B]")
    if workspace is None:
        workspace = torch.empty(max(positions_frames_workspace_bytes(b, n), 16),
                                dtype=torch.uint8, device=dev)
    if not workspace.is_cuda or workspace.device != dev or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor on the ids' device")
    ws_bytes = workspace.numel() * workspace.element_size()
    st_ptr = _status_ptr(device_status, dev)
    with torch.cuda.device(dev):
        _check(lib().cmr_positions_frames(ids.data_ptr() if n else None, cu_seqlens.data_ptr(),
                                          b, n, int(image_token_id), int(grid_side),
                                          pos.data_ptr() if n else None,
                                          start.data_ptr() if b else None,
                                          amount.data_ptr() if b else None,
                                          workspace.data_ptr(), ws_bytes, st_ptr,
                                          _stream_ptr(dev, stream)), "cmr_positions_frames")
    return pos, start, amount


def positions_step(cache_len: torch.Tensor, start: torch.Tensor, amount: torch.Tensor,
                   out: Optional[torch.Tensor] = None,
                   stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """cmr_positions_step: pos int32 [3, B] of the token at index cache_len[b]."""
    _want(cache_len, "cache_len", torch.int32)
    _want(start, "start", torch.int32, cache_len.device)
    _want(amount, "amount", torch.int32, cache_len.device)
    b = cache_len.numel()
    if start.numel() != b or amount.numel() != b:
        raise ValueError("cache_len, start and amount must have the same length")
    pos = out if out is not None else torch.empty((3, b), dtype=torch.int32,
                                                  device=cache_len.device)
    _want(pos, "out", torch.int32, cache_len.device)
    if pos.shape != (3, b):
        raise ValueError("out must be [3, B]")
    if b == 0:
        return pos
    with torch.cuda.device(cache_len.device):
        _check(lib().cmr_positions_step(cache_len.data_ptr(), start.data_ptr(), amount.data_ptr(),
                                        b, pos.data_ptr(),
                                        _stream_ptr(cache_len.device, stream)),
               "cmr_positions_step")
    return pos


def _want_pinned(t: torch.Tensor, name: str, dtype: torch.dtype):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.is_cuda or (t.numel() and not t.is_pinned()):
        raise ValueError(f"{name} must be a pinned (page-locked) CPU tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _qk_shapes(q, k, dev, n, host=False):
    def shape_of(t, name):
        if t is None:
            return None
        if host:
            _want_pinned(t, name, torch.bfloat16)
        else:
            _want(t, name, torch.bfloat16, dev)
        if t.dim() == 3:
            return (1,) + tuple(t.shape)
        if t.dim() != 4:
            raise ValueError(f"{name} must be [L, N, H, D] or [N, H, D]")
        return tuple(t.shape)

    qs, ks = shape_of(q, "q"), shape_of(k, "k")
    if qs is None and ks is None:
        raise ValueError("need q or k")
    ref = qs or ks
    L, D = ref[0], ref[3]
    for s, name in ((qs, "q"), (ks, "k")):
        if s is not None and (s[0] != L or s[1] != n or s[3] != D):
            raise ValueError(f"{name} shape {s} does not match L={L}, N={n}, D={D}")
    return L, (qs[2] if qs else 0), (ks[2] if ks else 0), D


def rotate_qk_shift(q: Optional[torch.Tensor], k: Optional[torch.Tensor],
                    start: torch.Tensor, amount: torch.Tensor,
                    cu_seqlens: Optional[torch.Tensor] = None,
                    pos_offset: Optional[torch.Tensor] = None, theta: float = 1e7,
                    sections: Sequence[int] = (11, 11, 10), rot_dim: int = 64,
                    stream: Optional[torch.cuda.Stream] = None,
                    device_status: Optional[torch.Tensor] = None):
    """cmr_rotate_qk_shift, in place: the planes of token t of prompt b are the
    canvas rows at pos_offset[b] + t - cu[b] under (start[b], amount[b]);
    cu_seqlens=None means one token per sequence (a decode step).
    device_status: optional int32 [1] on the device (CMR_DEVICE_* bits)."""
    _want(start, "start", torch.int32)
    dev = start.device
    _want(amount, "amount", torch.int32, dev)
    b = start.numel()
    if amount.numel() != b:
        raise ValueError("start and amount must have the same length")
    ref = q if q is not None else k
    n = ref.shape[-3] if ref is not None else 0
    L, hq, hk, D = _qk_shapes(q, k, dev, n)
    cu_ptr = off_ptr = None
    if cu_seqlens is not None:
        _want(cu_seqlens, "cu_seqlens", torch.int32, dev)
        if cu_seqlens.numel() != b + 1:
            raise ValueError("cu_seqlens needs num_seqs + 1 entries")
        cu_ptr = cu_seqlens.data_ptr()
    if pos_offset is not None:
        _want(pos_offset, "pos_offset", torch.int32, dev)
        if pos_offset.numel() != b:
            raise ValueError("pos_offset needs num_seqs entries")
        off_ptr = pos_offset.data_ptr()
    st_ptr = _status_ptr(device_status, dev)
    sec = (ctypes.c_int32 * 3)(*[int(v) for v in sections])
    with torch.cuda.device(dev):
        _check(lib().cmr_rotate_qk_shift(
            q.data_ptr() if q is not None and q.numel() else None,
            k.data_ptr() if k is not None and k.numel() else None, cu_ptr, b, off_ptr,
            start.data_ptr() if b else None, amount.data_ptr() if b else None, n, L, hq, hk, D,
            float(theta), sec, int(rot_dim), st_ptr, _stream_ptr(dev, stream)),
            "cmr_rotate_qk_shift")
    return q, k


def rotate_qk_cache(q: Optional[torch.Tensor], k: Optional[torch.Tensor],
                    v: Optional[torch.Tensor], start: torch.Tensor, amount: torch.Tensor,
                    k_cache: Optional[torch.Tensor], v_cache: Optional[torch.Tensor],
                    cu_seqlens: Optional[torch.Tensor] = None,
                    pos_offset: Optional[torch.Tensor] = None,
                    cache_slot: Optional[torch.Tensor] = None, theta: float = 1e7,
                    sections: Sequence[int] = (11, 11, 10), rot_dim: int = 64,
                    device_status: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None):
    """cmr_rotate_qk_cache: rotate q in place and write the rotated k rows and
    the v rows into k_cache / v_cache [L, S, hk, ctx, D] at each token's index.
    Returns q."""
    _want(start, "start", torch.int32)
    dev = start.device
    _want(amount, "amount", torch.int32, dev)
    b = start.numel()
    ref = q if q is not None else k
    n = ref.shape[-3] if ref is not None else 0
    L, hq, hk, D = _qk_shapes(q, k, dev, n)
    if hk:
        if v is None or k_cache is None or v_cache is None:
            raise ValueError("v, k_cache and v_cache are required with K heads")
        _qk_shapes(None, v, dev, n)
        if tuple(v.shape[-2:]) != (hk, D):
            raise ValueError("v must have the shape of k")
        for t, name in ((k_cache, "k_cache"), (v_cache, "v_cache")):
            _want(t, name, torch.bfloat16, dev)
            if t.dim() != 5 or t.shape[0] != L or t.shape[2] != hk or t.shape[4] != D:
                raise ValueError(f"{name} must be [L, S, hk, ctx, D] = [{L}, S, {hk}, ctx, {D}]")
        if k_cache.shape != v_cache.shape:
            raise ValueError("k_cache and v_cache must have the same shape")
        S, ctx = k_cache.shape[1], k_cache.shape[3]
    else:
        S = ctx = 0
    opt = {}
    for t, name, want_n in ((cu_seqlens, "cu_seqlens", b + 1), (pos_offset, "pos_offset", b),
                            (cache_slot, "cache_slot", b)):
        if t is not None:
            _want(t, name, torch.int32, dev)
            if t.numel() != want_n:
                raise ValueError(f"{name} needs {want_n} entries")
            opt[name] = t.data_ptr()
        else:
            opt[name] = None
    st_ptr = None
    if device_status is not None:
        _want(device_status, "device_status", torch.int32, dev)
        st_ptr = device_status.data_ptr()
    sec = (ctypes.c_int32 * 3)(*[int(x) for x in sections])

    def ptr(t):
        return t.data_ptr() if t is not None and t.numel() else None

    with torch.cuda.device(dev):
        _check(lib().cmr_rotate_qk_cache(
            ptr(q), ptr(k), ptr(v), opt["cu_seqlens"], b, opt["pos_offset"],
            start.data_ptr() if b else None, amount.data_ptr() if b else None, n, L, hq, hk, D,
            float(theta), sec, int(rot_dim), ptr(k_cache), ptr(v_cache), S, ctx,
            opt["cache_slot"], st_ptr, _stream_ptr(dev, stream)), "cmr_rotate_qk_cache")
    return q


def rotate_qk(q: Optional[torch.Tensor], k: Optional[torch.Tensor], pos: torch.Tensor,
              theta: float = 1e7, sections: Sequence[int] = (11, 11, 10), rot_dim: int = 64,
              stream: Optional[torch.cuda.Stream] = None,
              device_status: Optional[torch.Tensor] = None):
    """cmr_rotate_qk, in place.  q: bf16 [L, N, hq, D] (or [N, hq, D]); k likewise
    with hk heads; pos: int32 [3, N]; device_status: optional int32 [1] on the
    device (CMR_DEVICE_* bits).  Returns (q, k)."""
    _want(pos, "pos", torch.int32)
    dev = pos.device
    if pos.dim() != 2 or pos.shape[0] != 3:
        raise ValueError("pos must be [3, N]")
    n = pos.shape[1]
    L, hq, hk, D = _qk_shapes(q, k, dev, n)
    st_ptr = _status_ptr(device_status, dev)
    sec = (ctypes.c_int32 * 3)(*[int(v) for v in sections])
    with torch.cuda.device(dev):
        _check(lib().cmr_rotate_qk(q.data_ptr() if q is not None and q.numel() else None,
                                   k.data_ptr() if k is not None and k.numel() else None,
                                   pos.data_ptr() if n else None, n, L, hq, hk, D, float(theta),
                                   sec, int(rot_dim), st_ptr, _stream_ptr(dev, stream)),
               "cmr_rotate_qk")
    return q, k


def positions_rotate_qk(ids: torch.Tensor, cu_seqlens: torch.Tensor, q: Optional[torch.Tensor],
                        k: Optional[torch.Tensor], theta: float = 1e7,
                        sections: Sequence[int] = (11, 11, 10), rot_dim: int = 64,
                        image_token_id: int = IMAGE_TOKEN_ID,
                        out: Optional[Tuple[torch.Tensor, torch.Tensor, torch.Tensor]] = None,
                        device_status: Optional[torch.Tensor] = None,
                        stream: Optional[torch.cuda.Stream] = None):
    """cmr_positions_rotate_qk: positions, then the rotation of q and k in place
    with those planes, the rotation overlapping the positions kernels.
    Returns (pos [3, N], start [B], amount [B])."""
    _want(ids, "ids", torch.int32)
    dev = ids.device
    _want(cu_seqlens, "cu_seqlens", torch.int32, dev)
    n, b = ids.numel(), cu_seqlens.numel() - 1
    if b < 0:
        raise ValueError("cu_seqlens needs num_seqs + 1 entries")
    L, hq, hk, D = _qk_shapes(q, k, dev, n)
    if out is None:
        pos = torch.empty((3, n), dtype=torch.int32, device=dev)
        start = torch.empty(b, dtype=torch.int32, device=dev)
        amount = torch.empty(b, dtype=torch.int32, device=dev)
    else:
        pos, start, amount = out
        for t, name in ((pos, "pos"), (start, "start"), (amount, "amount")):
            _want(t, name, torch.int32, dev)
        if pos.shape != (3, n) or start.numel() != b or amount.numel() != b:
            raise ValueError("output shapes must be [3, N], [B], [B]")
    st_ptr = _status_ptr(device_status, dev)
    sec = (ctypes.c_int32 * 3)(*[int(v) for v in sections])
    with torch.cuda.device(dev):
        _check(lib().cmr_positions_rotate_qk(
            ids.data_ptr() if n else None, cu_seqlens.data_ptr(), b, n, int(image_token_id),
            pos.data_ptr() if n else None, start.data_ptr() if b else None,
            amount.data_ptr() if b else None,
            q.data_ptr() if q is not None and q.numel() else None,
            k.data_ptr() if k is not None and k.numel() else None, L, hq, hk, D, float(theta),
            sec, int(rot_dim), st_ptr, _stream_ptr(dev, stream)), "cmr_positions_rotate_qk")
    return pos, start, amount


def positions_rotate_qk_host(ids: torch.Tensor, cu_seqlens: torch.Tensor,
                             q: Optional[torch.Tensor], k: Optional[torch.Tensor],
                             theta: float = 1e7, sections: Sequence[int] = (11, 11, 10),
                             rot_dim: int = 64, image_token_id: int = IMAGE_TOKEN_ID,
                             out: Optional[Tuple[torch.Tensor, torch.Tensor, torch.Tensor]] = None,
                             device: Optional[torch.device] = None,
                             stream: Optional[torch.cuda.Stream] = None,
                             device_status: Optional[torch.Tensor] = None):
    """cmr_positions_rotate_qk_host: the whole path on a batch held in pinned
    host memory (ids, cu_seqlens, q, k and the outputs are pinned CPU
    tensors), run by the kernels of `device` (default: the current CUDA
    device), which read and write those buffers over PCIe.  Asynchronous on
    `stream` (default: the device's current stream): synchronise it before
    reading the results or touching the buffers.  device_status: an int32
    [1] tensor on that device or pinned on the host.  Returns (pos [3, N],
    start [B], amount [B]), pinned."""
    _want_pinned(ids, "ids", torch.int32)
    _want_pinned(cu_seqlens, "cu_seqlens", torch.int32)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None \
        else torch.device(device)
    n, b = ids.numel(), cu_seqlens.numel() - 1
    if b < 0:
        raise ValueError("cu_seqlens needs num_seqs + 1 entries")
    L, hq, hk, D = _qk_shapes(q, k, dev, n, host=True)
    if out is None:
        pos = torch.empty((3, n), dtype=torch.int32, pin_memory=True)
        start = torch.empty(b, dtype=torch.int32, pin_memory=True)
        amount = torch.empty(b, dtype=torch.int32, pin_memory=True)
    else:
        pos, start, amount = out
        for t, name in ((pos, "pos"), (start, "start"), (amount, "amount")):
            _want_pinned(t, name, torch.int32)
        if pos.shape != (3, n) or start.numel() != b or amount.numel() != b:
            raise ValueError("output shapes must be [3, N], [B], [B]")
    if device_status is None:
        st_ptr = None
    elif device_status.is_cuda:
        st_ptr = _status_ptr(device_status, dev)
    else:
        _want_pinned(device_status, "device_status", torch.int32)
        st_ptr = device_status.data_ptr()
    sec = (ctypes.c_int32 * 3)(*[int(v) for v in sections])
    with torch.cuda.device(dev):
        _check(lib().cmr_positions_rotate_qk_host(
            ids.data_ptr() if n else None, cu_seqlens.data_ptr(), b, n, int(image_token_id),
            pos.data_ptr() if n else None, start.data_ptr() if b else None,
            amount.data_ptr() if b else None,
            q.data_ptr() if q is not None and q.numel() else None,
            k.data_ptr() if k is not None and k.numel() else None, L, hq, hk, D, float(theta),
            sec, int(rot_dim), st_ptr, _stream_ptr(dev, stream)), "cmr_positions_rotate_qk_host")
    return pos, start, amount


def last_rotate_kernel() -> str:
    """Name of the rotate kernel this thread's last rotate call launched ('' before any)."""
    return lib().cmr_last_rotate_kernel().decode()


def rotate_qk_kernel(n_tokens: int, num_layers: int, hq: int, hk: int, head_dim: int = 256,
                     rot_dim: int = 64) -> Optional[str]:
    """Name of the kernel cmr_rotate_qk launches for these shapes (None if
    there is nothing to launch or the shapes are invalid)."""
    name = lib().cmr_rotate_qk_kernel(int(n_tokens), int(num_layers), int(hq), int(hk),
                                      int(head_dim), int(rot_dim))
    return None if name is None else name.decode()


def rotate_qk_cache_kernel(n_tokens: int, num_layers: int, hq: int, hk: int,
                           head_dim: int = 256, rot_dim: int = 64) -> Optional[str]:
    """Name of the kernel cmr_rotate_qk_cache launches for these shapes (None if
    there is nothing to launch or the shapes are invalid)."""
    name = lib().cmr_rotate_qk_cache_kernel(int(n_tokens), int(num_layers), int(hq), int(hk),
                                            int(head_dim), int(rot_dim))
    return None if name is None else name.decode()


def copy_rotated_dims(dst: torch.Tensor, src: torch.Tensor, rot_dim: int = 64,
                      stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """cmr_copy_rotated_dims: copy dims [0, rot_dim) of every head row of a bf16
    tensor [..., head_dim] between host (pinned) and device memory."""
    for t, name in ((dst, "dst"), (src, "src")):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 tensor")
    if dst.shape != src.shape:
        raise ValueError("dst and src must have the same shape")
    if dst.is_cuda == src.is_cuda:
        raise ValueError("one of dst, src must be on the GPU and the other on the host")
    dev = dst.device if dst.is_cuda else src.device
    head_dim = dst.shape[-1]
    rows = dst.numel() // head_dim if head_dim else 0
    with torch.cuda.device(dev):
        _check(lib().cmr_copy_rotated_dims(dst.data_ptr() if rows else None,
                                           src.data_ptr() if rows else None, rows, head_dim,
                                           int(rot_dim), 0 if dst.is_cuda else 1,
                                           _stream_ptr(dev, stream)), "cmr_copy_rotated_dims")
    return dst
