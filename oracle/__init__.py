"""The oracle for canvas M-RoPE -- TEST INFRASTRUCTURE ONLY.

A plain fp64 CPU restatement of the hot path (cmr_oracle.c), wrapped for NumPy.
Only tests/, ``__graft_entry__.smoke()`` and bench.py's CPU-baseline and
reference legs may import it.  It shares no code with the CUDA library in
``vlm_decoder_positional_b200`` and neither side imports the other.

Pages followed (see cmr_oracle.c for the passage behind each function):
  * Core AI model zoo, "MiniCPM-V-4.7-1B: canvas M-RoPE on the Qwen3.5 hybrid,
    on Core AI", section "The canvas rule and why the gate is on the planes";
  * HF card mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI, section "How the VLM rides the
    text-only engine" (canvas table) and "What it is" (sections [11, 11, 10]).

Every function is pinned by ``tests/test_oracle_*.py`` against the pages'
worked values, closed forms, invariants and textbook special cases.
"""
import ctypes

import numpy as np

from . import build as _build

RULE_CANVAS = 0
RULE_AMOUNT_PLUS_ONE = 1
RULE_PLANES_1D = 2
_RULES = {"canvas": RULE_CANVAS, "amount+1": RULE_AMOUNT_PLUS_ONE,
          "planes_1d": RULE_PLANES_1D}
CHUNK_RULES = {"canvas": 0, "qwen_vl": 1, "planes_1d": 2}
TEXT_ONLY_START = 1 << 30

_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_build.build())
        i32p = ctypes.POINTER(ctypes.c_int32)
        lib.oracle_positions.argtypes = [i32p, i32p, ctypes.c_int32, ctypes.c_int64,
                                         ctypes.c_int32, ctypes.c_int32, i32p, i32p, i32p]
        lib.oracle_positions.restype = ctypes.c_int
        lib.oracle_positions_chunk.argtypes = [i32p, i32p, ctypes.c_int32, ctypes.c_int64,
                                               ctypes.c_int32, ctypes.c_int32, i32p, i32p, i32p,
                                               i32p, i32p, i32p]
        lib.oracle_positions_chunk.restype = ctypes.c_int
        lib.oracle_positions_frames.argtypes = [i32p, i32p, ctypes.c_int32, ctypes.c_int64,
                                                ctypes.c_int32, ctypes.c_int32, i32p, i32p,
                                                i32p]
        lib.oracle_positions_frames.restype = ctypes.c_int
        lib.oracle_positions_step.argtypes = [i32p, i32p, i32p, ctypes.c_int32, i32p]
        lib.oracle_positions_step.restype = ctypes.c_int
        lib.oracle_freq_planes.argtypes = [ctypes.c_int32, i32p, i32p]
        lib.oracle_freq_planes.restype = ctypes.c_int
        lib.oracle_rotate_f64.argtypes = [ctypes.c_void_p, i32p, ctypes.c_int64,
                                          ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                          ctypes.c_double, i32p, ctypes.c_int32]
        lib.oracle_rotate_f64.restype = ctypes.c_int
        lib.oracle_rotate_bf16.argtypes = [ctypes.c_void_p, i32p, ctypes.c_int64,
                                           ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.c_double, i32p, ctypes.c_int32,
                                           ctypes.c_void_p]
        lib.oracle_rotate_bf16.restype = ctypes.c_int
        lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f64.restype = ctypes.c_double
        lib.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
        lib.oracle_f64_to_bf16.restype = ctypes.c_uint16
        _lib = lib
    return _lib


def _i32(a):
    a = np.ascontiguousarray(a, dtype=np.int32)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


class OracleError(ValueError):
    pass


def positions(ids, cu_seqlens, image_token_id=248078, rule="canvas"):
    """Canvas planes of a packed batch.  Returns (pos [3, N], start [B], amount [B])."""
    lib = _load()
    ids, ids_p = _i32(ids)
    cu, cu_p = _i32(cu_seqlens)
    n = int(ids.shape[0])
    b = int(cu.shape[0]) - 1
    pos = np.zeros((3, n), dtype=np.int32)
    start = np.zeros(max(b, 0), dtype=np.int32)
    amount = np.zeros(max(b, 0), dtype=np.int32)
    st = lib.oracle_positions(ids_p, cu_p, b, n, int(image_token_id), _RULES[rule],
                              _i32(pos)[1], _i32(start)[1], _i32(amount)[1])
    if st != 0:
        raise OracleError("oracle_positions: invalid arguments")
    return pos, start, amount


def positions_chunk(ids, cu_seqlens, image_token_id=248078, rule="canvas", pos_offset=None,
                    in_start=None, in_amount=None):
    """Planes of a batch of prompt chunks at absolute offsets, continuing each
    sequence's (start, amount) state.  Returns (pos [3, N], start [B], amount [B])."""
    lib = _load()
    ids, ids_p = _i32(ids)
    cu, cu_p = _i32(cu_seqlens)
    n = int(ids.shape[0])
    b = int(cu.shape[0]) - 1
    opt = []
    for a in (pos_offset, in_start, in_amount):
        if a is None:
            opt.append((None, None))
        else:
            arr, ptr = _i32(a)
            if arr.shape[0] != b:
                raise OracleError("per-sequence arrays need num_seqs entries")
            opt.append((arr, ptr))
    pos = np.zeros((3, n), dtype=np.int32)
    start = np.zeros(max(b, 0), dtype=np.int32)
    amount = np.zeros(max(b, 0), dtype=np.int32)
    st = lib.oracle_positions_chunk(ids_p, cu_p, b, n, int(image_token_id), CHUNK_RULES[rule],
                                    opt[0][1], opt[1][1], opt[2][1], _i32(pos)[1],
                                    _i32(start)[1], _i32(amount)[1])
    if st != 0:
        raise OracleError("oracle_positions_chunk: invalid arguments")
    return pos, start, amount


def positions_frames(ids, cu_seqlens, image_token_id=248078, grid_side=8):
    """Planes of a packed batch in which every <image> marker opens a frame of
    grid_side^2 + 3 tokens (the multi-frame reading of cmr_oracle.c).  Returns
    (pos [3, N], start [B], amount [B])."""
    lib = _load()
    ids, ids_p = _i32(ids)
    cu, cu_p = _i32(cu_seqlens)
    n = int(ids.shape[0])
    b = int(cu.shape[0]) - 1
    pos = np.zeros((3, n), dtype=np.int32)
    start = np.zeros(max(b, 0), dtype=np.int32)
    amount = np.zeros(max(b, 0), dtype=np.int32)
    st = lib.oracle_positions_frames(ids_p, cu_p, b, n, int(image_token_id), int(grid_side),
                                     _i32(pos)[1], _i32(start)[1], _i32(amount)[1])
    if st != 0:
        raise OracleError("oracle_positions_frames: invalid arguments")
    return pos, start, amount


def positions_step(cache_len, start, amount):
    """Planes of the token at index cache_len[b] of each sequence.  Returns pos [3, B]."""
    lib = _load()
    cl, cl_p = _i32(cache_len)
    s, s_p = _i32(start)
    a, a_p = _i32(amount)
    b = int(cl.shape[0])
    pos = np.zeros((3, b), dtype=np.int32)
    if lib.oracle_positions_step(cl_p, s_p, a_p, b, _i32(pos)[1]) != 0:
        raise OracleError("oracle_positions_step: invalid arguments")
    return pos


def freq_planes(rot_dim=64, sections=(11, 11, 10)):
    """Plane (0 = T, 1 = H, 2 = W) of each of the rot_dim/2 frequencies."""
    lib = _load()
    sec, sec_p = _i32(sections)
    plane = np.zeros(max(rot_dim // 2, 1), dtype=np.int32)
    if lib.oracle_freq_planes(int(rot_dim), sec_p, _i32(plane)[1]) != 0:
        raise OracleError("oracle_freq_planes: sections do not fit rot_dim")
    return plane[: rot_dim // 2]


def rotate_f64(x, pos, theta=1e7, sections=(11, 11, 10), rot_dim=64):
    """Rotate a float64 array [L, N, H, D] (returns a rotated copy)."""
    lib = _load()
    x = np.array(x, dtype=np.float64, order="C", copy=True)
    if x.ndim != 4:
        raise OracleError("x must be [L, N, H, D]")
    L, n, h, d = x.shape
    pos, pos_p = _i32(pos)
    sec, sec_p = _i32(sections)
    st = lib.oracle_rotate_f64(x.ctypes.data, pos_p, n, L, h, d, float(theta), sec_p,
                               int(rot_dim))
    if st != 0:
        raise OracleError("oracle_rotate_f64: invalid arguments")
    return x


def rotate_bf16(x_bits, pos, theta=1e7, sections=(11, 11, 10), rot_dim=64,
                return_f64=False):
    """Rotate bf16 bit patterns (uint16 [L, N, H, D]); returns the rotated copy
    (and the unrounded fp64 rows if return_f64)."""
    lib = _load()
    x = np.array(x_bits, dtype=np.uint16, order="C", copy=True)
    if x.ndim != 4:
        raise OracleError("x must be [L, N, H, D]")
    L, n, h, d = x.shape
    pos, pos_p = _i32(pos)
    sec, sec_p = _i32(sections)
    f64 = np.zeros(x.shape, dtype=np.float64) if return_f64 else None
    st = lib.oracle_rotate_bf16(x.ctypes.data, pos_p, n, L, h, d, float(theta), sec_p,
                                int(rot_dim), f64.ctypes.data if return_f64 else None)
    if st != 0:
        raise OracleError("oracle_rotate_bf16: invalid arguments")
    return (x, f64) if return_f64 else x


def bf16_to_f64(bits):
    lib = _load()
    flat = np.asarray(bits, dtype=np.uint16).ravel()
    out = np.array([lib.oracle_bf16_to_f64(int(b)) for b in flat], dtype=np.float64)
    return out.reshape(np.shape(bits))


def f64_to_bf16(values):
    lib = _load()
    flat = np.asarray(values, dtype=np.float64).ravel()
    out = np.array([lib.oracle_f64_to_bf16(float(v)) for v in flat], dtype=np.uint16)
    return out.reshape(np.shape(values))


def token_index(n_tokens, num_seqs, cu_seqlens=None, pos_offset=None):
    """Sequence b and absolute index p of every packed token (cu_seqlens None:
    token b is sequence b)."""
    if cu_seqlens is None:
        b = np.arange(n_tokens, dtype=np.int64)
        local = np.zeros(n_tokens, dtype=np.int64)
    else:
        cu = np.asarray(cu_seqlens, dtype=np.int64)
        b = np.repeat(np.arange(num_seqs), np.diff(cu))
        local = np.arange(n_tokens, dtype=np.int64) - cu[b]
    off = np.zeros(num_seqs, np.int64) if pos_offset is None else np.asarray(pos_offset, np.int64)
    return b, off[b] + local


def rotate_qk_cache(q_bits, k_bits, v_bits, start, amount, k_cache_bits, v_cache_bits,
                    cu_seqlens=None, pos_offset=None, cache_slot=None, theta=1e7,
                    sections=(11, 11, 10), rot_dim=64):
    """Rotate Q, and place the rotated K rows and the V rows into the KV cache
    [L, S, hk, ctx, D] at each token's absolute index (the engine's keyCache /
    valueCache of HF card mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI, "How the VLM
    rides the text-only engine").  Planes: the decode form at the token's index
    under its sequence's (start, amount).  Returns (q, k_cache, v_cache,
    status) with status bit 2 set when a token falls outside the cache."""
    start = np.asarray(start, np.int32)
    amount = np.asarray(amount, np.int32)
    n = q_bits.shape[1] if q_bits is not None else k_bits.shape[1]
    b, p = token_index(n, start.shape[0], cu_seqlens, pos_offset)
    pos = positions_step(p.astype(np.int32), start[b], amount[b])
    q_out = rotate_bf16(q_bits, pos, theta, sections, rot_dim) if q_bits is not None else None
    kc = np.array(k_cache_bits, copy=True) if k_cache_bits is not None else None
    vc = np.array(v_cache_bits, copy=True) if v_cache_bits is not None else None
    status = 0
    if k_bits is not None:
        k_rot = rotate_bf16(k_bits, pos, theta, sections, rot_dim)
        slot = b if cache_slot is None else np.asarray(cache_slot, np.int64)[b]
        S, ctx = kc.shape[1], kc.shape[3]
        for t in range(n):
            if 0 <= p[t] < ctx and 0 <= slot[t] < S:
                kc[:, slot[t], :, p[t], :] = k_rot[:, t]
                vc[:, slot[t], :, p[t], :] = v_bits[:, t]
            else:
                status |= 2
    return q_out, kc, vc, status
