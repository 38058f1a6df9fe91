"""Canvas M-RoPE for the Qwen3.5-hybrid decoder of MiniCPM-V-4.7-1B, on B200.

    pos, start, amount = positions(ids, cu_seqlens)        # planes (T, H, W)
    rotate_qk(q, k, pos, theta=1e7, sections=(11, 11, 10), rot_dim=64)
    pos, start, amount = positions_rotate_qk(ids, cu_seqlens, q, k)   # both, overlapped
    pos, start, amount = positions_rotate_qk_host(ids, cu_seqlens, q, k)  # pinned host batch

Both run hand-written sm_100a kernels in libcmr.so through its C ABI
(include/cmr.h); build it with ``python -m vlm_decoder_positional_b200.build``.
"""
from .cmr import (CMR_DEVICE_BAD_CU_SEQLENS, CMR_DEVICE_CACHE_RANGE, CMR_DEVICE_WAIT_TIMEOUT,
                  CMR_ECUDA, CMR_EINVAL, CMR_EUNSUPPORTED, CMR_OK, CmrError, last_rotate_kernel,
                  lib, positions, positions_chunk, positions_frames,
                  positions_frames_workspace_bytes, positions_rotate_qk,
                  positions_rotate_qk_host, positions_step, rotate_qk,
                  rotate_qk_cache, rotate_qk_cache_kernel, rotate_qk_kernel, rotate_qk_shift,
                  version)

__all__ = ["positions", "positions_chunk", "positions_step", "positions_rotate_qk",
           "positions_rotate_qk_host",
           "positions_frames", "positions_frames_workspace_bytes",
           "rotate_qk", "rotate_qk_shift", "last_rotate_kernel",
           "rotate_qk_kernel", "rotate_qk_cache_kernel",
           "rotate_qk_cache", "CMR_DEVICE_CACHE_RANGE", "CMR_DEVICE_WAIT_TIMEOUT",
           "lib", "version", "CmrError",
           "CMR_OK", "CMR_EINVAL", "CMR_ECUDA", "CMR_EUNSUPPORTED", "CMR_DEVICE_BAD_CU_SEQLENS"]
