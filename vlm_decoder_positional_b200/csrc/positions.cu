// Canvas position planes (T, H, W) from token ids, on sm_100a.
//
// Rule: the canvas table of the HF card mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI,
// section "How the VLM rides the text-only engine", with start = O + 67 and
// amount = start - (O + 9) from the Core AI port notes ("The canvas rule and
// why the gate is on the planes").  The port notes' CoreAIKit section gives
// Qwen-VL's shift for comparison (+64 from the pads, 56: start = O + 65), and
// the LiteRT card's runtime uses plain 1-D positions; both are selectable.
//
// Work split: two kernels over CTAs (b, s), one per slice s of prompt chunk b,
// with the outgoing start as the only cross-CTA state:
//   1. the caller's out_start is set to a sentinel (0x7F7F7F7F, above any
//      start) by a memset; canvas_origin_kernel then scans each slice's own
//      ids for its first marker m (16 loads in flight per thread, warp
//      `redux.sync` min, a shared-memory min) and, if it has one, lowers
//      out_start[b] to offset + m + (frame length) with atomicMin -- the start
//      that the chunk's first marker gives, since the shift is the same for
//      every marker.  Every id is read once.
//   2. canvas_positions_kernel, launched programmatically behind it (it
//      starts while the scan runs and waits for it before reading out_start),
//      turns out_start[b] into (start, amount), writes the slice's planes
//      (12 B per token, no id reads), and slice 0 writes the state.  For a
//      text-only chunk slice 0 replaces the sentinel by 2^30 while other CTAs
//      of the chunk may still read out_start[b]; both values mean "no frame".
// No CTA waits on another and there is no scratch memory: the state lives in
// the caller's output.  A chunk whose frame is already known (in_start[b] <
// 2^30), and the 1-D rule, skip the scan.
#include <climits>

#include "canvas.cuh"
#include "pdl.cuh"

namespace cmr {
namespace {

constexpr int kPosThreads = 512;
constexpr int kIdsPerThread = 16;
constexpr int kScanChunk = kPosThreads * kIdsPerThread;  // 8192 ids per step
constexpr int kSliceTarget = 2048;                       // tokens per CTA (target)
constexpr int kMaxSlices = 65535;                        // gridDim.y limit
constexpr int kQwenVlFrameShift = kGridRows + 1;         // start = O + 65
constexpr int32_t kStartSentinel = 0x7F7F7F7F;           // memset byte 0x7F; >= 2^30

// Index of the first marker in seq[0, len), or -1.  Block-uniform result;
// all threads of the CTA must call it.
__device__ __forceinline__ int64_t first_marker(const int32_t* __restrict__ seq, int64_t len,
                                                int32_t marker, int* s_warp_min) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  for (int64_t c = 0; c < len; c += kScanChunk) {
    int32_t v[kIdsPerThread];
#pragma unroll
    for (int m = 0; m < kIdsPerThread; ++m) {
      const int64_t e = c + m * kPosThreads + threadIdx.x;
      v[m] = (e < len) ? __ldg(seq + e) : ~marker;
    }
    int best = INT_MAX;  // offset within the chunk; smaller m = smaller index
#pragma unroll
    for (int m = kIdsPerThread - 1; m >= 0; --m)
      if (v[m] == marker) best = m * kPosThreads + threadIdx.x;
    best = __reduce_min_sync(0xffffffffu, best);
    if (lane == 0) s_warp_min[warp] = best;
    __syncthreads();
    int block_best = INT_MAX;
#pragma unroll
    for (int i = 0; i < kPosThreads / 32; ++i) block_best = min(block_best, s_warp_min[i]);
    __syncthreads();  // s_warp_min is rewritten by the next chunk
    if (block_best != INT_MAX) return c + block_best;
  }
  return -1;
}

// Bounds of prompt chunk b and of this CTA's slice; false (uniform over the
// CTA) when cu_seqlens is malformed around b or the slice is empty.
struct Slice {
  int64_t first, len, p0, p1;
};

__device__ __forceinline__ bool cta_slice(const int32_t* __restrict__ cu, int32_t num_seqs,
                                          int64_t n_tokens, bool* bad, Slice* sl) {
  const int32_t b = blockIdx.x;
  const int64_t first = __ldg(cu + b);
  const int64_t last = __ldg(cu + b + 1);
  *bad = first < 0 || last < first || last > n_tokens || (b == 0 && first != 0) ||
         (b == num_seqs - 1 && last != n_tokens);
  if (*bad) return false;
  const int64_t len = last - first;
  const int64_t per = (len + gridDim.y - 1) / gridDim.y;
  sl->first = first;
  sl->len = len;
  sl->p0 = min(len, static_cast<int64_t>(blockIdx.y) * per);
  sl->p1 = min(len, sl->p0 + per);
  return true;
}

__device__ __forceinline__ int32_t frame_shift(int32_t rule) {
  return rule == CMR_RULE_QWEN_VL ? kQwenVlFrameShift : kFrameTokens;
}

// out_start[b] is read by every CTA of chunk b while its slice 0 may write it
// (text-only: sentinel -> 2^30), so both sides use relaxed (strong) accesses.
__device__ __forceinline__ int32_t load_relaxed(const int32_t* p) {
  int32_t v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void store_relaxed(int32_t* p, int32_t v) {
  asm volatile("st.relaxed.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__global__ void __launch_bounds__(kPosThreads)
    canvas_origin_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ cu,
                         int32_t num_seqs, int64_t n_tokens, int32_t marker, int32_t rule,
                         const int32_t* __restrict__ pos_offset,
                         const int32_t* __restrict__ in_start, int32_t* out_start,
                         int32_t* __restrict__ status) {
  __shared__ int s_warp_min[kPosThreads / 32];
  pdl::launch_dependents();
  bool bad;
  Slice sl;
  if (!cta_slice(cu, num_seqs, n_tokens, &bad, &sl)) {
    if (bad && blockIdx.y == 0 && threadIdx.x == 0 && status != nullptr)
      atomicOr(status, CMR_DEVICE_BAD_CU_SEQLENS);
    return;
  }
  const int32_t b = blockIdx.x;
  if (rule == CMR_RULE_PLANES_1D || sl.p0 >= sl.p1) return;
  if (in_start != nullptr && __ldg(in_start + b) < kTextOnlyStart) return;  // frame known
  const int64_t m = first_marker(ids + sl.first + sl.p0, sl.p1 - sl.p0, marker, s_warp_min);
  if (m >= 0 && threadIdx.x == 0) {
    const int64_t offset = pos_offset ? __ldg(pos_offset + b) : 0;
    atomicMin(out_start + b, static_cast<int32_t>(offset + sl.p0 + m + frame_shift(rule)));
  }
}

__global__ void __launch_bounds__(kPosThreads)
    canvas_positions_kernel(const int32_t* __restrict__ cu, int32_t num_seqs, int64_t n_tokens,
                            int32_t rule, const int32_t* __restrict__ pos_offset,
                            const int32_t* __restrict__ in_start,
                            const int32_t* __restrict__ in_amount, int32_t* __restrict__ pos,
                            int32_t* out_start, int32_t* __restrict__ out_amount) {
  pdl::launch_dependents();
  bool bad;
  Slice sl;
  const bool ok = cta_slice(cu, num_seqs, n_tokens, &bad, &sl);
  if (!ok || (blockIdx.y != 0 && sl.p0 >= sl.p1)) return;
  const int32_t b = blockIdx.x;
  // The sequence's state before this chunk: (2^30, 0) while no frame is known.
  const int64_t offset = pos_offset ? __ldg(pos_offset + b) : 0;
  int64_t start = in_start ? __ldg(in_start + b) : kTextOnlyStart;
  int64_t amount = in_amount ? __ldg(in_amount + b) : 0;
  pdl::wait();  // the origin scan's atomicMin on out_start[b] is visible
  if (rule == CMR_RULE_PLANES_1D) {
    start = kTextOnlyStart;
    amount = 0;
  } else if (start >= kTextOnlyStart) {
    const int64_t found = load_relaxed(out_start + b);
    if (found < kTextOnlyStart) {
      start = found;  // origin + frame_shift(rule)
      amount = start - (start - frame_shift(rule) + kCanvasSpan);
    } else {
      start = kTextOnlyStart;
      amount = 0;
    }
  }
  if (blockIdx.y == 0 && threadIdx.x == 0) {
    store_relaxed(out_start + b, static_cast<int32_t>(start));
    out_amount[b] = static_cast<int32_t>(amount);
  }

  int32_t* __restrict__ pt = pos + sl.first;
  int32_t* __restrict__ ph = pos + n_tokens + sl.first;
  int32_t* __restrict__ pw = pos + 2 * n_tokens + sl.first;
  if (start >= kTextOnlyStart) {
    for (int64_t p = sl.p0 + threadIdx.x; p < sl.p1; p += kPosThreads) {
      const int32_t v = static_cast<int32_t>(offset + p);
      pt[p] = v;
      ph[p] = v;
      pw[p] = v;
    }
  } else {
    for (int64_t p = sl.p0 + threadIdx.x; p < sl.p1; p += kPosThreads) {
      const Planes r = canvas_row(offset + p, start, amount);
      pt[p] = r.t;
      ph[p] = r.h;
      pw[p] = r.w;
    }
  }
}

__global__ void canvas_positions_step_kernel(const int32_t* __restrict__ cache_len,
                                             const int32_t* __restrict__ start,
                                             const int32_t* __restrict__ amount,
                                             int32_t num_seqs, int32_t* __restrict__ pos) {
  for (int64_t b = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; b < num_seqs;
       b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    // The engine binds only start and amount; canvas_row recovers the origin
    // from amount = start - (O + 9).
    const Planes r = canvas_row(__ldg(cache_len + b), __ldg(start + b), __ldg(amount + b));
    pos[b] = r.t;
    pos[num_seqs + b] = r.h;
    pos[2 * static_cast<int64_t>(num_seqs) + b] = r.w;
  }
}

}  // namespace

cudaError_t launch_positions(const int32_t* ids, const int32_t* cu_seqlens, int32_t num_seqs,
                             int64_t n_tokens, int32_t image_token_id, int32_t rule,
                             const int32_t* pos_offset, const int32_t* in_start,
                             const int32_t* in_amount, int32_t* out_pos, int32_t* out_start,
                             int32_t* out_amount, int32_t* device_status, cudaStream_t stream) {
  if (num_seqs == 0) return cudaSuccess;
  const int64_t avg = (n_tokens + num_seqs - 1) / num_seqs;
  int64_t slices = (avg + kSliceTarget - 1) / kSliceTarget;
  slices = slices < 1 ? 1 : (slices > kMaxSlices ? kMaxSlices : slices);
  const dim3 grid(static_cast<unsigned>(num_seqs), static_cast<unsigned>(slices));
  cudaError_t e = cudaMemsetAsync(out_start, 0x7F, static_cast<size_t>(num_seqs) * sizeof(int32_t),
                                  stream);
  static_assert(kStartSentinel == 0x7F7F7F7F && kStartSentinel >= kTextOnlyStart,
                "the memset byte must give a sentinel start above every real start");
  if (e != cudaSuccess) return e;
  canvas_origin_kernel<<<grid, kPosThreads, 0, stream>>>(ids, cu_seqlens, num_seqs, n_tokens,
                                                         image_token_id, rule, pos_offset,
                                                         in_start, out_start, device_status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return pdl::launch(canvas_positions_kernel, grid, dim3(kPosThreads), 0, stream, true,
                     cu_seqlens, num_seqs, n_tokens, rule, pos_offset, in_start, in_amount,
                     out_pos, out_start, out_amount);
}

cudaError_t launch_positions_step(const int32_t* cache_len, const int32_t* start,
                                  const int32_t* amount, int32_t num_seqs, int32_t* out_pos,
                                  cudaStream_t stream) {
  if (num_seqs == 0) return cudaSuccess;
  const int threads = 256;
  int64_t blocks = (static_cast<int64_t>(num_seqs) + threads - 1) / threads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  canvas_positions_step_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      cache_len, start, amount, num_seqs, out_pos);
  return cudaGetLastError();
}

}  // namespace cmr
