// Canvas position planes (T, H, W) from token ids, on sm_100a.
//
// Rule: the canvas table of the HF card mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI,
// section "How the VLM rides the text-only engine", with start = O + 67 and
// amount = start - (O + 9) from the Core AI port notes ("The canvas rule and
// why the gate is on the planes").  The port notes' CoreAIKit section gives
// Qwen-VL's shift for comparison (+64 from the pads, 56: start = O + 65), and
// the LiteRT card's runtime uses plain 1-D positions; both are selectable.
//
// Work split: CTA (b, s) owns slice s of prompt chunk b.  When the chunk's
// sequence has no frame yet, the CTA finds the origin by scanning the chunk's
// ids from index 0 up to the end of its own slice (slice 0 scans the whole
// chunk, since it also writes the state), in chunks of 8192 ids (16 loads in
// flight per thread), and stops at the first chunk that holds a marker.  A
// marker past the slice cannot change the slice's planes (every token there
// is p < O -> (p, p, p), the same as text-only), so no CTA waits on another
// and there is no scratch memory and no atomics on data.  Ids re-read by later
// slices hit L2.
#include <climits>

#include "canvas.cuh"

namespace cmr {
namespace {

constexpr int kPosThreads = 512;
constexpr int kIdsPerThread = 16;
constexpr int kScanChunk = kPosThreads * kIdsPerThread;  // 8192 ids per step
constexpr int kSliceTarget = 2048;                       // tokens per CTA (target)
constexpr int kMaxSlices = 65535;                        // gridDim.y limit
constexpr int kQwenVlFrameShift = kGridRows + 1;         // start = O + 65

// Smallest local index in [0, scan_end) whose id is the marker, or -1.
// Block-uniform result; all threads of the CTA must call it.
__device__ __forceinline__ int64_t find_origin(const int32_t* __restrict__ seq, int64_t scan_end,
                                               int32_t marker, int* s_warp_min) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  for (int64_t c = 0; c < scan_end; c += kScanChunk) {
    int32_t v[kIdsPerThread];
#pragma unroll
    for (int m = 0; m < kIdsPerThread; ++m) {
      const int64_t e = c + m * kPosThreads + threadIdx.x;
      v[m] = (e < scan_end) ? __ldg(seq + e) : ~marker;
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

__global__ void __launch_bounds__(kPosThreads)
    canvas_positions_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ cu,
                            int32_t num_seqs, int64_t n_tokens, int32_t marker, int32_t rule,
                            const int32_t* __restrict__ pos_offset,
                            const int32_t* __restrict__ in_start,
                            const int32_t* __restrict__ in_amount, int32_t* __restrict__ pos,
                            int32_t* __restrict__ out_start, int32_t* __restrict__ out_amount,
                            int32_t* __restrict__ status) {
  __shared__ int s_warp_min[kPosThreads / 32];
  const int32_t b = blockIdx.x;
  const int64_t first = __ldg(cu + b);
  const int64_t last = __ldg(cu + b + 1);
  const bool bad = first < 0 || last < first || last > n_tokens ||
                   (b == 0 && first != 0) || (b == num_seqs - 1 && last != n_tokens);
  if (bad) {  // uniform over the CTA
    if (threadIdx.x == 0 && status != nullptr) atomicOr(status, CMR_DEVICE_BAD_CU_SEQLENS);
    return;
  }
  const int64_t len = last - first;
  const int64_t per = (len + gridDim.y - 1) / gridDim.y;
  const int64_t p0 = min(len, static_cast<int64_t>(blockIdx.y) * per);
  const int64_t p1 = min(len, p0 + per);
  if (blockIdx.y != 0 && p0 >= p1) return;

  // The sequence's state before this chunk: (2^30, 0) while no frame is known.
  const int64_t offset = pos_offset ? __ldg(pos_offset + b) : 0;
  int64_t start = in_start ? __ldg(in_start + b) : kTextOnlyStart;
  int64_t amount = in_amount ? __ldg(in_amount + b) : 0;
  if (rule == CMR_RULE_PLANES_1D) {
    start = kTextOnlyStart;
    amount = 0;
  } else if (start >= kTextOnlyStart) {
    const int64_t scan_end = (blockIdx.y == 0) ? len : p1;
    const int64_t m = find_origin(ids + first, scan_end, marker, s_warp_min);
    if (m >= 0) {
      const int64_t origin = offset + m;
      start = origin + (rule == CMR_RULE_QWEN_VL ? kQwenVlFrameShift : kFrameTokens);
      amount = start - (origin + kCanvasSpan);
    } else {
      start = kTextOnlyStart;
      amount = 0;
    }
  }
  if (blockIdx.y == 0 && threadIdx.x == 0) {
    out_start[b] = static_cast<int32_t>(start);
    out_amount[b] = static_cast<int32_t>(amount);
  }

  int32_t* __restrict__ pt = pos + first;
  int32_t* __restrict__ ph = pos + n_tokens + first;
  int32_t* __restrict__ pw = pos + 2 * n_tokens + first;
  if (start >= kTextOnlyStart) {
    for (int64_t p = p0 + threadIdx.x; p < p1; p += kPosThreads) {
      const int32_t v = static_cast<int32_t>(offset + p);
      pt[p] = v;
      ph[p] = v;
      pw[p] = v;
    }
  } else {
    for (int64_t p = p0 + threadIdx.x; p < p1; p += kPosThreads) {
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
  dim3 grid(static_cast<unsigned>(num_seqs), static_cast<unsigned>(slices));
  canvas_positions_kernel<<<grid, kPosThreads, 0, stream>>>(
      ids, cu_seqlens, num_seqs, n_tokens, image_token_id, rule, pos_offset, in_start, in_amount,
      out_pos, out_start, out_amount, device_status);
  return cudaGetLastError();
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
