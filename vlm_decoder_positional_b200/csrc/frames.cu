// Position planes of prompts with several image frames on an s x s grid, on
// sm_100a.
//
// Rule (a reading of the HF card mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI, "How
// the VLM rides the text-only engine", extended from its one-thumbnail table
// as the MNN card's "Validation" says sliced and multi-image prompts were
// checked): a running counter gives text tokens (c, c, c) and advances by 1;
// every <image> marker opens a frame of s*s + 3 tokens anchored at the
// counter's value f -- <image> (f, f-1, f-1), row k (f, f + k/s, f + k%s),
// </image> (f, f+s, f+s), "\n" (f, f, f) -- after which the counter stands at
// f + s + 1, one past the frame's largest coordinate (9 = max(H, W) + 1 for the
// 8x8 thumbnail), even when the next marker or the end of the prompt cuts the
// frame short.
//
// As a scan: with O_0 < O_1 < ... the markers of a prompt, frame i's anchor is
//   f_i = O_0 + i (s + 1) + sum_{j < i} max(0, O_{j+1} - O_j - (s*s + 3)),
// so token p needs only the inclusive prefix, over the tokens up to p, of
// (marker count, first marker, last marker, summed excess gaps) -- an
// associative (not commutative) combine.  Two kernels over CTAs (b, s), one
// per slice s of prompt b:
//   1. frames_summary_kernel reduces its slice's tokens to that 16-byte summary
//      in a caller-provided workspace [num_seqs][slices];
//   2. frames_positions_kernel, launched programmatically behind it, folds the
//      summaries of the slices before its own into a carry (slice 0 folds all
//      of them for the state), then walks its slice in chunks of kFrThreads
//      tokens: a warp scan by shuffles, a scan of the warp totals, the carry,
//      and the planes of every token.
// Ids are read twice (once per kernel; the second read mostly hits L2); the
// planes are written once.  No CTA waits on another.
#include <mutex>

#include "canvas.cuh"
#include "pdl.cuh"

namespace cmr {
namespace {

constexpr int kFrThreads = 512;
constexpr int kFrWarps = kFrThreads / 32;
constexpr int kFrPerThread = 4;                              // ids in flight per thread
constexpr int kFrSliceTarget = kFrThreads * kFrPerThread;    // 2048 tokens per CTA
constexpr int kFrMaxSlices = 65535;                          // gridDim.y limit

// Prefix summary of a run of tokens: n markers, the first and last of them
// (local indices), and the sum over consecutive marker pairs of the text
// between a complete frame and the next marker.
struct Summary {
  int32_t n, first, last, gaps;
};

__device__ __forceinline__ Summary combine(const Summary& l, const Summary& r, int32_t frame_len) {
  if (l.n == 0) return r;
  if (r.n == 0) return l;
  return {l.n + r.n, l.first, r.last, l.gaps + r.gaps + max(0, r.first - l.last - frame_len)};
}

__device__ __forceinline__ Summary shfl_up(const Summary& v, int delta) {
  return {__shfl_up_sync(0xffffffffu, v.n, delta), __shfl_up_sync(0xffffffffu, v.first, delta),
          __shfl_up_sync(0xffffffffu, v.last, delta), __shfl_up_sync(0xffffffffu, v.gaps, delta)};
}

// Inclusive scan over the warp's lanes in lane order.
__device__ __forceinline__ Summary warp_scan(Summary v, int32_t frame_len) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const Summary u = shfl_up(v, d);
    if (lane >= d) v = combine(u, v, frame_len);
  }
  return v;
}

// Block-wide inclusive scan in thread order; *total receives the block's
// summary.  All threads must call it; it uses s_warp[kFrWarps] and two
// barriers.
__device__ __forceinline__ Summary block_scan(Summary v, int32_t frame_len, Summary* s_warp,
                                              Summary* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_scan(v, frame_len);
  if (lane == 31) s_warp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    Summary w = lane < kFrWarps ? s_warp[lane] : Summary{0, 0, 0, 0};
    w = warp_scan(w, frame_len);
    if (lane < kFrWarps) s_warp[lane] = w;  // inclusive prefix of the warp totals
  }
  __syncthreads();
  const Summary before = warp > 0 ? s_warp[warp - 1] : Summary{0, 0, 0, 0};
  *total = s_warp[kFrWarps - 1];
  __syncthreads();  // s_warp is rewritten by the next call
  return combine(before, v, frame_len);
}

struct FrSlice {
  int64_t first, len, p0, p1;
};

__device__ __forceinline__ bool fr_slice(const int32_t* __restrict__ cu, int32_t num_seqs,
                                         int64_t n_tokens, bool* bad, FrSlice* sl) {
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

__global__ void __launch_bounds__(kFrThreads)
    frames_summary_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ cu,
                          int32_t num_seqs, int64_t n_tokens, int32_t marker, int32_t frame_len,
                          Summary* __restrict__ work, int32_t* __restrict__ status) {
  __shared__ Summary s_warp[kFrWarps];
  pdl::launch_dependents();
  bool bad;
  FrSlice sl;
  if (!fr_slice(cu, num_seqs, n_tokens, &bad, &sl)) {
    if (bad && blockIdx.y == 0 && threadIdx.x == 0 && status != nullptr)
      atomicOr(status, CMR_DEVICE_BAD_CU_SEQLENS);
    return;
  }
  const int32_t* __restrict__ seq = ids + sl.first;
  Summary run{0, 0, 0, 0};
  for (int64_t c = sl.p0; c < sl.p1; c += kFrSliceTarget) {
    int32_t v[kFrPerThread];
#pragma unroll
    for (int m = 0; m < kFrPerThread; ++m) {
      const int64_t p = c + m * kFrThreads + threadIdx.x;
      v[m] = (p < sl.p1) ? __ldg(seq + p) : ~marker;
    }
#pragma unroll
    for (int m = 0; m < kFrPerThread; ++m) {
      const int32_t p = static_cast<int32_t>(c + m * kFrThreads + threadIdx.x);
      Summary e = (v[m] == marker) ? Summary{1, p, p, 0} : Summary{0, 0, 0, 0};
      Summary total;
      block_scan(e, frame_len, s_warp, &total);
      run = combine(run, total, frame_len);
    }
  }
  if (threadIdx.x == 0)
    work[static_cast<int64_t>(blockIdx.x) * gridDim.y + blockIdx.y] = run;
}

// Ordered fold of summaries[0, count) by the whole block.  The summaries come
// from the kernel before (plain loads, not the read-only path).
__device__ __forceinline__ Summary fold(const Summary* sums, int32_t count,
                                        int32_t frame_len, Summary* s_warp) {
  Summary acc{0, 0, 0, 0};
  for (int32_t base = 0; base < count; base += kFrThreads) {
    const int32_t j = base + threadIdx.x;
    Summary e = j < count ? sums[j] : Summary{0, 0, 0, 0};
    Summary total;
    block_scan(e, frame_len, s_warp, &total);
    acc = combine(acc, total, frame_len);
  }
  return acc;
}

__global__ void __launch_bounds__(kFrThreads)
    frames_positions_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ cu,
                            int32_t num_seqs, int64_t n_tokens, int32_t marker, int32_t side,
                            const Summary* work, int32_t* __restrict__ pos,
                            int32_t* __restrict__ out_start, int32_t* __restrict__ out_amount) {
  __shared__ Summary s_warp[kFrWarps];
  bool bad;
  FrSlice sl;
  if (!fr_slice(cu, num_seqs, n_tokens, &bad, &sl)) return;
  if (blockIdx.y != 0 && sl.p0 >= sl.p1) return;
  const int32_t frame_len = side * side + 3;
  const int64_t span = side + 1;  // counter advance per frame
  const Summary* sums = work + static_cast<int64_t>(blockIdx.x) * gridDim.y;
  pdl::wait();  // the summaries are written
  if (blockIdx.y == 0) {
    const Summary all = fold(sums, gridDim.y, frame_len, s_warp);
    if (threadIdx.x == 0) {
      if (all.n == 0) {
        out_start[blockIdx.x] = kTextOnlyStart;
        out_amount[blockIdx.x] = 0;
      } else {
        const int64_t start = static_cast<int64_t>(all.last) + frame_len;
        const int64_t anchor = all.first + static_cast<int64_t>(all.n - 1) * span + all.gaps;
        out_start[blockIdx.x] = static_cast<int32_t>(start);
        out_amount[blockIdx.x] = static_cast<int32_t>(start - (anchor + span));
      }
    }
  }
  Summary carry = fold(sums, blockIdx.y, frame_len, s_warp);

  const int32_t* __restrict__ seq = ids + sl.first;
  int32_t* __restrict__ pt = pos + sl.first;
  int32_t* __restrict__ ph = pos + n_tokens + sl.first;
  int32_t* __restrict__ pw = pos + 2 * n_tokens + sl.first;
  const int64_t rows = static_cast<int64_t>(side) * side;
  for (int64_t c = sl.p0; c < sl.p1; c += kFrSliceTarget) {
    int32_t v[kFrPerThread];
#pragma unroll
    for (int m = 0; m < kFrPerThread; ++m) {
      const int64_t p = c + m * kFrThreads + threadIdx.x;
      v[m] = (p < sl.p1) ? __ldg(seq + p) : ~marker;
    }
#pragma unroll
    for (int m = 0; m < kFrPerThread; ++m) {
      const int64_t p = c + m * kFrThreads + threadIdx.x;
      const int32_t p32 = static_cast<int32_t>(p);
      Summary e = (v[m] == marker) ? Summary{1, p32, p32, 0} : Summary{0, 0, 0, 0};
      Summary total;
      const Summary incl = combine(carry, block_scan(e, frame_len, s_warp, &total), frame_len);
      carry = combine(carry, total, frame_len);
      if (p >= sl.p1) continue;
      int64_t t, h, w;
      if (incl.n == 0) {
        t = h = w = p;
      } else {
        const int64_t anchor = incl.first + static_cast<int64_t>(incl.n - 1) * span + incl.gaps;
        const int64_t d = p - incl.last;  // offset into the last frame opened
        if (d == 0) {
          t = anchor;
          h = w = anchor - 1;
        } else if (d <= rows) {
          const int64_t k = d - 1;
          t = anchor;
          h = anchor + k / side;
          w = anchor + k % side;
        } else if (d == rows + 1) {
          t = anchor;
          h = w = anchor + side;
        } else if (d == rows + 2) {
          t = h = w = anchor;
        } else {
          t = h = w = anchor + span + (d - frame_len);
        }
      }
      pt[p] = static_cast<int32_t>(t);
      ph[p] = static_cast<int32_t>(h);
      pw[p] = static_cast<int32_t>(w);
    }
  }
}

}  // namespace

int64_t frames_slices(int32_t num_seqs, int64_t n_tokens, size_t workspace_bytes) {
  if (num_seqs <= 0) return 0;
  const int64_t avg = (n_tokens + num_seqs - 1) / num_seqs;
  int64_t slices = (avg + kFrSliceTarget - 1) / kFrSliceTarget;
  slices = slices < 1 ? 1 : (slices > kFrMaxSlices ? kFrMaxSlices : slices);
  // a smaller workspace takes fewer, longer slices
  const int64_t fit = static_cast<int64_t>(workspace_bytes / (sizeof(Summary) * num_seqs));
  return slices < fit ? slices : fit;
}

size_t frames_summary_bytes() { return sizeof(Summary); }

// ---- built-in scratch for callers that cannot allocate device memory ----
//
// cmr_positions_frames_noalloc keeps its slice summaries here instead of in a
// caller's workspace: kStaticFrameSummaries summaries of 16 bytes (256 KB),
// held by every device that loads the library until the process exits.  All
// calls share it, so calls that overlap on the device race; a call writes
// every summary it reads, so nothing needs clearing between calls.
constexpr int64_t kStaticFrameSummaries = 16384;
static __device__ __align__(256) Summary g_frame_scratch[kStaticFrameSummaries];

// The device address of g_frame_scratch on the current device: in host code
// the array's name stands for a host-side shadow, not device memory, so the
// address is looked up once per device (with that device current) and cached.
cudaError_t frames_static_scratch(void** ptr, size_t* bytes) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_frame_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *ptr = addr[dev];
  *bytes = sizeof(g_frame_scratch);
  return cudaSuccess;
}

int64_t frames_static_max_seqs() { return kStaticFrameSummaries; }

cudaError_t launch_positions_frames(const int32_t* ids, const int32_t* cu_seqlens,
                                    int32_t num_seqs, int64_t n_tokens, int32_t image_token_id,
                                    int32_t grid_side, int32_t* out_pos, int32_t* out_start,
                                    int32_t* out_amount, void* workspace,
                                    size_t workspace_bytes, int32_t* device_status,
                                    cudaStream_t stream) {
  const int64_t slices = frames_slices(num_seqs, n_tokens, workspace_bytes);
  if (slices < 1) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(num_seqs), static_cast<unsigned>(slices));
  Summary* work = static_cast<Summary*>(workspace);
  const int32_t frame_len = grid_side * grid_side + 3;
  frames_summary_kernel<<<grid, kFrThreads, 0, stream>>>(ids, cu_seqlens, num_seqs, n_tokens,
                                                         image_token_id, frame_len, work,
                                                         device_status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return pdl::launch(frames_positions_kernel, grid, dim3(kFrThreads), 0, stream, true, ids,
                     cu_seqlens, num_seqs, n_tokens, image_token_id, grid_side,
                     static_cast<const Summary*>(work), out_pos, out_start, out_amount);
}

}  // namespace cmr
