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
//      of them for the state), then walks its slice in chunks of
//      kFrThreads x kFrItems tokens: each thread folds its own kFrItems
//      consecutive tokens, one block scan of the threads' summaries gives
//      each thread its prefix, and the thread walks its tokens again writing
//      their planes.
// Each thread owns 8 consecutive tokens at an 8-aligned index of the packed
// batch, so ids are read and planes written as 16-byte vectors (plane rows
// are 16-byte aligned when n_tokens is a multiple of 4; otherwise, and at
// the edges of a slice, element by element).  Ids are read twice (once per
// kernel; the second read mostly hits L2); the planes are written once.  No
// CTA waits on another.
#include <mutex>

#include "canvas.cuh"
#include "pdl.cuh"

namespace cmr {
namespace {

constexpr int kFrThreads = 256;
constexpr int kFrWarps = kFrThreads / 32;
constexpr int kFrItems = 8;                                  // consecutive tokens per thread
constexpr int kFrChunk = kFrThreads * kFrItems;              // 2048 tokens per block step
constexpr int kFrSliceTarget = kFrChunk;                     // tokens per CTA (target)
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

// Inclusive scan over the warp's lanes in lane order.  A warp holding no
// marker (the common case: frames are sparse) is all identities already.
__device__ __forceinline__ Summary warp_scan(Summary v, int32_t frame_len) {
  if (!__any_sync(0xffffffffu, v.n != 0)) return v;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const Summary u = shfl_up(v, d);
    if (lane >= d) v = combine(u, v, frame_len);
  }
  return v;
}

// Block-wide scans and reductions in thread order, with one barrier each.
// Each call takes the next of two shared buffers of warp totals (BlockBufs):
// two calls in a row never share a buffer, and a call reusing one runs after
// the barrier of the call between, which every thread passes only once it
// has read the older call's totals.  All threads must make the same calls.
struct BlockBufs {
  Summary warp[2][kFrWarps];
};

// Exclusive prefix of v in thread order (thread 0: the identity); *total
// receives the block's summary.
__device__ __forceinline__ Summary block_exclusive_scan(Summary v, int32_t frame_len,
                                                        BlockBufs& bufs, int& turn,
                                                        Summary* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  Summary* const buf = bufs.warp[turn];
  turn ^= 1;
  const Summary incl = warp_scan(v, frame_len);
  Summary excl = shfl_up(incl, 1);
  if (lane == 0) excl = Summary{0, 0, 0, 0};
  if (lane == 31) buf[warp] = incl;
  __syncthreads();
  Summary before{0, 0, 0, 0}, all{0, 0, 0, 0};
#pragma unroll
  for (int w = 0; w < kFrWarps; ++w) {
    const Summary t = buf[w];
    if (w < warp) before = combine(before, t, frame_len);
    all = combine(all, t, frame_len);
  }
  *total = all;
  return combine(before, excl, frame_len);
}

// The block's summary of v in thread order.
__device__ __forceinline__ Summary block_reduce(Summary v, int32_t frame_len, BlockBufs& bufs,
                                                int& turn) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  Summary* const buf = bufs.warp[turn];
  turn ^= 1;
  const Summary incl = warp_scan(v, frame_len);
  if (lane == 31) buf[warp] = incl;
  __syncthreads();
  Summary all{0, 0, 0, 0};
#pragma unroll
  for (int w = 0; w < kFrWarps; ++w) all = combine(all, buf[w], frame_len);
  return all;
}

// The kFrItems ids of the 8-aligned group at global index g of the packed
// batch; entries outside [lo, hi) read as `none`.  Two 16-byte loads when the
// group lies inside and ids is 16-byte aligned, else one load per id.
__device__ __forceinline__ void load_group(const int32_t* __restrict__ ids, int64_t g,
                                           int64_t lo, int64_t hi, int32_t none,
                                           int32_t (&v)[kFrItems]) {
  const bool aligned = (reinterpret_cast<uintptr_t>(ids) & 15u) == 0;
  if (aligned && g >= lo && g + kFrItems <= hi) {
    const int4 a = __ldg(reinterpret_cast<const int4*>(ids + g));
    const int4 b = __ldg(reinterpret_cast<const int4*>(ids + g) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
#pragma unroll
    for (int j = 0; j < kFrItems; ++j)
      v[j] = (g + j >= lo && g + j < hi) ? __ldg(ids + g + j) : none;
  }
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
  __shared__ BlockBufs bufs;
  int turn = 0;
  pdl::launch_dependents();
  bool bad;
  FrSlice sl;
  if (!fr_slice(cu, num_seqs, n_tokens, &bad, &sl)) {
    if (bad && blockIdx.y == 0 && threadIdx.x == 0 && status != nullptr)
      atomicOr(status, CMR_DEVICE_BAD_CU_SEQLENS);
    return;
  }
  // the slice as global indices of the packed batch, walked in 8-aligned
  // groups of kFrItems tokens, kFrChunk tokens per block step
  const int64_t lo = sl.first + sl.p0, hi = sl.first + sl.p1;
  Summary run{0, 0, 0, 0};
  for (int64_t c = lo & ~static_cast<int64_t>(kFrItems - 1); c < hi; c += kFrChunk) {
    const int64_t g = c + static_cast<int64_t>(threadIdx.x) * kFrItems;
    int32_t v[kFrItems];
    load_group(ids, g, lo, hi, ~marker, v);
    Summary mine{0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < kFrItems; ++j)
      if (v[j] == marker) {
        const int32_t p = static_cast<int32_t>(g + j - sl.first);  // local index
        mine = combine(mine, Summary{1, p, p, 0}, frame_len);
      }
    run = combine(run, block_reduce(mine, frame_len, bufs, turn), frame_len);
  }
  if (threadIdx.x == 0)
    work[static_cast<int64_t>(blockIdx.x) * gridDim.y + blockIdx.y] = run;
}

// Ordered fold of summaries[0, count) by the whole block.  The summaries come
// from the kernel before (plain loads, not the read-only path).
__device__ __forceinline__ Summary fold(const Summary* sums, int32_t count, int32_t frame_len,
                                        BlockBufs& bufs, int& turn) {
  Summary acc{0, 0, 0, 0};
  for (int32_t base = 0; base < count; base += kFrThreads) {
    const int32_t j = base + threadIdx.x;
    const Summary e = j < count ? sums[j] : Summary{0, 0, 0, 0};
    acc = combine(acc, block_reduce(e, frame_len, bufs, turn), frame_len);
  }
  return acc;
}

__global__ void __launch_bounds__(kFrThreads, 5)
    frames_positions_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ cu,
                            int32_t num_seqs, int64_t n_tokens, int32_t marker, int32_t side,
                            const Summary* work, int32_t* __restrict__ pos,
                            int32_t* __restrict__ out_start, int32_t* __restrict__ out_amount) {
  __shared__ BlockBufs bufs;
  int turn = 0;
  bool bad;
  FrSlice sl;
  if (!fr_slice(cu, num_seqs, n_tokens, &bad, &sl)) return;
  if (blockIdx.y != 0 && sl.p0 >= sl.p1) return;
  const int32_t frame_len = side * side + 3;
  const int64_t span = side + 1;  // counter advance per frame
  const Summary* sums = work + static_cast<int64_t>(blockIdx.x) * gridDim.y;
  pdl::wait();  // the summaries are written
  if (blockIdx.y == 0) {
    const Summary all = fold(sums, gridDim.y, frame_len, bufs, turn);
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
  Summary carry = fold(sums, blockIdx.y, frame_len, bufs, turn);

  const int64_t lo = sl.first + sl.p0, hi = sl.first + sl.p1;
  // per-token arithmetic in 32 bits: every coordinate fits in int32 (a
  // documented limit), and so does every intermediate below
  const int32_t rows = side * side;
  const uint32_t uside = static_cast<uint32_t>(side);
  const int32_t span32 = side + 1;
  // plane rows start 16-byte aligned when pos is and n_tokens is a multiple of 4
  const bool vec = (n_tokens & 3) == 0 && (reinterpret_cast<uintptr_t>(pos) & 15u) == 0;
  for (int64_t c = lo & ~static_cast<int64_t>(kFrItems - 1); c < hi; c += kFrChunk) {
    const int64_t g = c + static_cast<int64_t>(threadIdx.x) * kFrItems;
    int32_t v[kFrItems];
    load_group(ids, g, lo, hi, ~marker, v);
    Summary mine{0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < kFrItems; ++j)
      if (v[j] == marker) {
        const int32_t p = static_cast<int32_t>(g + j - sl.first);
        mine = combine(mine, Summary{1, p, p, 0}, frame_len);
      }
    Summary total;
    Summary pre = combine(carry, block_exclusive_scan(mine, frame_len, bufs, turn, &total),
                          frame_len);
    carry = combine(carry, total, frame_len);
    int32_t t[kFrItems], h[kFrItems], w[kFrItems];
#pragma unroll
    for (int j = 0; j < kFrItems; ++j) {
      const int32_t p = static_cast<int32_t>(g + j - sl.first);  // local index
      if (v[j] == marker) pre = combine(pre, Summary{1, p, p, 0}, frame_len);
      int32_t pt, ph, pw;
      if (pre.n == 0) {
        pt = ph = pw = p;
      } else {
        const int32_t anchor = pre.first + (pre.n - 1) * span32 + pre.gaps;
        const int32_t d = p - pre.last;  // offset into the last frame opened
        if (d == 0) {
          pt = anchor;
          ph = pw = anchor - 1;
        } else if (d <= rows) {
          const uint32_t k = static_cast<uint32_t>(d - 1);
          const uint32_t q = k / uside;
          pt = anchor;
          ph = anchor + static_cast<int32_t>(q);
          pw = anchor + static_cast<int32_t>(k - q * uside);
        } else if (d == rows + 1) {
          pt = anchor;
          ph = pw = anchor + side;
        } else if (d == rows + 2) {
          pt = ph = pw = anchor;
        } else {
          pt = ph = pw = anchor + span32 + (d - frame_len);
        }
      }
      t[j] = pt;
      h[j] = ph;
      w[j] = pw;
    }
    int32_t* const planes[3] = {pos + g, pos + n_tokens + g, pos + 2 * n_tokens + g};
    const int32_t* const vals[3] = {t, h, w};
    if (vec && g >= lo && g + kFrItems <= hi) {
#pragma unroll
      for (int r = 0; r < 3; ++r) {
        int4* dst = reinterpret_cast<int4*>(planes[r]);
        dst[0] = make_int4(vals[r][0], vals[r][1], vals[r][2], vals[r][3]);
        dst[1] = make_int4(vals[r][4], vals[r][5], vals[r][6], vals[r][7]);
      }
    } else {
#pragma unroll
      for (int j = 0; j < kFrItems; ++j)
        if (g + j >= lo && g + j < hi)
          for (int r = 0; r < 3; ++r) planes[r][j] = vals[r][j];
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
