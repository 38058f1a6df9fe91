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
// associative (not commutative) combine.  Each prompt b is cut into slices
// of about 4,096 tokens, and two kernels run over CTAs (b, slice):
//   1. frames_summary_kernel reduces its slice's tokens to that 16-byte
//      summary in a caller-provided workspace [num_seqs][slices], with the
//      ids of kFrSumUnroll block steps in flight before it folds any;
//   2. frames_positions_kernel, launched programmatically behind it, walks
//      the slices in the reverse of the summary kernel's order (the ids that
//      kernel read last are the likeliest to be in L2 still), loads its
//      first ids before it waits for the summaries, has one warp fold the
//      summaries of the slices before its own into a carry, then walks its
//      slice in chunks of kFrThreads x kFrItems tokens: each thread folds its
//      own kFrItems consecutive tokens, one block scan of the threads'
//      summaries gives each thread its prefix, and the thread walks its
//      tokens again writing their planes.  The CTA holding the prompt's last
//      token ends with the whole prompt's summary and writes its state.
// Each thread owns 8 consecutive tokens at an 8-aligned index of the packed
// batch, so ids are read as 16-byte vectors and each plane row is written in
// the widest stores its alignment allows (16 bytes when n_tokens is a
// multiple of 4, 8 when it is even; element by element at the edges of a
// slice).  A thread whose tokens are all text after a frame (or before the
// first) writes p + offset on every plane without the per-token cases.  Ids
// are read twice, once per kernel; the plane stores and the second reads are
// evict-first, so the second read finds the ids in L2 where it can.  No CTA
// waits on another.
#include <mutex>

#include "canvas.cuh"
#include "pdl.cuh"

namespace cmr {
namespace {

constexpr int kFrThreads = 256;
constexpr int kFrWarps = kFrThreads / 32;
constexpr int kFrItems = 8;                                  // consecutive tokens per thread
constexpr int kFrChunk = kFrThreads * kFrItems;              // 2048 tokens per block step
constexpr int kFrSliceTarget = 2 * kFrChunk;                 // tokens per slice (target)
constexpr int kFrMaxSlices = 65535;                          // gridDim.y limit
constexpr int kFrSumUnroll = 2;                              // summary block steps in flight
constexpr int kFrPosBlocks = 5;                              // positions CTAs per SM

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
  // a block without a marker (the common case) has identities everywhere
  if (!__syncthreads_or(v.n != 0)) {
    *total = Summary{0, 0, 0, 0};
    return excl;
  }
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
  if (!__syncthreads_or(v.n != 0)) return Summary{0, 0, 0, 0};
  Summary all{0, 0, 0, 0};
#pragma unroll
  for (int w = 0; w < kFrWarps; ++w) all = combine(all, buf[w], frame_len);
  return all;
}

// The kFrItems ids of the 8-aligned group at global index g of the packed
// batch; entries outside [lo, hi) read as `none`.  Two 16-byte loads when the
// group lies inside and ids is 16-byte aligned, else one load per id.  The
// summary kernel's loads keep normal L2 priority, so that the ids are still in
// L2 for the positions kernel's loads, the last of the call, which mark them
// evict-first (kLast).
template <bool kLast>
__device__ __forceinline__ int4 ld_ids4(const int32_t* p) {
  return kLast ? __ldcs(reinterpret_cast<const int4*>(p)) : __ldg(reinterpret_cast<const int4*>(p));
}
template <bool kLast>
__device__ __forceinline__ int32_t ld_id(const int32_t* p) {
  return kLast ? __ldcs(p) : __ldg(p);
}

template <bool kLast>
__device__ __forceinline__ void load_group(const int32_t* __restrict__ ids, int64_t g,
                                           int64_t lo, int64_t hi, int32_t none,
                                           int32_t (&v)[kFrItems]) {
  const bool aligned = (reinterpret_cast<uintptr_t>(ids) & 15u) == 0;
  if (aligned && g >= lo && g + kFrItems <= hi) {
    const int4 a = ld_ids4<kLast>(ids + g);
    const int4 b = ld_ids4<kLast>(ids + g + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
#pragma unroll
    for (int j = 0; j < kFrItems; ++j)
      v[j] = (g + j >= lo && g + j < hi) ? ld_id<kLast>(ids + g + j) : none;
  }
}

// A prompt's tokens [first, first + len) of the packed batch and the local
// range [p0, p1) of one of its slices (a prompt's length fits int32).
struct FrSlice {
  int64_t first;
  int32_t len, p0, p1;
};

// Prompt b of the batch: false (and *bad set) when its cu_seqlens entries
// are malformed.
__device__ __forceinline__ bool fr_prompt(const int32_t* __restrict__ cu, int32_t num_seqs,
                                          int64_t n_tokens, int32_t b, bool* bad, FrSlice* sl) {
  const int64_t first = __ldg(cu + b);
  const int64_t last = __ldg(cu + b + 1);
  *bad = first < 0 || last < first || last > n_tokens || (b == 0 && first != 0) ||
         (b == num_seqs - 1 && last != n_tokens);
  if (*bad) return false;
  sl->first = first;
  sl->len = static_cast<int32_t>(last - first);
  return true;
}

// Slice y of `slices` of the prompt: local tokens [p0, p1), ceil(len / slices)
// per slice (the last ones may be empty).
__device__ __forceinline__ void fr_range(uint32_t y, uint32_t slices, FrSlice* sl) {
  const uint32_t len = static_cast<uint32_t>(sl->len);
  const uint32_t per = len / slices + (len % slices != 0);
  const uint64_t p0 = static_cast<uint64_t>(y) * per;
  sl->p0 = static_cast<int32_t>(p0 < len ? p0 : len);
  sl->p1 = static_cast<int32_t>(min(len, static_cast<uint32_t>(sl->p0) + per));
}

// The summary of the marker tokens among v (local indices from p_base): a
// bit mask of the markers first, so that a group without one (nearly all of
// them) costs a compare per token.
__device__ __forceinline__ Summary fold_group(const int32_t (&v)[kFrItems], int32_t p_base,
                                              int32_t marker, int32_t frame_len) {
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < kFrItems; ++j) m |= static_cast<uint32_t>(v[j] == marker) << j;
  Summary mine{0, 0, 0, 0};
  while (m != 0) {
    const int32_t p = p_base + __ffs(m) - 1;
    m &= m - 1;
    mine = combine(mine, Summary{1, p, p, 0}, frame_len);
  }
  return mine;
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
  if (!fr_prompt(cu, num_seqs, n_tokens, blockIdx.x, &bad, &sl)) {
    if (bad && blockIdx.y == 0 && threadIdx.x == 0 && status != nullptr)
      atomicOr(status, CMR_DEVICE_BAD_CU_SEQLENS);
    return;
  }
  // the slice as global indices of the packed batch, walked in 8-aligned
  // groups of kFrItems tokens, kFrChunk tokens per block step; the groups of
  // kFrSumUnroll steps are loaded before any is folded
  fr_range(blockIdx.y, gridDim.y, &sl);
  const int64_t lo = sl.first + sl.p0, hi = sl.first + sl.p1;
  Summary run{0, 0, 0, 0};
  for (int64_t c = lo & ~static_cast<int64_t>(kFrItems - 1); c < hi;
       c += kFrSumUnroll * kFrChunk) {
    int32_t v[kFrSumUnroll][kFrItems];
#pragma unroll
    for (int u = 0; u < kFrSumUnroll; ++u)
      load_group<false>(ids, c + u * kFrChunk + static_cast<int64_t>(threadIdx.x) * kFrItems, lo,
                        hi, ~marker, v[u]);
#pragma unroll
    for (int u = 0; u < kFrSumUnroll; ++u) {
      if (c + u * kFrChunk >= hi) break;  // the same for every thread
      const int64_t g = c + u * kFrChunk + static_cast<int64_t>(threadIdx.x) * kFrItems;
      const Summary mine = fold_group(v[u], static_cast<int32_t>(g - sl.first), marker, frame_len);
      run = combine(run, block_reduce(mine, frame_len, bufs, turn), frame_len);
    }
  }
  if (threadIdx.x == 0) work[static_cast<int64_t>(blockIdx.x) * gridDim.y + blockIdx.y] = run;
}

// Ordered fold of summaries[0, count) by one warp (all 32 lanes call it);
// every lane receives the result.  The summaries come from the kernel before
// (plain loads, not the read-only path).
__device__ __forceinline__ Summary warp_fold(const Summary* sums, int32_t count,
                                             int32_t frame_len) {
  const int lane = threadIdx.x & 31;
  Summary acc{0, 0, 0, 0};
  for (int32_t base = 0; base < count; base += 32) {
    const int32_t j = base + lane;
    Summary e = j < count ? sums[j] : Summary{0, 0, 0, 0};
    e = warp_scan(e, frame_len);
    const Summary all = {__shfl_sync(0xffffffffu, e.n, 31), __shfl_sync(0xffffffffu, e.first, 31),
                         __shfl_sync(0xffffffffu, e.last, 31),
                         __shfl_sync(0xffffffffu, e.gaps, 31)};
    acc = combine(acc, all, frame_len);
  }
  return acc;
}

// Four consecutive plane values at dst, in the widest stores dst's alignment
// allows (16, 8 or 4 bytes; the same for every thread of a plane row, whose
// groups start at multiples of 8 tokens).  The planes are written once and
// not read back here: evict-first stores, which leave the ids in L2 for the
// positions kernel's second read.
__device__ __forceinline__ void store4(int32_t* dst, int32_t a, int32_t b, int32_t c, int32_t d) {
  const uintptr_t al = reinterpret_cast<uintptr_t>(dst);
  if ((al & 15u) == 0) {
    __stcs(reinterpret_cast<int4*>(dst), make_int4(a, b, c, d));
  } else if ((al & 7u) == 0) {
    __stcs(reinterpret_cast<int2*>(dst), make_int2(a, b));
    __stcs(reinterpret_cast<int2*>(dst) + 1, make_int2(c, d));
  } else {
    __stcs(dst, a);
    __stcs(dst + 1, b);
    __stcs(dst + 2, c);
    __stcs(dst + 3, d);
  }
}

__global__ void __launch_bounds__(kFrThreads, kFrPosBlocks)
    frames_positions_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ cu,
                            int32_t num_seqs, int64_t n_tokens, int32_t marker, int32_t side,
                            uint32_t side_magic, const Summary* work, int32_t* __restrict__ pos,
                            int32_t* __restrict__ out_start, int32_t* __restrict__ out_amount) {
  __shared__ BlockBufs bufs;
  __shared__ Summary s_carry;
  int turn = 0;
  bool bad;
  FrSlice sl;
  // slices in the reverse of the summary kernel's order: the ids it read last
  // are the likeliest to be in L2 still
  const uint32_t bx = gridDim.x - 1 - blockIdx.x, by = gridDim.y - 1 - blockIdx.y;
  if (!fr_prompt(cu, num_seqs, n_tokens, static_cast<int32_t>(bx), &bad, &sl)) return;
  fr_range(by, gridDim.y, &sl);
  // The CTA holding the prompt's last token (slice 0 of an empty prompt)
  // ends with the summary of the whole prompt and writes its state.
  const bool writer = sl.len == 0 ? by == 0 : (sl.p0 < sl.p1 && sl.p1 == sl.len);
  if (sl.p0 >= sl.p1 && !writer) return;
  const int32_t frame_len = side * side + 3;
  const int64_t lo = sl.first + sl.p0, hi = sl.first + sl.p1;
  const int64_t c0 = lo & ~static_cast<int64_t>(kFrItems - 1);
  // The first group of ids is an input that the summary kernel never writes:
  // it is loaded before the wait, so its latency overlaps that kernel's tail.
  int32_t v[kFrItems];
  if (c0 < hi)
    load_group<true>(ids, c0 + static_cast<int64_t>(threadIdx.x) * kFrItems, lo, hi, ~marker, v);
  pdl::wait();  // the summaries are written
  // warp 0 folds the summaries of the slices before this one; the other
  // warps read the carry after the first block scan's barrier
  if (threadIdx.x < 32) {
    const Summary before =
        warp_fold(work + static_cast<int64_t>(bx) * gridDim.y, by, frame_len);
    if (threadIdx.x == 0) s_carry = before;
  }
  Summary carry{0, 0, 0, 0};  // the prompt's summary up to the current chunk

  // per-token arithmetic in 32 bits: every coordinate fits in int32 (a
  // documented limit), and so does every intermediate below
  const int32_t rows = side * side;
  const int32_t span32 = side + 1;  // counter advance per frame
  for (int64_t c = c0; c < hi; c += kFrChunk) {
    const int64_t g = c + static_cast<int64_t>(threadIdx.x) * kFrItems;
    if (c != c0) load_group<true>(ids, g, lo, hi, ~marker, v);
    const int32_t p_base = static_cast<int32_t>(g - sl.first);  // local index of v[0]
    const Summary mine = fold_group(v, p_base, marker, frame_len);
    Summary total;
    const Summary excl = block_exclusive_scan(mine, frame_len, bufs, turn, &total);
    if (c == c0) carry = s_carry;  // written before that scan's barrier
    Summary pre = combine(carry, excl, frame_len);
    carry = combine(carry, total, frame_len);
    const bool inside = g >= lo && g + kFrItems <= hi;
    if (mine.n == 0 && (pre.n == 0 || p_base - pre.last > rows + 2)) {
      // no marker among the thread's tokens and none of them inside a frame:
      // all text, (p + off) on every plane
      const int32_t off =
          pre.n == 0 ? 0
                     : pre.first + (pre.n - 1) * span32 + pre.gaps + span32 - frame_len - pre.last;
      const int32_t b = p_base + off;
      if (inside) {
#pragma unroll
        for (int r = 0; r < 3; ++r) {
          store4(pos + r * n_tokens + g, b, b + 1, b + 2, b + 3);
          store4(pos + r * n_tokens + g + 4, b + 4, b + 5, b + 6, b + 7);
        }
      } else {
#pragma unroll
        for (int j = 0; j < kFrItems; ++j)
          if (g + j >= lo && g + j < hi)
            for (int r = 0; r < 3; ++r) __stcs(pos + r * n_tokens + g + j, b + j);
      }
      continue;
    }
    // the planes of the thread's tokens, four at a time
#pragma unroll
    for (int half = 0; half < kFrItems / 4; ++half) {
      int32_t t[4], h[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int j = 4 * half + i;
        const int32_t p = p_base + j;  // local index
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
            // row k = d - 1 of the grid: k / side by a multiply-high with
            // ceil(2^32 / side), exact since k * side < side^3 <= 2^21
            const uint32_t k = static_cast<uint32_t>(d - 1);
            const uint32_t q = __umulhi(k, side_magic);
            pt = anchor;
            ph = anchor + static_cast<int32_t>(q);
            pw = anchor + static_cast<int32_t>(k - q * static_cast<uint32_t>(side));
          } else if (d == rows + 1) {
            pt = anchor;
            ph = pw = anchor + side;
          } else if (d == rows + 2) {
            pt = ph = pw = anchor;
          } else {
            pt = ph = pw = anchor + span32 + (d - frame_len);
          }
        }
        t[i] = pt;
        h[i] = ph;
        w[i] = pw;
      }
      const int64_t gh = g + 4 * half;
      int32_t* const planes[3] = {pos + gh, pos + n_tokens + gh, pos + 2 * n_tokens + gh};
      const int32_t* const vals[3] = {t, h, w};
      if (inside) {
#pragma unroll
        for (int r = 0; r < 3; ++r)
          store4(planes[r], vals[r][0], vals[r][1], vals[r][2], vals[r][3]);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (gh + i >= lo && gh + i < hi)
            for (int r = 0; r < 3; ++r) __stcs(planes[r] + i, vals[r][i]);
      }
    }
  }
  if (writer && threadIdx.x == 0) {
    // an empty prompt ran no chunk: its carry is slice 0's, the identity
    if (carry.n == 0) {
      out_start[bx] = kTextOnlyStart;
      out_amount[bx] = 0;
    } else {
      const int64_t span = side + 1;
      const int64_t start = static_cast<int64_t>(carry.last) + frame_len;
      const int64_t anchor = carry.first + static_cast<int64_t>(carry.n - 1) * span + carry.gaps;
      out_start[bx] = static_cast<int32_t>(start);
      out_amount[bx] = static_cast<int32_t>(start - (anchor + span));
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
  // ceil(2^32 / side); side 1 has only grid row 0, for which 0 serves
  const uint32_t side_magic =
      grid_side == 1 ? 0u
                     : static_cast<uint32_t>(((uint64_t{1} << 32) + grid_side - 1) / grid_side);
  return pdl::launch(frames_positions_kernel, grid, dim3(kFrThreads), 0, stream, true, ids,
                     cu_seqlens, num_seqs, n_tokens, image_token_id, grid_side, side_magic,
                     static_cast<const Summary*>(work), out_pos, out_start, out_amount);
}

}  // namespace cmr
