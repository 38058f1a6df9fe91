// Canvas position planes (T, H, W) from token ids, on sm_100a.
//
// Rule: the canvas table of the HF card mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI,
// section "How the VLM rides the text-only engine", with start = O + 67 and
// amount = start - (O + 9) from the Core AI port notes ("The canvas rule and
// why the gate is on the planes").  The port notes' CoreAIKit section gives
// Qwen-VL's shift for comparison (+64 from the pads, 56: start = O + 65), and
// the LiteRT card's runtime uses plain 1-D positions; both are selectable.
//
// Work split: two kernels.
//   1. canvas_origin_kernel, one CTA per prompt chunk (or, for long chunks, a
//      cluster of K <= 16 CTAs that deal the blocks of ids round-robin and
//      exchange their minima through distributed shared memory after each
//      round),
//      finds the chunk's first marker (16 loads in flight per thread, warp
//      `redux.sync` min, a shared-memory min) and stops at the first block
//      (round) of ids that holds one, so no id is read twice; it writes the
//      chunk's outgoing state (start, amount) -- carried over when a frame is
//      already known, (2^30, 0) for text and for the 1-D rule.
//   2. canvas_positions_kernel, CTAs (b, s) over slices of 2,048 to 8,192 tokens,
//      launched programmatically behind the first (it starts while the scan
//      runs and waits for it before reading the state), writes the planes:
//      12 B per token, no ids read.
// No CTA waits on another and there is no scratch memory; the state passes
// through the caller's out_start / out_amount.  The one-call path
// (cmr_positions_rotate_qk) launches only the first kernel and lets the
// rotation write the planes.
#include <cooperative_groups.h>

#include <climits>
#include <mutex>

#include "canvas.cuh"
#include "pdl.cuh"

namespace cg = cooperative_groups;

namespace cmr {
namespace {

constexpr int kOriginThreads = 1024;
constexpr int kIdsPerThread = 16;
constexpr int kScanChunk = kOriginThreads * kIdsPerThread;  // 16,384 ids per step
constexpr int kPosThreads = 512;
constexpr int kSliceMin = 2048;                             // tokens per planes CTA, and
constexpr int kSliceMax = 8192;                             //   for batches of many waves
constexpr int kMaxSlices = 65535;                           // gridDim.y limit
constexpr int kQwenVlFrameShift = kGridRows + 1;            // start = O + 65
constexpr int kOriginMaxCluster = 16;                       // CTAs per long chunk
constexpr int kPortableCluster = 8;                         // above: opt-in per kernel

// The ids of the block seq[c, c + kScanChunk) this thread reads (16 loads in
// flight), entries past len reading as a non-marker.
__device__ __forceinline__ void load_block(const int32_t* __restrict__ seq, int64_t c,
                                           int64_t len, int32_t marker,
                                           int32_t (&v)[kIdsPerThread]) {
#pragma unroll
  for (int m = 0; m < kIdsPerThread; ++m) {
    const int64_t e = c + m * kOriginThreads + threadIdx.x;
    v[m] = (e < len) ? __ldg(seq + e) : ~marker;
  }
}

// Smallest offset in a block of ids (loaded by load_block) whose id is the
// marker, or INT_MAX.  Block-uniform result; all threads of the CTA must call
// it.
__device__ __forceinline__ int block_min(const int32_t (&v)[kIdsPerThread], int32_t marker,
                                         int* s_warp_min) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  int best = INT_MAX;  // offset within the block; smaller m = smaller index
#pragma unroll
  for (int m = kIdsPerThread - 1; m >= 0; --m)
    if (v[m] == marker) best = m * kOriginThreads + threadIdx.x;
  best = __reduce_min_sync(0xffffffffu, best);
  if (lane == 0) s_warp_min[warp] = best;
  __syncthreads();
  int block_best = INT_MAX;
#pragma unroll
  for (int i = 0; i < kOriginThreads / 32; ++i) block_best = min(block_best, s_warp_min[i]);
  __syncthreads();  // s_warp_min is rewritten by the next block
  return block_best;
}

// Smallest local index in seq[0, len) whose id is the marker, or -1.
// Block-uniform result; all threads of the CTA must call it.
__device__ __forceinline__ int64_t first_marker(const int32_t* __restrict__ seq, int64_t len,
                                                int32_t marker, int* s_warp_min) {
  for (int64_t c = 0; c < len; c += kScanChunk) {
    int32_t v[kIdsPerThread];
    load_block(seq, c, len, marker, v);
    const int best = block_min(v, marker, s_warp_min);
    if (best != INT_MAX) return c + best;
  }
  return -1;
}

// first_marker by the K CTAs of this CTA's cluster: in round i, rank r scans
// block i * K + r; each warp's minimum goes straight into the leader CTA's
// slot for the round (an atomicMin in its shared memory, through distributed
// shared memory), one cluster barrier ends the round, and lane 0 of every
// warp reads the slot back for its warp; all stop at the first round that
// found a marker.  Three slots rotate: the leader resets the slot of round
// i + 2 after round i's barrier, when every CTA has read it (in round i - 1)
// and none can write it before round i + 1's barrier.  Each rank's loads for
// the next round are issued before the exchange; no id is read twice, and
// at most one round past the first marker is read.  Cluster-uniform result;
// every thread of every CTA of the cluster must call it.  Local indices fit
// in int32 (a chunk's length comes from int32 cu_seqlens).
__device__ __forceinline__ int64_t first_marker_cluster(const int32_t* __restrict__ seq,
                                                        int64_t len, int32_t marker,
                                                        int* s_slots) {
  cg::cluster_group cluster = cg::this_cluster();
  const int64_t K = cluster.num_blocks();
  const int64_t r = cluster.block_rank();
  const int lane = threadIdx.x & 31;
  const int64_t blocks = (len + kScanChunk - 1) / kScanChunk;
  int* const leader = cluster.map_shared_rank(s_slots, 0);
  if (threadIdx.x < 3) s_slots[threadIdx.x] = INT_MAX;
  cluster.sync();  // the leader's slots are set before any rank writes them
  int64_t result = -1;
  int32_t v[kIdsPerThread];
  load_block(seq, r * kScanChunk, len, marker, v);
  for (int64_t i = 0; i * K < blocks; ++i) {
    const int64_t c = (i * K + r) * kScanChunk;
    int best = INT_MAX;
    if (c < len) {
#pragma unroll
      for (int m = kIdsPerThread - 1; m >= 0; --m)
        if (v[m] == marker) best = static_cast<int>(c) + m * kOriginThreads + threadIdx.x;
    }
    best = __reduce_min_sync(0xffffffffu, best);
    if ((i + 1) * K < blocks) load_block(seq, c + K * kScanChunk, len, marker, v);
    const int slot = static_cast<int>(i % 3);
    if (lane == 0 && best != INT_MAX) atomicMin(leader + slot, best);
    cluster.sync();
    if (r == 0 && threadIdx.x == 0) s_slots[(i + 2) % 3] = INT_MAX;
    int all = 0;
    if (lane == 0) all = leader[slot];
    all = __shfl_sync(0xffffffffu, all, 0);
    if (all != INT_MAX) {
      result = all;
      break;
    }
  }
  cluster.sync();  // no CTA leaves while a peer may still read or write its slots
  return result;
}

// Bounds of prompt chunk b; false (uniform over the CTA) when cu_seqlens is
// malformed around b.
__device__ __forceinline__ bool chunk_bounds(const int32_t* __restrict__ cu, int32_t num_seqs,
                                             int64_t n_tokens, int32_t b, int64_t* first,
                                             int64_t* len) {
  const int64_t f = __ldg(cu + b);
  const int64_t l = __ldg(cu + b + 1);
  if (f < 0 || l < f || l > n_tokens || (b == 0 && f != 0) ||
      (b == num_seqs - 1 && l != n_tokens))
    return false;
  *first = f;
  *len = l - f;
  return true;
}

// kCluster: launched in clusters of K CTAs per chunk (grid num_seqs * K);
// otherwise one CTA per chunk.
template <bool kCluster>
__global__ void __launch_bounds__(kOriginThreads)
    canvas_origin_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ cu,
                         int32_t num_seqs, int64_t n_tokens, int32_t marker, int32_t rule,
                         const int32_t* __restrict__ pos_offset,
                         const int32_t* __restrict__ in_start,
                         const int32_t* __restrict__ in_amount, int32_t* __restrict__ out_start,
                         int32_t* __restrict__ out_amount, int32_t* __restrict__ status) {
  __shared__ int s_warp_min[kOriginThreads / 32];
  __shared__ int s_slots[3];
  pdl::launch_dependents();
  // the chunk of this CTA (of its cluster), and whether it writes the results
  int32_t b = blockIdx.x;
  bool leader = true;
  if constexpr (kCluster) {
    cg::cluster_group cluster = cg::this_cluster();
    b = static_cast<int32_t>(blockIdx.x / cluster.num_blocks());
    leader = cluster.block_rank() == 0;
  }
  int64_t first, len;
  // every CTA of a cluster takes the same branches below (same chunk)
  if (!chunk_bounds(cu, num_seqs, n_tokens, b, &first, &len)) {
    if (leader && threadIdx.x == 0 && status != nullptr)
      atomicOr(status, CMR_DEVICE_BAD_CU_SEQLENS);
    return;
  }
  // The sequence's state before this chunk: (2^30, 0) while no frame is known.
  int64_t start = in_start ? __ldg(in_start + b) : kTextOnlyStart;
  int64_t amount = in_amount ? __ldg(in_amount + b) : 0;
  if (rule == CMR_RULE_PLANES_1D) {
    start = kTextOnlyStart;
    amount = 0;
  } else if (start >= kTextOnlyStart) {
    const int64_t m = kCluster ? first_marker_cluster(ids + first, len, marker, s_slots)
                               : first_marker(ids + first, len, marker, s_warp_min);
    if (m >= 0) {
      const int64_t origin = (pos_offset ? __ldg(pos_offset + b) : 0) + m;
      start = origin + (rule == CMR_RULE_QWEN_VL ? kQwenVlFrameShift : kFrameTokens);
      amount = start - (origin + kCanvasSpan);
    } else {
      start = kTextOnlyStart;
      amount = 0;
    }
  }
  if (leader && threadIdx.x == 0) {
    out_start[b] = static_cast<int32_t>(start);
    out_amount[b] = static_cast<int32_t>(amount);
  }
}

__global__ void __launch_bounds__(kPosThreads)
    canvas_positions_kernel(const int32_t* __restrict__ cu, int32_t num_seqs, int64_t n_tokens,
                            const int32_t* __restrict__ pos_offset, const int32_t* state_start,
                            const int32_t* state_amount, int32_t* __restrict__ pos) {
  const int32_t b = blockIdx.x;
  int64_t first, len;
  if (!chunk_bounds(cu, num_seqs, n_tokens, b, &first, &len)) return;
  const int64_t per = (len + gridDim.y - 1) / gridDim.y;
  const int64_t p0 = min(len, static_cast<int64_t>(blockIdx.y) * per);
  const int64_t p1 = min(len, p0 + per);
  if (p0 >= p1) return;
  const int64_t offset = pos_offset ? __ldg(pos_offset + b) : 0;
  pdl::wait();  // the origin kernel's state is written
  const int64_t start = __ldcg(state_start + b);
  const int64_t amount = __ldcg(state_amount + b);
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

// Whether clusters of more than kPortableCluster origin CTAs are enabled on the
// current device: the opt-in is a function attribute, set once per device
// and never while `stream` is being captured (that call then keeps to the
// portable size).
bool origin_large_clusters(cudaStream_t stream) {
  static std::mutex mu;
  static bool enabled[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return false;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (enabled[dev]) return true;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (cap != cudaStreamCaptureStatusNone) return false;
  if (cudaFuncSetAttribute(canvas_origin_kernel<true>,
                           cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  enabled[dev] = true;
  return true;
}

// Whether the current device can hold at least one cluster of k origin CTAs
// (occupancy query, no launch; cached per device and k).
bool origin_clusters_fit(int k, const cudaLaunchConfig_t& cfg) {
  static std::mutex mu;
  static int8_t known[64][kOriginMaxCluster + 1] = {};  // 0 unknown, 1 fits, -1 does not
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return false;
  }
  std::lock_guard<std::mutex> lock(mu);
  int8_t& state = known[dev][k];
  if (state == 0) {
    cudaLaunchConfig_t one = cfg;
    one.gridDim = dim3(static_cast<unsigned>(k));
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, canvas_origin_kernel<true>, &one) !=
        cudaSuccess) {
      cudaGetLastError();
      return false;  // not cached: the next call asks again
    }
    state = clusters > 0 ? 1 : -1;
  }
  return state > 0;
}

}  // namespace

cudaError_t launch_positions_origin(const int32_t* ids, const int32_t* cu_seqlens,
                                   int32_t num_seqs, int64_t n_tokens, int32_t image_token_id,
                                   int32_t rule, const int32_t* pos_offset,
                                   const int32_t* in_start, const int32_t* in_amount,
                                   int32_t* out_start, int32_t* out_amount,
                                   int32_t* device_status, cudaStream_t stream) {
  if (num_seqs == 0) return cudaSuccess;
  // Chunks averaging more than two blocks of ids get a cluster of K CTAs: K a
  // power of two up to kOriginMaxCluster, one CTA per two blocks, and no
  // more CTAs in all than the SMs (each cluster CTA fills an SM), so that
  // every cluster runs in the first wave.
  const int64_t avg = (n_tokens + num_seqs - 1) / num_seqs;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  int k = 1;
  while (k < kOriginMaxCluster && static_cast<int64_t>(k) * 2 * kScanChunk < avg &&
         static_cast<int64_t>(num_seqs) * 2 * k <= 2 * static_cast<int64_t>(sms))
    k *= 2;
  if (k > kPortableCluster && !origin_large_clusters(stream)) k = kPortableCluster;
  if (k == 1) {
    canvas_origin_kernel<false><<<static_cast<unsigned>(num_seqs), kOriginThreads, 0, stream>>>(
        ids, cu_seqlens, num_seqs, n_tokens, image_token_id, rule, pos_offset, in_start,
        in_amount, out_start, out_amount, device_status);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(static_cast<int64_t>(num_seqs) * k));
  cfg.blockDim = dim3(kOriginThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(k);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (!origin_clusters_fit(k, cfg)) {
    // a device (or a share of one) that cannot place such clusters: one CTA
    // per chunk gives the same results
    canvas_origin_kernel<false><<<static_cast<unsigned>(num_seqs), kOriginThreads, 0, stream>>>(
        ids, cu_seqlens, num_seqs, n_tokens, image_token_id, rule, pos_offset, in_start,
        in_amount, out_start, out_amount, device_status);
    return cudaGetLastError();
  }
  return cudaLaunchKernelEx(&cfg, canvas_origin_kernel<true>, ids, cu_seqlens, num_seqs,
                            n_tokens, image_token_id, rule, pos_offset, in_start, in_amount,
                            out_start, out_amount, device_status);
}

cudaError_t launch_positions(const int32_t* ids, const int32_t* cu_seqlens, int32_t num_seqs,
                             int64_t n_tokens, int32_t image_token_id, int32_t rule,
                             const int32_t* pos_offset, const int32_t* in_start,
                             const int32_t* in_amount, int32_t* out_pos, int32_t* out_start,
                             int32_t* out_amount, int32_t* device_status, cudaStream_t stream) {
  if (num_seqs == 0) return cudaSuccess;
  cudaError_t e = launch_positions_origin(ids, cu_seqlens, num_seqs, n_tokens, image_token_id,
                                          rule, pos_offset, in_start, in_amount, out_start,
                                          out_amount, device_status, stream);
  if (e != cudaSuccess || n_tokens == 0) return e;
  // Slices of kSliceMin tokens, or of kSliceMax where even those leave at
  // least three resident waves of CTAs: each CTA's start (the bounds, the
  // programmatic wait, the state) is two dependent memory round trips, which
  // long slices spread over more stores, while a grid of one or two waves
  // loses more to its partly filled last wave than it saves.
  const int64_t avg = (n_tokens + num_seqs - 1) / num_seqs;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  const int64_t wave = static_cast<int64_t>(sms) * (2048 / kPosThreads);
  int64_t slices = (avg + kSliceMax - 1) / kSliceMax;
  if (static_cast<int64_t>(num_seqs) * slices < 3 * wave)
    slices = (avg + kSliceMin - 1) / kSliceMin;
  slices = slices < 1 ? 1 : (slices > kMaxSlices ? kMaxSlices : slices);
  const dim3 grid(static_cast<unsigned>(num_seqs), static_cast<unsigned>(slices));
  return pdl::launch(canvas_positions_kernel, grid, dim3(kPosThreads), 0, stream, true,
                     cu_seqlens, num_seqs, n_tokens, pos_offset,
                     static_cast<const int32_t*>(out_start),
                     static_cast<const int32_t*>(out_amount), out_pos);
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
