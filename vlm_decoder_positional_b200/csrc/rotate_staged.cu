// Staged form of the fused cos/sin + rotate of Q and K (rot_dim 64): the
// rotated 128 B of each head row travel HBM -> shared memory -> HBM as TMA
// boxes through a ring of stages, and the threads only rotate in shared memory.
// Same math, same bits as rotate_qk_kernel (rotate.cu): frequency j of F = 32
// reads the plane the interleaved sections give it, a = pos[plane_j][t] *
// theta^(-2j/64), and turns the pair (x_j, x_{j+32}) of every head (HF card
// mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI, "What it is"; port notes, the
// decoder's `_mrope_freq_masks` and `forward_stateful_core(cos_sin=...)`).
//
// Why staged: the op is bound by HBM and touches 128 of every 512 B of a head
// row.  Holding the rows in registers (rotate.cu) caps the bytes in flight per
// SM at what the register file allows; TMA boxes in shared memory keep several
// layers' rows of a tile in flight with a handful of threads, and the copy
// engine forms the strided 128-B requests itself.
//
// One CTA per tile of kTileTokens tokens (a one-shot grid):
//   - Q is viewed as a 4-D tensor {d, t, h, l} = {head_dim, N, hq, L} and K as
//     {head_dim, N, hk, L}; a box {64, kTileTokens, heads, 1} is the rotated
//     dims of every head of the tile's tokens in one layer, landing in shared
//     memory as [h][t][64 dims] rows of 128 B, 128-B swizzled;
//   - stage = the Q box and the K box of one layer; min(kStages, layers) stages
//     in a ring (shared memory is sized to the stages used, so that 1- and
//     2-layer batches fit more CTAs on an SM);
//   - one producer thread waits for a free stage, arms its "full" mbarrier with
//     the boxes' bytes and issues the two loads (layer after layer);
//   - kConsumers threads, four per token (8 frequencies each), compute their
//     cos/sin once and rotate their 2 x 16 B of every row of every layer in
//     shared memory, then one of them stores the boxes back with TMA and frees
//     the previous stage once its store has read it.
// Launches that move up to 4 L2 sizes mark their loads and stores evict-first
// in L2 (host side, below, has the measurements behind that choice).
// Every mbarrier wait is bounded (tma::kWaitLimitNs): on time-out the kernel
// ORs CMR_DEVICE_WAIT_TIMEOUT into the status word, waits (bounded again) for
// the loads it issued, and returns.
#include <mutex>

#include "pdl.cuh"
#include "rotate_common.cuh"
#include "tma.cuh"

namespace cmr {
namespace {

using namespace rot;

constexpr int kStagedRotDim = 64;
constexpr int kUnits = kStagedRotDim / 16;             // 4 threads per token
constexpr uint32_t kRowBytes = kStagedRotDim * 2;      // 128 B: one swizzle span
constexpr int kTileTokens = 8;                         // tokens per CTA
constexpr int kStages = 3;                             // ring depth (at most)
constexpr int kConsumers = kTileTokens * kUnits;       // 32
constexpr int kThreads = kConsumers + 32;              // + the producer warp
constexpr uint32_t kMaxStageBytes = 24 * 1024;         // keeps >= 2 CTAs per SM
static_assert(kTileTokens % 8 == 0, "the swizzle phase of a row is its token index mod 8");

struct StagedArgs {
  RotateArgs r;
  uint32_t q_box_bytes;  // 128 * kTileTokens * hq
  uint32_t k_box_bytes;  // 128 * kTileTokens * hk
  uint32_t stage_bytes;  // q_box_bytes + k_box_bytes (a multiple of 1024)
  int32_t stages;        // ring depth: min(kStages, num_layers)
  int32_t evict_first;   // loads and stores mark their L2 lines evict-first
};

__device__ __forceinline__ void report_timeout(int32_t* status) {
  if (status != nullptr) atomicOr(status, CMR_DEVICE_WAIT_TIMEOUT);
}

template <bool kFromShift>
__global__ void __launch_bounds__(kThreads)
    rotate_qk_staged_kernel(const __grid_constant__ CUtensorMap q_map,
                            const __grid_constant__ CUtensorMap k_map, const StagedArgs args,
                            const FreqTable table) {
  __shared__ double s_inv[kStagedRotDim / 2];
  __shared__ int32_t s_plane[kStagedRotDim / 2];
  extern __shared__ uint8_t dyn[];
  // ring of stages, 1024-B aligned for the 128-B swizzle, then the barriers
  const uint32_t dyn_addr = tma::smem_addr(dyn);
  const uint32_t ring = (dyn_addr + 1023u) & ~1023u;
  uint8_t* const ring_ptr = dyn + (ring - dyn_addr);
  const int S = args.stages;
  const uint32_t full0 = ring + S * args.stage_bytes;  // full[s] = full0 + 8 s
  const uint32_t empty0 = full0 + 8 * S;               // empty[s] = empty0 + 8 s

  for (int j = threadIdx.x; j < kStagedRotDim / 2; j += blockDim.x) {
    s_inv[j] = table.inv_freq[j];
    s_plane[j] = table.plane[j];
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      tma::mbar_init(full0 + 8 * s, 1);
      tma::mbar_init(empty0 + 8 * s, 1);
    }
    tma::mbar_init_fence();
  }
  __syncthreads();

  const int L = args.r.num_layers;
  const int hq = args.r.hq, hk = args.r.hk;
  const int t0 = static_cast<int>(blockIdx.x) * kTileTokens;

  if (threadIdx.x >= kConsumers) {
    if (threadIdx.x != kConsumers) return;
    // ---- producer: layer l goes to stage s = l % S, in use number l / S ----
    int issued = 0;
    int s = 0;
    uint32_t phase = 0;  // (l / S) & 1
    for (int l = 0; l < L; ++l) {
      // a fresh barrier counts as having completed the phase before its first
      if (!tma::mbar_wait(empty0 + 8 * s, phase ^ 1u)) {
        report_timeout(args.r.status);
        break;
      }
      const uint32_t full = full0 + 8 * s;
      tma::mbar_arrive_expect_tx(full, args.stage_bytes);
      const uint32_t dst = ring + s * args.stage_bytes;
      if (args.evict_first) {
        const uint64_t pol = tma::l2_evict_first_policy();
        if (hq > 0) tma::load_4d_hint(dst, &q_map, full, 0, t0, 0, l, pol);
        if (hk > 0) tma::load_4d_hint(dst + args.q_box_bytes, &k_map, full, 0, t0, 0, l, pol);
      } else {
        if (hq > 0) tma::load_4d(dst, &q_map, full, 0, t0, 0, l);
        if (hk > 0) tma::load_4d(dst + args.q_box_bytes, &k_map, full, 0, t0, 0, l);
      }
      ++issued;
      if (++s == S) {
        s = 0;
        phase ^= 1u;
      }
    }
    // no load may still be landing when the CTA's shared memory goes away
    for (int l = issued > S ? issued - S : 0; l < issued; ++l)
      if (!tma::mbar_wait(full0 + 8 * (l % S), static_cast<uint32_t>(l / S) & 1u))
        report_timeout(args.r.status);
    return;
  }

  // ---- consumers: thread (token tl, unit u) ----
  // Lanes 8p .. 8p+7 hold tokens p and p + 4 of their warp's eight, so that in
  // each 8-lane phase of a 16-B shared access the two tokens' rows, whose
  // swizzle differs in bit 2, cover all 32 banks once.
  const int lane = threadIdx.x & 31;
  const int u = lane & 3;
  const int tl = (threadIdx.x >> 5) * 8 + ((lane >> 3) | (((lane >> 2) & 1) << 2));
  const int64_t t = static_cast<int64_t>(t0) + tl;
  int32_t p0 = 0, p1 = 0, p2 = 0;  // rows past the last token are zeros and are not stored
  // The token's sequence and index come from cu_seqlens (and pos_offset),
  // which the kernels this one may be launched behind never write: the
  // search's chain of dependent loads runs before the wait below.
  int32_t seq = 0;
  int64_t idx = 0;
  if (kFromShift && t < args.r.n_tokens) token_seq(args.r, t, seq, idx);
  // Launched programmatically behind the positions kernels, the producer's
  // loads of Q and K (which those kernels never touch) are already under way;
  // pos (or the shift state) is ready after this wait.  Otherwise it returns
  // at once.
  pdl::wait();
  if (t < args.r.n_tokens) {
    if constexpr (kFromShift) {
      shift_planes(args.r, seq, idx, p0, p1, p2);
      if (args.r.pos_out != nullptr && u == 0) store_planes(args.r, t, p0, p1, p2);
    } else {
      token_planes<false>(args.r, t, p0, p1, p2);
    }
  }
  float c[8], s[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int j = 8 * u + e;
    const int pl = s_plane[j];
    cos_sin(pl == 0 ? p0 : (pl == 1 ? p1 : p2), s_inv[j], c[e], s[e]);
  }
  // 16-B chunk c of a row r sits at chunk position c ^ (r & 7); r & 7 = tl & 7.
  const uint32_t sw = static_cast<uint32_t>(tl & 7);
  const uint32_t off_x = (static_cast<uint32_t>(u) ^ sw) * 16u;
  const uint32_t off_y = (static_cast<uint32_t>(u + 4) ^ sw) * 16u;

  int st = 0, prev = S - 1;  // this layer's stage and the previous layer's
  uint32_t phase = 0;        // (l / S) & 1
  for (int l = 0; l < L; ++l) {
    const bool landed = tma::mbar_wait(full0 + 8 * st, phase, tma::kConsumerWaitLimitNs);
    if (tma::named_any(1, kConsumers, !landed)) {
      if (threadIdx.x == 0) report_timeout(args.r.status);
      break;
    }
    uint8_t* const stage = ring_ptr + st * args.stage_bytes;
    uint8_t* row = stage + static_cast<uint32_t>(tl) * kRowBytes;
    const int rows = hq + hk;  // the K box follows the Q box, same row pitch
#pragma unroll 2
    for (int h = 0; h < rows; ++h, row += kTileTokens * kRowBytes) {
      uint4* const px = reinterpret_cast<uint4*>(row + off_x);
      uint4* const py = reinterpret_cast<uint4*>(row + off_y);
      uint4 x1 = *px, x2 = *py;
      rotate_unit(x1, x2, c, s);
      *px = x1;
      *py = x2;
    }
    tma::fence_async_shared();
    tma::named_sync(1, kConsumers);
    if (threadIdx.x == 0) {
      const uint32_t src = ring + st * args.stage_bytes;
      if (args.evict_first) {
        const uint64_t pol = tma::l2_evict_first_policy();
        if (hq > 0) tma::store_4d_hint(&q_map, src, 0, t0, 0, l, pol);
        if (hk > 0) tma::store_4d_hint(&k_map, src + args.q_box_bytes, 0, t0, 0, l, pol);
      } else {
        if (hq > 0) tma::store_4d(&q_map, src, 0, t0, 0, l);
        if (hk > 0) tma::store_4d(&k_map, src + args.q_box_bytes, 0, t0, 0, l);
      }
      tma::bulk_commit();
      tma::bulk_wait_read<1>();  // the previous layer's store has read its stage
      if (l > 0) tma::mbar_arrive(empty0 + 8 * prev);
    }
    prev = st;
    if (++st == S) {
      st = 0;
      phase ^= 1u;
    }
  }
  if (threadIdx.x == 0) tma::bulk_wait_read<0>();
}

// ---- host side ----

// Tensor map of x [L, N, heads, head_dim] bf16 seen as {d, t, h, l}, with a
// {64, kTileTokens, heads, 1} box, 128-B swizzle.
bool encode_map(CUtensorMap* map, void* base, int64_t n_tokens, int heads, int layers,
                int head_dim) {
  const uint64_t row = static_cast<uint64_t>(head_dim) * 2;
  const uint64_t dims[4] = {static_cast<uint64_t>(head_dim), static_cast<uint64_t>(n_tokens),
                            static_cast<uint64_t>(heads), static_cast<uint64_t>(layers)};
  const uint64_t strides[3] = {row * heads, row, row * heads * static_cast<uint64_t>(n_tokens)};
  const uint32_t box[4] = {kStagedRotDim, kTileTokens, static_cast<uint32_t>(heads), 1};
  return encode_bf16_tensor_map(map, base, 4, dims, strides, box, true);
}

using StagedFn = void (*)(CUtensorMap, CUtensorMap, StagedArgs, FreqTable);

struct DeviceCache {
  std::mutex mu;
  bool smem_set[64][2] = {};
};
DeviceCache g_dev;

// Launches that move at most this many L2 sizes mark their lines evict-first.
constexpr int64_t kEvictFirstL2Multiple = 4;

}  // namespace

bool staged_rotate_fits(const RotateArgs& a) {
  const uint64_t stage = static_cast<uint64_t>(kRowBytes) * kTileTokens * (a.hq + a.hk);
  return a.rot_dim == kStagedRotDim && a.hq <= 256 && a.hk <= 256 && stage <= kMaxStageBytes &&
         a.n_tokens <= INT32_MAX;
}

int64_t staged_rotate_tiles(int64_t n_tokens) { return (n_tokens + kTileTokens - 1) / kTileTokens; }

// Launch the staged kernel; *launched is false (and nothing was enqueued)
// when the tensor maps cannot describe these buffers.
cudaError_t launch_rotate_qk_staged(const RotateArgs& a, const FreqTable& table,
                                    cudaStream_t stream, bool programmatic, bool* launched) {
  *launched = false;
  CUtensorMap q_map{}, k_map{};
  if (a.hq > 0 && !encode_map(&q_map, a.q, a.n_tokens, a.hq, a.num_layers, a.head_dim))
    return cudaSuccess;
  if (a.hk > 0 && !encode_map(&k_map, a.k, a.n_tokens, a.hk, a.num_layers, a.head_dim))
    return cudaSuccess;
  StagedArgs sa;
  sa.r = a;
  sa.q_box_bytes = kRowBytes * kTileTokens * a.hq;
  sa.k_box_bytes = kRowBytes * kTileTokens * a.hk;
  sa.stage_bytes = sa.q_box_bytes + sa.k_box_bytes;
  sa.stages = a.num_layers < kStages ? a.num_layers : kStages;
  const bool from_shift = a.pos == nullptr;
  const int64_t l2_bytes = device_l2_bytes();
  // L2 policy.  A launch that moves a few L2 sizes or less ends with most of
  // its rows still dirty in L2, and whatever reads them next competes with
  // their write-back (measured: the device-to-host copies of a 16,384-token,
  // 6-layer chunk ran about 20 % slower behind them); evict-first loads and
  // stores, like the register kernel's streaming accesses, avoid that.  A
  // larger launch keeps normal priority, which lets the L2 gather write-backs
  // (1.2 % faster on a 4-GB launch).
  const int64_t moved = 2 * static_cast<int64_t>(a.n_tokens) * a.num_layers * (a.hq + a.hk) *
                        static_cast<int64_t>(kRowBytes);
  sa.evict_first = moved <= kEvictFirstL2Multiple * l2_bytes ? 1 : 0;
  const int64_t tiles = staged_rotate_tiles(a.n_tokens);
  cudaError_t e;
  const StagedFn fn = from_shift ? rotate_qk_staged_kernel<true> : rotate_qk_staged_kernel<false>;
  const size_t smem = 1024 + static_cast<size_t>(sa.stages) * (sa.stage_bytes + 16);
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(g_dev.mu);
    // Only shapes whose ring exceeds the default 48 KB of dynamic shared
    // memory need the opt-in (10 KB stages of 8 + 2 heads never do), so the
    // common launch makes no attribute call, inside a graph capture or not.
    bool& done = g_dev.smem_set[dev & 63][from_shift ? 1 : 0];
    if (!done && smem > 48 * 1024) {
      // A capture may forbid the attribute call: that first launch takes the
      // register kernel instead.  The query itself fails on the legacy stream
      // while another stream captures in global mode; that launch takes the
      // register kernel too.
      cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
      if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) {
        cudaGetLastError();
        return cudaSuccess;
      }
      if (cap != cudaStreamCaptureStatusNone) return cudaSuccess;
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(1024 + kStages * (kMaxStageBytes + 16)));
      if (e != cudaSuccess) return e;
      done = true;
    }
  }
  e = pdl::launch(fn, dim3(static_cast<unsigned>(tiles)), dim3(kThreads), smem, stream,
                  programmatic, q_map, k_map, sa, table);
  if (e == cudaSuccess) {
    *launched = true;
    note_kernel("rotate_qk_staged_kernel");
  }
  return e;
}

}  // namespace cmr
