// Fused cos/sin + rotate-half M-RoPE of Q and K, in place, on sm_100a, with
// the rows held in registers: the kernel for decode-sized batches and for
// rot_dim other than 64 (larger rot_dim-64 batches go to the TMA-staged kernel
// of rotate_staged.cu, which launch_rotate_qk below picks; same bits).
// The planes come from pos [3, N] (cmr_rotate_qk) or are derived in the kernel
// from each prompt's (start, amount) state (cmr_rotate_qk_shift).
//
// Math (HF card mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI, "What it is": planes
// T, H, W with interleaved sections [11, 11, 10]; port notes: the decoder's
// `_mrope_freq_masks` and `forward_stateful_core(cos_sin=...)`): frequency j
// of F = rot_dim/2 reads the position of its plane, a = pos[plane_j][t] *
// theta^(-2j/rot_dim), and turns the pair (x_j, x_{j+F}) of every head.
//
// The op touches rot_dim of head_dim dims per head (128 B of every 512-B head
// row for this model), reads and writes each byte once, and is bound by HBM;
// it is not a contraction, so there are no tensor cores here.
//
// Thread map: a token's rotated dims split into U = rot_dim/16 "units" of 8
// frequencies; thread (t, u) owns dims [8u, 8u+8) and their partners
// [F+8u, F+8u+8) of token t in every head of Q and K and every layer.  It
// computes the cos/sin of its 8 frequencies once (fp64 angle, fp64 reduction
// modulo 2*pi, fp32 sincos) and reuses them for all (hq + hk) * num_layers
// head rows, so each (token, frequency) pair is evaluated exactly once and no
// thread waits on another: there is no shared cos/sin table and no barrier
// in the loop.  Lanes 4t'..4t'+3 of a warp hold one token, so every warp access
// is 8 tokens x 64 contiguous bytes (whole 32-B sectors), and the x / partner
// loads of one head row together cover its 128-B line.  kBatch head rows are
// loaded (two 16-byte loads each, evict-first) before any is rotated and
// stored back (two 16-byte stores each); kBatch is 4, or 5 where that saves a
// load round.  Tiles of many rows get one CTA each (a one-shot grid); tiles
// of few rows are walked by a persistent grid (choose_plan has the numbers).
// When a batch has too few tokens to fill the GPU (decode), each token's
// (layer, head) rows are split into groups handled by different threads,
// each computing the same 8 cos/sin.
#include <mutex>

#include "pdl.cuh"
#include "rotate_common.cuh"

namespace cmr {
namespace {

using namespace rot;

constexpr int kThreads = 128;
constexpr int kOneShotRows = 16;  // rows per item from which a CTA serves one tile
// From this many 8-token tiles on, rot_dim 64 goes to the TMA-staged kernel
// (rotate_staged.cu); smaller batches (decode) keep this one, whose job groups
// spread a token's rows over several threads.
constexpr int64_t kMinStagedTiles = 1024;

// kBatch head rows are in flight per thread; the launch bounds keep the
// batch's registers within the occupancy each variant was tuned for.
template <int kBatch>
struct BatchShape;
template <>
struct BatchShape<4> {
  static constexpr int kMinBlocksPerSm = 4;
};
template <>
struct BatchShape<5> {
  static constexpr int kMinBlocksPerSm = 3;
};

template <bool kFromShift, int kBatch>
__global__ void __launch_bounds__(kThreads, BatchShape<kBatch>::kMinBlocksPerSm)
    rotate_qk_kernel(const RotateArgs args, const FreqTable table) {
  __shared__ double s_inv[kMaxFreqs];
  __shared__ int32_t s_plane[kMaxFreqs];
  const int F = args.rot_dim >> 1;
  for (int j = threadIdx.x; j < F; j += blockDim.x) {
    s_inv[j] = table.inv_freq[j];
    s_plane[j] = table.plane[j];
  }
  __syncthreads();  // the only barrier: the tables are read-only from here on

  const int U = args.units_per_head;
  const int items_per_cta = kThreads / U;
  const int local = threadIdx.x / U;
  const int u = threadIdx.x - local * U;
  if (local >= items_per_cta) return;  // spare threads when U does not divide kThreads

  const int64_t N = args.n_tokens;
  const int H = args.hq + args.hk;
  const int J = H * args.num_layers;  // (layer, head) rows per token
  const int G = args.job_groups;
  const int jpg = args.jobs_per_group;
  const int64_t D = args.head_dim;
  const int64_t q_tok = static_cast<int64_t>(args.hq) * D;  // elements per token
  const int64_t k_tok = static_cast<int64_t>(args.hk) * D;
  const int64_t q_layer = N * q_tok;
  const int64_t k_layer = N * k_tok;
  const int half4 = F / 8;  // partner offset in 16-byte vectors

  // Work item v = g * N + t: rows [g * jpg, (g + 1) * jpg) of token t, row
  // j being head j % H of layer j / H.  With one group (large batches) an
  // item is a whole token.
  const int64_t n_items = N * G;
  const int64_t v_step = static_cast<int64_t>(gridDim.x) * items_per_cta;
  int64_t v = static_cast<int64_t>(blockIdx.x) * items_per_cta + local;
  // Planes of the current item's token, loaded one item ahead so that their
  // latency overlaps the previous item's head rows.
  int32_t p0 = 0, p1 = 0, p2 = 0;
  // The first token's sequence and index come from cu_seqlens (and
  // pos_offset), which the kernels this one may be launched behind never
  // write: that search runs before the wait below.
  int32_t seq = 0;
  int64_t idx = 0;
  if (kFromShift && v < n_items) token_seq(args, G == 1 ? v : v % N, seq, idx);
  // Launched programmatically behind the positions kernels, pos (or the
  // shift state) is only ready after this wait; otherwise it returns at once.
  pdl::wait();
  if (v < n_items) {
    if constexpr (kFromShift)
      shift_planes(args, seq, idx, p0, p1, p2);
    else
      token_planes<false>(args, G == 1 ? v : v % N, p0, p1, p2);
  }
  for (; v < n_items; v += v_step) {
    const int64_t g = (G == 1) ? 0 : v / N;
    const int64_t t = v - g * N;
    if (kFromShift && args.pos_out != nullptr && u == 0 && g == 0)
      store_planes(args, t, p0, p1, p2);
    const int j_lo = static_cast<int>(g) * jpg;
    const int rows = min(J, j_lo + jpg) - j_lo;
    // Base of this thread's unit in head 0 of layer 0; K rows are indexed by
    // h - hq, folded into the base so that row h sits at base + h * D.
    uint16_t* const q_base = args.q + t * q_tok + 8 * u;
    uint16_t* const k_base = args.k + t * k_tok + 8 * u - static_cast<int64_t>(args.hq) * D;

    // First batch of head rows in flight before the cos/sin work below.
    int h = j_lo % H, l = j_lo / H;  // the next row: head h of layer l
    uint4 x1[kBatch], x2[kBatch];
    uint4* ptr[kBatch];
    auto load_batch = [&](int j0) {
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        ptr[b] = nullptr;
        if (j0 + b < rows) {
          uint16_t* row = (h < args.hq) ? q_base + l * q_layer : k_base + l * k_layer;
          ptr[b] = reinterpret_cast<uint4*>(row + h * D);
          x1[b] = __ldcs(ptr[b]);
          x2[b] = __ldcs(ptr[b] + half4);
          if (++h == H) {
            h = 0;
            ++l;
          }
        }
      }
    };
    load_batch(0);

    // cos/sin of the unit's 8 frequencies at token t.
    float c[8], s[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int j = 8 * u + e;
      const int pl = s_plane[j];
      cos_sin(pl == 0 ? p0 : (pl == 1 ? p1 : p2), s_inv[j], c[e], s[e]);
    }
    const int64_t vn = v + v_step;
    if (vn < n_items) token_planes<kFromShift>(args, G == 1 ? vn : vn % N, p0, p1, p2);

    for (int j0 = 0;;) {
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        if (ptr[b] != nullptr) {
          rotate_unit(x1[b], x2[b], c, s);
          __stcs(ptr[b], x1[b]);
          __stcs(ptr[b] + half4, x2[b]);
        }
      }
      j0 += kBatch;
      if (j0 >= rows) break;
      load_batch(j0);
    }
  }
}

// The kernel variants: plane source x rows in flight per thread (4 or 5).
using KernelFn = void (*)(RotateArgs, FreqTable);
KernelFn variant(bool from_shift, int batch_index) {
  static const KernelFn table[2][2] = {
      {rotate_qk_kernel<false, 4>, rotate_qk_kernel<false, 5>},
      {rotate_qk_kernel<true, 4>, rotate_qk_kernel<true, 5>}};
  return table[from_shift ? 1 : 0][batch_index];
}

struct OccupancyCache {
  std::mutex mu;
  int device = -1;
  int ctas[2][2] = {};
};
OccupancyCache g_occ[64];

// CTAs of each variant resident on the whole device at full occupancy
// (cached per device).
cudaError_t resident_ctas(bool from_shift, int batch_index, int* total) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  OccupancyCache& c = g_occ[dev & 63];
  std::lock_guard<std::mutex> lock(c.mu);
  if (c.device != dev) {
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    for (int f = 0; f < 2; ++f)
      for (int bi = 0; bi < 2; ++bi) {
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, variant(f == 1, bi), kThreads, 0);
        if (e != cudaSuccess) return e;
        c.ctas[f][bi] = sms * (per_sm > 0 ? per_sm : 1);
      }
    c.device = dev;
  }
  *total = c.ctas[from_shift ? 1 : 0][batch_index];
  return cudaSuccess;
}

// Rows in flight per thread and grid shape for a given number of rows per
// work item.
struct Plan {
  int batch_index;  // 0: 4 rows in flight per thread, 1: 5 rows
  bool one_shot;    // one CTA per tile, else a persistent grid of resident CTAs
};
// Measured on B200 (64 x 4096 tokens, graph replay):
//  - from 16 rows per item (2+ layers of 8 + 2 heads) one CTA per tile beats a
//    persistent grid, 6.02-6.12 vs 5.85-5.92 TB/s: the scheduler hands CTAs out
//    as earlier ones finish and the addresses in flight stay in one window;
//  - where 5 rows per batch saves a load round (5, 9 or 10 rows: one layer of
//    8 + 2 heads takes 2 rounds instead of 3), 5 rows with one CTA per tile win,
//    5.82 vs 5.65 TB/s (4 rows, persistent) and 5.40 (4 rows, one-shot);
//  - otherwise a persistent grid, whose one-item-ahead plane prefetch hides the
//    planes' latency.
Plan choose_plan(int rows_per_item) {
  const bool fewer_rounds_with_5 = (rows_per_item + 4) / 5 < (rows_per_item + 3) / 4;
  if (rows_per_item <= 10 && fewer_rounds_with_5) return {1, true};
  return {0, rows_per_item >= kOneShotRows};
}

}  // namespace

bool rotate_qk_uses_staged(const RotateArgs& a) {
  return staged_rotate_tiles(a.n_tokens) >= kMinStagedTiles && staged_rotate_fits(a);
}

cudaError_t launch_rotate_qk(const RotateArgs& in, const FreqTable& table, cudaStream_t stream,
                             bool programmatic) {
  if (rotate_qk_uses_staged(in)) {
    bool launched = false;
    const cudaError_t e = launch_rotate_qk_staged(in, table, stream, programmatic, &launched);
    if (e != cudaSuccess || launched) return e;
  }
  return launch_rotate_qk_register(in, table, stream, programmatic);
}

cudaError_t launch_rotate_qk_register(const RotateArgs& in, const FreqTable& table,
                                      cudaStream_t stream, bool programmatic) {
  RotateArgs a = in;
  const bool from_shift = a.pos == nullptr;
  const int64_t items_per_cta = kThreads / a.units_per_head;
  // Split each token's (layer, head) rows into groups only when there are too
  // few tokens to fill one wave of resident CTAs (sized with the default
  // variant).
  int wave_ctas = 0;
  cudaError_t e = resident_ctas(from_shift, 0, &wave_ctas);
  if (e != cudaSuccess) return e;
  const int64_t rows = static_cast<int64_t>(a.hq + a.hk) * a.num_layers;
  const int64_t wave_items = static_cast<int64_t>(wave_ctas) * items_per_cta;
  int64_t groups = (wave_items + a.n_tokens - 1) / a.n_tokens;
  groups = groups < 1 ? 1 : (groups > rows ? rows : groups);
  a.jobs_per_group = static_cast<int32_t>((rows + groups - 1) / groups);
  a.job_groups = static_cast<int32_t>((rows + a.jobs_per_group - 1) / a.jobs_per_group);
  const Plan plan = choose_plan(a.jobs_per_group);
  int max_ctas = 0;
  e = resident_ctas(from_shift, plan.batch_index, &max_ctas);
  if (e != cudaSuccess) return e;
  const int64_t items = a.n_tokens * a.job_groups;
  const int64_t needed = (items + items_per_cta - 1) / items_per_cta;
  const int64_t ctas = (plan.one_shot || needed <= max_ctas) ? needed : max_ctas;
  e = pdl::launch(variant(from_shift, plan.batch_index), dim3(static_cast<unsigned>(ctas)),
                  dim3(kThreads), 0, stream, programmatic, a, table);
  if (e == cudaSuccess) note_kernel("rotate_qk_kernel");
  return e;
}

}  // namespace cmr
