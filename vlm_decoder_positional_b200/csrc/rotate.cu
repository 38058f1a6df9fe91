// Fused cos/sin + rotate-half M-RoPE of Q and K, in place, on sm_100a.
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
// stored back (two 16-byte stores each).  When a batch has too few tokens to
// fill the GPU (decode), each token's heads are split into groups handled by
// different threads, each computing the same 8 cos/sin for its group.
#include <cuda_bf16.h>

#include <mutex>

#include "canvas.cuh"

namespace cmr {
namespace {

constexpr int kThreads = 128;
constexpr int kMinBlocksPerSm = 4;
constexpr int kBatch = 4;  // head rows in flight per thread

// 2*pi split in two doubles (Cody & Waite's additive range reduction):
// kTwoPiHi is 2*pi rounded to double and kTwoPiLo the rounding remainder.
constexpr double kTwoPiHi = 6.283185307179586232e+00;
constexpr double kTwoPiLo = 2.449293598294706414e-16;
constexpr double kInvTwoPi = 1.591549430918953358e-01;
constexpr double kInvPi = 3.183098861837906715e-01;

// cos/sin of p * inv_freq: the product and its reduction to r in [-pi, pi] in
// fp64 (absolute error ~1e-16 for |p| < 2^31), then sincospif(r / pi) in fp32,
// whose own reduction of an argument in [-1, 1] is exact.
__device__ __forceinline__ void cos_sin(int32_t p, double inv_freq, float& c, float& s) {
  const double a = static_cast<double>(p) * inv_freq;
  const double n = rint(a * kInvTwoPi);
  double r = fma(-n, kTwoPiHi, a);
  r = fma(-n, kTwoPiLo, r);
  sincospif(static_cast<float>(r * kInvPi), &s, &c);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Rotate one unit: x1 holds dims [8u, 8u+8), x2 their partners [F+8u, F+8u+8).
__device__ __forceinline__ void rotate_unit(uint4& x1, uint4& x2, const float (&c)[8],
                                            const float (&s)[8]) {
  uint32_t* a = reinterpret_cast<uint32_t*>(&x1);
  uint32_t* b = reinterpret_cast<uint32_t*>(&x2);
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const float a0 = bf16_lo(a[m]), a1 = bf16_hi(a[m]);
    const float b0 = bf16_lo(b[m]), b1 = bf16_hi(b[m]);
    const float c0 = c[2 * m], s0 = s[2 * m], c1 = c[2 * m + 1], s1 = s[2 * m + 1];
    a[m] = pack_bf16x2(a0 * c0 - b0 * s0, a1 * c1 - b1 * s1);
    b[m] = pack_bf16x2(b0 * c0 + a0 * s0, b1 * c1 + a1 * s1);
  }
}

// Planes (T, H, W) of token t: read from pos [3, N], or derived from the
// shift state of the token's prompt (binary search of t in cu_seqlens).
template <bool kFromShift>
__device__ __forceinline__ void token_planes(const RotateArgs& a, int64_t t, int32_t& p0,
                                             int32_t& p1, int32_t& p2) {
  if constexpr (!kFromShift) {
    p0 = __ldg(a.pos + t);
    p1 = __ldg(a.pos + a.n_tokens + t);
    p2 = __ldg(a.pos + 2 * a.n_tokens + t);
  } else {
    int32_t b = static_cast<int32_t>(t);
    int64_t local = 0;
    if (a.cu != nullptr) {  // last b with cu[b] <= t; cu[0] = 0 <= t < cu[num_seqs]
      int32_t lo = 0, hi = a.num_seqs;
      while (hi - lo > 1) {
        const int32_t mid = (lo + hi) >> 1;
        if (__ldg(a.cu + mid) <= t)
          lo = mid;
        else
          hi = mid;
      }
      b = lo;
      local = t - __ldg(a.cu + b);
    }
    const int64_t p = (a.pos_offset ? __ldg(a.pos_offset + b) : 0) + local;
    const Planes r = canvas_row(p, __ldg(a.start + b), __ldg(a.amount + b));
    p0 = r.t;
    p1 = r.h;
    p2 = r.w;
  }
}

template <bool kFromShift>
__global__ void __launch_bounds__(kThreads, kMinBlocksPerSm)
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
  const int G = args.head_groups;
  const int hpg = args.heads_per_group;
  const int64_t D = args.head_dim;
  const int64_t q_tok = static_cast<int64_t>(args.hq) * D;  // elements per token
  const int64_t k_tok = static_cast<int64_t>(args.hk) * D;
  const int64_t q_layer = N * q_tok;
  const int64_t k_layer = N * k_tok;
  const int half4 = F / 8;  // partner offset in 16-byte vectors

  // Work item v = g * N + t: the head rows of head group g of token t, in
  // every layer.  With one group (large batches) an item is a whole token.
  const int64_t n_items = N * G;
  const int64_t v_step = static_cast<int64_t>(gridDim.x) * items_per_cta;
  int64_t v = static_cast<int64_t>(blockIdx.x) * items_per_cta + local;
  // Planes of the current item's token, loaded one item ahead so that their
  // latency overlaps the previous item's head rows.
  int32_t p0 = 0, p1 = 0, p2 = 0;
  if (v < n_items) token_planes<kFromShift>(args, G == 1 ? v : v % N, p0, p1, p2);
  for (; v < n_items; v += v_step) {
    const int64_t g = (G == 1) ? 0 : v / N;
    const int64_t t = v - g * N;
    const int h_lo = static_cast<int>(g) * hpg;
    const int h_hi = min(H, h_lo + hpg);
    const int J = (h_hi - h_lo) * args.num_layers;  // head rows of this item
    // Base of this thread's unit in head 0 of layer 0; K rows are indexed by
    // h - hq, folded into the base so that row h sits at base + h * D.
    uint16_t* const q_base = args.q + t * q_tok + 8 * u;
    uint16_t* const k_base = args.k + t * k_tok + 8 * u - static_cast<int64_t>(args.hq) * D;

    // First batch of head rows in flight before the cos/sin work below.
    int h = h_lo, l = 0;  // head row of the next job: head h of layer l
    uint4 x1[kBatch], x2[kBatch];
    uint4* ptr[kBatch];
    auto load_batch = [&](int j0) {
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        ptr[b] = nullptr;
        if (j0 + b < J) {
          uint16_t* row = (h < args.hq) ? q_base + l * q_layer : k_base + l * k_layer;
          ptr[b] = reinterpret_cast<uint4*>(row + h * D);
          x1[b] = __ldcs(ptr[b]);
          x2[b] = __ldcs(ptr[b] + half4);
          if (++h == h_hi) {
            h = h_lo;
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
      if (j0 >= J) break;
      load_batch(j0);
    }
  }
}

struct OccupancyCache {
  std::mutex mu;
  int device = -1;
  int ctas[2] = {0, 0};
};
OccupancyCache g_occ[64];

// CTAs of each variant resident on the whole device at full occupancy
// (cached per device).
cudaError_t resident_ctas(bool from_shift, int* total) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  OccupancyCache& c = g_occ[dev & 63];
  std::lock_guard<std::mutex> lock(c.mu);
  if (c.device != dev) {
    int sms = 0, per_sm[2] = {0, 0};
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm[0], rotate_qk_kernel<false>,
                                                      kThreads, 0);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm[1], rotate_qk_kernel<true>,
                                                      kThreads, 0);
    if (e != cudaSuccess) return e;
    c.device = dev;
    for (int i = 0; i < 2; ++i) c.ctas[i] = sms * (per_sm[i] > 0 ? per_sm[i] : 1);
  }
  *total = c.ctas[from_shift ? 1 : 0];
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_rotate_qk(const RotateArgs& in, const FreqTable& table, cudaStream_t stream) {
  RotateArgs a = in;
  const bool from_shift = a.pos == nullptr;
  int max_ctas = 0;
  cudaError_t e = resident_ctas(from_shift, &max_ctas);
  if (e != cudaSuccess) return e;
  const int64_t items_per_cta = kThreads / a.units_per_head;
  // Split each token's heads into groups only when there are too few tokens
  // to fill one wave of resident CTAs.
  const int heads = a.hq + a.hk;
  const int64_t wave_items = static_cast<int64_t>(max_ctas) * items_per_cta;
  int64_t groups = (wave_items + a.n_tokens - 1) / a.n_tokens;
  groups = groups < 1 ? 1 : (groups > heads ? heads : groups);
  a.heads_per_group = static_cast<int32_t>((heads + groups - 1) / groups);
  a.head_groups = (heads + a.heads_per_group - 1) / a.heads_per_group;
  const int64_t items = a.n_tokens * a.head_groups;
  const int64_t needed = (items + items_per_cta - 1) / items_per_cta;
  const int64_t ctas = needed < max_ctas ? needed : max_ctas;
  if (from_shift)
    rotate_qk_kernel<true><<<static_cast<unsigned>(ctas), kThreads, 0, stream>>>(a, table);
  else
    rotate_qk_kernel<false><<<static_cast<unsigned>(ctas), kThreads, 0, stream>>>(a, table);
  return cudaGetLastError();
}

}  // namespace cmr
