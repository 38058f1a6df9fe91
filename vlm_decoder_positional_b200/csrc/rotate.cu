// Fused cos/sin + rotate-half M-RoPE of Q and K, in place, on sm_100a.
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
// stored back (two 16-byte stores each).
#include <cuda_bf16.h>

#include <mutex>

#include "cmr_internal.cuh"

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
  const int tokens_per_cta = kThreads / U;
  const int local = threadIdx.x / U;
  const int u = threadIdx.x - local * U;
  if (local >= tokens_per_cta) return;  // spare threads when U does not divide kThreads

  const int64_t N = args.n_tokens;
  const int H = args.hq + args.hk;
  const int J = H * args.num_layers;  // head rows per token
  const int64_t D = args.head_dim;
  const int64_t q_tok = static_cast<int64_t>(args.hq) * D;  // elements per token
  const int64_t k_tok = static_cast<int64_t>(args.hk) * D;
  const int64_t q_layer = N * q_tok;
  const int64_t k_layer = N * k_tok;
  const int half4 = F / 8;  // partner offset in 16-byte vectors

  const int64_t t_step = static_cast<int64_t>(gridDim.x) * tokens_per_cta;
  int64_t t = static_cast<int64_t>(blockIdx.x) * tokens_per_cta + local;
  // Planes of the current token, loaded one token ahead so that their latency
  // overlaps the previous token's head rows.
  int32_t p0 = 0, p1 = 0, p2 = 0;
  if (t < N) {
    p0 = __ldg(args.pos + t);
    p1 = __ldg(args.pos + N + t);
    p2 = __ldg(args.pos + 2 * N + t);
  }
  for (; t < N; t += t_step) {
    // Base of this thread's unit in head 0 of layer 0; K rows are indexed by
    // h - hq, folded into the base so that row h sits at base + h * D.
    uint16_t* const q_base = args.q + t * q_tok + 8 * u;
    uint16_t* const k_base = args.k + t * k_tok + 8 * u - static_cast<int64_t>(args.hq) * D;

    // First batch of head rows in flight before the cos/sin work below.
    int h = 0, l = 0;  // head row of the next job: head h of layer l
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
    const int64_t tn = t + t_step;
    if (tn < N) {
      p0 = __ldg(args.pos + tn);
      p1 = __ldg(args.pos + N + tn);
      p2 = __ldg(args.pos + 2 * N + tn);
    }

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
  int ctas = 0;
};
OccupancyCache g_occ[64];

// CTAs resident on the whole device at full occupancy (cached per device).
cudaError_t resident_ctas(int* total) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  OccupancyCache& c = g_occ[dev & 63];
  std::lock_guard<std::mutex> lock(c.mu);
  if (c.device != dev) {
    int sms = 0, per_sm = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rotate_qk_kernel, kThreads, 0);
    if (e != cudaSuccess) return e;
    c.device = dev;
    c.ctas = sms * (per_sm > 0 ? per_sm : 1);
  }
  *total = c.ctas;
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_rotate_qk(const RotateArgs& a, const FreqTable& table, cudaStream_t stream) {
  int max_ctas = 0;
  cudaError_t e = resident_ctas(&max_ctas);
  if (e != cudaSuccess) return e;
  const int64_t tokens_per_cta = kThreads / a.units_per_head;
  const int64_t needed = (a.n_tokens + tokens_per_cta - 1) / tokens_per_cta;
  const int64_t ctas = needed < max_ctas ? needed : max_ctas;
  rotate_qk_kernel<<<static_cast<unsigned>(ctas), kThreads, 0, stream>>>(a, table);
  return cudaGetLastError();
}

}  // namespace cmr
