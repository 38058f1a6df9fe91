// Fused cos/sin + rotate-half M-RoPE of Q and K, in place, on sm_100a.
//
// Math (HF card mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI, "What it is": planes
// T, H, W with interleaved sections [11, 11, 10]; port notes: the decoder's
// `_mrope_freq_masks` and `forward_stateful_core(cos_sin=...)`): frequency j
// of F = rot_dim/2 reads the position of its plane, a = pos[plane_j][t] *
// theta^(-2j/rot_dim), and turns the pair (x_j, x_{j+F}) of every head.
//
// Memory: the op touches rot_dim of head_dim dims per head (128 B of every
// 512-B head row for this model) and is bound by HBM.  Each thread owns one
// "unit" = 8 consecutive dims of the first half plus their 8 partners of the
// second half of one head: two 16-byte loads and two 16-byte stores, the pair
// partner in the same thread, no shuffles.  Four consecutive lanes cover one
// head's 64 B + 64 B, so every warp access covers whole 32-B sectors.
//
// Per tile of tokens, a CTA first computes cos/sin for every (token,
// frequency) once -- fp64 angle and fp64 reduction modulo 2*pi, fp32 sincos --
// into shared memory, then applies it to every head of Q and K of every layer
// (num_layers layers share pos).  Up to kJobs (token, layer) jobs per thread
// are loaded before any is computed, which keeps 8 x 32 B in flight per
// thread.  The grid is persistent: one wave of CTAs at full occupancy on all
// SMs striding over tiles.
#include <cuda_bf16.h>

#include <mutex>

#include "cmr_internal.cuh"

namespace cmr {
namespace {

constexpr int kJobs = 8;          // (token, layer) jobs in flight per thread
constexpr int kMaxThreads = 512;  // CTA size bound (slots * units_per_token)

// 2*pi split in two doubles (Cody & Waite's additive range reduction):
// kTwoPiHi is 2*pi rounded to double and kTwoPiLo the rounding remainder.
constexpr double kTwoPiHi = 6.283185307179586232e+00;
constexpr double kTwoPiLo = 2.449293598294706414e-16;
constexpr double kInvTwoPi = 1.591549430918953358e-01;

// cos/sin of p * inv_freq: the product and its reduction to [-pi, pi] in
// fp64 (exact to ~1e-16 relative for |p| < 2^31), then fp32 sincos.
__device__ __forceinline__ float2 cos_sin(int32_t p, double inv_freq) {
  const double a = static_cast<double>(p) * inv_freq;
  const double n = rint(a * kInvTwoPi);
  double r = fma(-n, kTwoPiHi, a);
  r = fma(-n, kTwoPiLo, r);
  float s, c;
  sincosf(static_cast<float>(r), &s, &c);
  return make_float2(c, s);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Rotate one unit: x1 = dims [8u, 8u+8), x2 = their partners [F+8u, F+8u+8).
// cs points at the 8 (cos, sin) pairs of those frequencies in shared memory.
__device__ __forceinline__ void rotate_unit(uint4& x1, uint4& x2, const float2* __restrict__ cs) {
  const float4* c4 = reinterpret_cast<const float4*>(cs);
  uint32_t* a = reinterpret_cast<uint32_t*>(&x1);
  uint32_t* b = reinterpret_cast<uint32_t*>(&x2);
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const float4 t = c4[m];  // (cos, sin) of frequencies 2m and 2m+1 of the unit
    const float a0 = bf16_lo(a[m]), a1 = bf16_hi(a[m]);
    const float b0 = bf16_lo(b[m]), b1 = bf16_hi(b[m]);
    const float y0 = a0 * t.x - b0 * t.y;
    const float z0 = b0 * t.x + a0 * t.y;
    const float y1 = a1 * t.z - b1 * t.w;
    const float z1 = b1 * t.z + a1 * t.w;
    a[m] = pack_bf16x2(y0, y1);
    b[m] = pack_bf16x2(z0, z1);
  }
}

__global__ void __launch_bounds__(kMaxThreads)
    rotate_qk_kernel(const RotateArgs args, const FreqTable table) {
  extern __shared__ float4 s_dyn[];
  float2* s_cs = reinterpret_cast<float2*>(s_dyn);  // [slots * group][F]
  __shared__ double s_inv[kMaxFreqs];
  __shared__ int32_t s_plane[kMaxFreqs];

  const int F = args.rot_dim >> 1;
  for (int j = threadIdx.x; j < F; j += blockDim.x) {
    s_inv[j] = table.inv_freq[j];
    s_plane[j] = table.plane[j];
  }

  // Fixed role of this thread inside its token slot.
  const int W = args.units_per_token;
  const int U = args.units_per_head;
  const int slot = threadIdx.x / W;
  const int w = threadIdx.x - slot * W;
  const int head = w / U;
  const int unit = w - head * U;
  const bool active = slot < args.slots;
  const bool is_q = head < args.hq;
  uint16_t* const base = is_q ? args.q : args.k;
  const int64_t heads_here = is_q ? args.hq : args.hk;
  const int64_t head_idx = is_q ? head : head - args.hq;
  const int64_t tok_stride = heads_here * args.head_dim;
  const int64_t layer_stride = args.n_tokens * tok_stride;
  const int64_t unit_off = head_idx * args.head_dim + unit * 8;

  const int L = args.num_layers;
  const int G = args.group;
  const int tile_tokens = args.slots * G;
  const int jobs = G * L;
  const int64_t n_tiles = (args.n_tokens + tile_tokens - 1) / tile_tokens;
  __syncthreads();

  for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const int64_t t0 = tile * tile_tokens;

    // Phase 1: cos/sin of every (token, frequency) in the tile.
    for (int idx = threadIdx.x; idx < tile_tokens * F; idx += blockDim.x) {
      const int lt = idx / F;
      const int j = idx - lt * F;
      const int64_t t = t0 + lt;
      float2 v = make_float2(1.f, 0.f);
      if (t < args.n_tokens) v = cos_sin(__ldg(args.pos + s_plane[j] * args.n_tokens + t), s_inv[j]);
      s_cs[idx] = v;
    }
    __syncthreads();

    // Phase 2: every head of Q and K, every layer, of the slot's G tokens.
    if (active) {
      const int64_t slot_t0 = t0 + static_cast<int64_t>(slot) * G;
      for (int jb = 0; jb < jobs; jb += kJobs) {
        uint4 x1[kJobs], x2[kJobs];
        int gi[kJobs];
        bool ok[kJobs];
        int g = jb / L, l = jb - (jb / L) * L;
#pragma unroll
        for (int x = 0; x < kJobs; ++x) {
          gi[x] = g;
          ok[x] = (jb + x < jobs) && (slot_t0 + g < args.n_tokens);
          if (ok[x]) {
            const uint4* p = reinterpret_cast<const uint4*>(
                base + l * layer_stride + (slot_t0 + g) * tok_stride + unit_off);
            x1[x] = __ldcs(p);
            x2[x] = __ldcs(reinterpret_cast<const uint4*>(
                reinterpret_cast<const uint16_t*>(p) + F));
          }
          if (++l == L) {
            l = 0;
            ++g;
          }
        }
        g = jb / L;
        l = jb - g * L;
#pragma unroll
        for (int x = 0; x < kJobs; ++x) {
          if (ok[x]) {
            const float2* cs = s_cs + (slot * G + gi[x]) * F + unit * 8;
            rotate_unit(x1[x], x2[x], cs);
            uint4* p = reinterpret_cast<uint4*>(base + l * layer_stride +
                                                (slot_t0 + g) * tok_stride + unit_off);
            __stcs(p, x1[x]);
            __stcs(reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p) + F), x2[x]);
          }
          if (++l == L) {
            l = 0;
            ++g;
          }
        }
      }
    }
    __syncthreads();  // s_cs is rewritten by the next tile
  }
}

struct OccupancyCache {
  std::mutex mu;
  int device = -1;
  int sms = 0;
  int threads = 0;
  size_t smem = 0;
  int blocks_per_sm = 0;
};
OccupancyCache g_occ[64];

cudaError_t resident_ctas(int threads, size_t smem, int* total) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  OccupancyCache& c = g_occ[dev & 63];
  std::lock_guard<std::mutex> lock(c.mu);
  if (c.device != dev || c.threads != threads || c.smem != smem) {
    int sms = 0, per_sm = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rotate_qk_kernel, threads, smem);
    if (e != cudaSuccess) return e;
    c.device = dev;
    c.sms = sms;
    c.threads = threads;
    c.smem = smem;
    c.blocks_per_sm = per_sm > 0 ? per_sm : 1;
  }
  *total = c.sms * c.blocks_per_sm;
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_rotate_qk(const RotateArgs& in, const FreqTable& table, cudaStream_t stream) {
  RotateArgs a = in;
  const int W = a.units_per_token;
  // Token slots per CTA: as many whole tokens as fit in 320 threads (8 for
  // 8 Q + 2 K heads at rot_dim 64), at least one.
  int slots = 320 / W;
  if (slots < 1) slots = 1;
  if (slots > 32) slots = 32;
  a.slots = slots;
  // Tokens per slot per tile: enough (token, layer) jobs to fill kJobs.
  int group = kJobs / (a.num_layers > 0 ? a.num_layers : 1);
  a.group = group < 1 ? 1 : group;
  const int threads = ((slots * W + 31) / 32) * 32;
  const size_t smem = sizeof(float2) * static_cast<size_t>(slots) * a.group * (a.rot_dim / 2);
  int max_ctas = 0;
  cudaError_t e = resident_ctas(threads, smem, &max_ctas);
  if (e != cudaSuccess) return e;
  const int64_t tile_tokens = static_cast<int64_t>(slots) * a.group;
  const int64_t n_tiles = (a.n_tokens + tile_tokens - 1) / tile_tokens;
  const int64_t ctas = n_tiles < max_ctas ? n_tiles : max_ctas;
  rotate_qk_kernel<<<static_cast<unsigned>(ctas), threads, smem, stream>>>(a, table);
  return cudaGetLastError();
}

}  // namespace cmr
