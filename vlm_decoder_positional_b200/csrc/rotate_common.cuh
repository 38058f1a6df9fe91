// Device helpers shared by the rotate kernels: cos/sin of one frequency,
// bf16 packing, the rotation of one 8-frequency unit, and the planes of one
// token (from pos [3, N] or from its prompt's shift state).
#pragma once

#include <cuda_bf16.h>

#include "canvas.cuh"

namespace cmr {
namespace rot {

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
// Sequence b of token t and the token's absolute index p in it:
// b is the last sequence with cu[b] <= t (cu[0] = 0 <= t < cu[num_seqs]);
// cu == nullptr means one token per sequence (b = t).
__device__ __forceinline__ void token_seq(const RotateArgs& a, int64_t t, int32_t& b,
                                          int64_t& p) {
  b = static_cast<int32_t>(t);
  int64_t local = 0;
  if (a.cu != nullptr) {
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
  p = (a.pos_offset ? __ldg(a.pos_offset + b) : 0) + local;
}

// The one-call path's rotation writes the planes of token t that it derived.
__device__ __forceinline__ void store_planes(const RotateArgs& a, int64_t t, int32_t p0,
                                             int32_t p1, int32_t p2) {
  a.pos_out[t] = p0;
  a.pos_out[a.n_tokens + t] = p1;
  a.pos_out[2 * a.n_tokens + t] = p2;
}

// Planes of the token at absolute index p of sequence b, from the sequence's
// shift state.  start / amount may come from the kernel just before (the
// one-call path's origin scan): read through L2, not the read-only path.
__device__ __forceinline__ void shift_planes(const RotateArgs& a, int32_t b, int64_t p,
                                             int32_t& p0, int32_t& p1, int32_t& p2) {
  const Planes r = canvas_row(p, __ldcg(a.start + b), __ldcg(a.amount + b));
  p0 = r.t;
  p1 = r.h;
  p2 = r.w;
}

template <bool kFromShift>
__device__ __forceinline__ void token_planes(const RotateArgs& a, int64_t t, int32_t& p0,
                                             int32_t& p1, int32_t& p2) {
  if constexpr (!kFromShift) {
    p0 = __ldg(a.pos + t);
    p1 = __ldg(a.pos + a.n_tokens + t);
    p2 = __ldg(a.pos + 2 * a.n_tokens + t);
  } else {
    int32_t b;
    int64_t p;
    token_seq(a, t, b, p);
    shift_planes(a, b, p, p0, p1, p2);
  }
}

}  // namespace rot
}  // namespace cmr
