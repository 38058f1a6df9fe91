// Rotate Q in place and write the rotated K and the V rows of the same tokens
// into a KV cache, in one pass, on sm_100a, with the rows held in registers:
// the kernel for decode-sized batches and other shapes (larger rot_dim-64
// batches go to rotate_cache_staged.cu, which launch_rotate_qk_cache below
// picks; same bits).
//
// The cache is the engine's keyCache / valueCache of the HF card
// mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI ("How the VLM rides the text-only
// engine": [6, 1, 2, -1, 256], the 6 full-attention layers x batch x KV heads x
// positions x head_dim), here [num_layers, cache_seqs, hk, cache_ctx, head_dim]
// bf16.  Token t of sequence b sits at absolute index p = pos_offset[b] +
// t - cu[b]; its planes are the canvas rows at p under the sequence's
// (start, amount) state, exactly as in cmr_rotate_qk_shift, and its K / V rows
// land at [l, slot_b, h, p, :].  K and V themselves are only read.
//
// Thread map as in the rotate kernel: thread (item, u) owns the 8 frequencies
// [8u, 8u+8) of its token and computes their cos/sin once per item.  A token's
// Q rows and its KV rows are separate items: a Q item rotates its unit of
// every Q row in place; a KV item rotates its unit of every K row on the way
// to the cache and copies the untouched K dims and the whole V row in 16-byte
// chunks, chunk c going to thread c % U, so the U threads of a token move 16U
// contiguous bytes per instruction.  Small batches (decode) split a token's
// (layer, head) rows over several items.  Tokens whose index or slot falls outside the cache
// write no K/V (Q is still rotated) and set CMR_DEVICE_CACHE_RANGE.
#include <mutex>

#include "rotate_common.cuh"

namespace cmr {
namespace {

using namespace rot;

constexpr int kThreads = 128;
constexpr int kMinBlocksPerSm = 4;
constexpr int kQBatch = 4;   // Q head rows in flight per thread
constexpr int kCopyBatch = 4;  // copy chunks in flight per thread

__global__ void __launch_bounds__(kThreads, kMinBlocksPerSm)
    rotate_qk_cache_kernel(const CacheArgs ca, const FreqTable table) {
  const RotateArgs& a = ca.r;
  __shared__ double s_inv[kMaxFreqs];
  __shared__ int32_t s_plane[kMaxFreqs];
  const int F = a.rot_dim >> 1;
  for (int j = threadIdx.x; j < F; j += blockDim.x) {
    s_inv[j] = table.inv_freq[j];
    s_plane[j] = table.plane[j];
  }
  __syncthreads();  // the only barrier

  const int U = a.units_per_head;
  const int items_per_cta = kThreads / U;
  const int local = threadIdx.x / U;
  const int u = threadIdx.x - local * U;
  if (local >= items_per_cta) return;

  const int64_t N = a.n_tokens;
  const int L = a.num_layers;
  const int64_t D = a.head_dim;
  const int D8 = a.head_dim / 8;  // 16-byte chunks per head row
  const int R8 = a.rot_dim / 8;   // chunks holding rotated dims
  const int half4 = F / 8;
  const int64_t q_tok = static_cast<int64_t>(a.hq) * D;
  const int64_t kv_tok = static_cast<int64_t>(a.hk) * D;
  const int64_t q_layer = N * q_tok;
  const int64_t kv_layer = N * kv_tok;
  const int64_t cache_head = static_cast<int64_t>(ca.cache_ctx) * D;  // one KV head
  const int64_t cache_seq = a.hk * cache_head;
  const int64_t cache_layer = static_cast<int64_t>(ca.cache_seqs) * cache_seq;

  // Items [0, N * q_groups) rotate Q rows; the rest move KV rows.  Item
  // g * N + t of a kind covers that kind's rows [g * rpg, (g + 1) * rpg) of
  // token t, row j being head j % heads of layer j / heads.
  const int64_t n_q = N * ca.q_groups;
  const int64_t n_items = n_q + N * ca.kv_groups;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * items_per_cta + local; v < n_items;
       v += static_cast<int64_t>(gridDim.x) * items_per_cta) {
    const bool is_q = v < n_q;
    const int64_t w = is_q ? v : v - n_q;
    const int groups = is_q ? ca.q_groups : ca.kv_groups;
    const int rpg = is_q ? ca.q_rows_per_group : ca.kv_rows_per_group;
    const int heads = is_q ? a.hq : a.hk;
    const int64_t g = (groups == 1) ? 0 : w / N;
    const int64_t t = w - g * N;
    const int j_lo = static_cast<int>(g) * rpg;
    const int j_hi = min(heads * L, j_lo + rpg);

    int32_t b;
    int64_t p;
    token_seq(a, t, b, p);
    const Planes pl3 = canvas_row(p, __ldg(a.start + b), __ldg(a.amount + b));
    float c[8], s[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int j = 8 * u + e;
      const int pl = s_plane[j];
      cos_sin(pl == 0 ? pl3.t : (pl == 1 ? pl3.h : pl3.w), s_inv[j], c[e], s[e]);
    }

    if (is_q) {
      // Q rows, kQBatch at a time, rotated in place.
      int h = j_lo % a.hq, l = j_lo / a.hq;
      for (int j0 = j_lo; j0 < j_hi; j0 += kQBatch) {
        uint4 x1[kQBatch], x2[kQBatch];
        uint4* ptr[kQBatch];
#pragma unroll
        for (int i = 0; i < kQBatch; ++i) {
          ptr[i] = nullptr;
          if (j0 + i < j_hi) {
            ptr[i] = reinterpret_cast<uint4*>(a.q + l * q_layer + t * q_tok + h * D + 8 * u);
            x1[i] = __ldcs(ptr[i]);
            x2[i] = __ldcs(ptr[i] + half4);
            if (++h == a.hq) {
              h = 0;
              ++l;
            }
          }
        }
#pragma unroll
        for (int i = 0; i < kQBatch; ++i) {
          if (ptr[i] != nullptr) {
            rotate_unit(x1[i], x2[i], c, s);
            __stcs(ptr[i], x1[i]);
            __stcs(ptr[i] + half4, x2[i]);
          }
        }
      }
      continue;
    }

    // KV rows: the rotated K unit, the untouched K chunks and the V row go to
    // the cache row [l, slot, h, p, :].
    const int32_t slot = ca.cache_slot ? __ldg(ca.cache_slot + b) : b;
    const bool in_cache = p >= 0 && p < ca.cache_ctx && slot >= 0 && slot < ca.cache_seqs;
    if (!in_cache) {
      if (u == 0 && j_lo == 0 && ca.status != nullptr) atomicOr(ca.status, CMR_DEVICE_CACHE_RANGE);
      continue;
    }
    for (int j = j_lo; j < j_hi; ++j) {
      const int l = j / a.hk, kh = j - (j / a.hk) * a.hk;
      const int64_t src = l * kv_layer + t * kv_tok + kh * D;
      const int64_t dst = l * cache_layer + slot * cache_seq + kh * cache_head + p * D;
      const uint4* ksrc = reinterpret_cast<const uint4*>(a.k + src);
      const uint4* vsrc = reinterpret_cast<const uint4*>(ca.v + src);
      uint4* kdst = reinterpret_cast<uint4*>(ca.k_cache + dst);
      uint4* vdst = reinterpret_cast<uint4*>(ca.v_cache + dst);
      uint4 x1 = __ldcs(ksrc + u);
      uint4 x2 = __ldcs(ksrc + half4 + u);
      // chunk c of K (c >= R8) and of V goes to thread c % U
      for (int m0 = 0; u + m0 * U < D8; m0 += kCopyBatch) {
        uint4 kt[kCopyBatch], vt[kCopyBatch];
#pragma unroll
        for (int i = 0; i < kCopyBatch; ++i) {
          const int cv = u + (m0 + i) * U;
          const int ck = R8 + cv;
          if (ck < D8) kt[i] = __ldcs(ksrc + ck);
          if (cv < D8) vt[i] = __ldcs(vsrc + cv);
        }
#pragma unroll
        for (int i = 0; i < kCopyBatch; ++i) {
          const int cv = u + (m0 + i) * U;
          const int ck = R8 + cv;
          if (ck < D8) __stcs(kdst + ck, kt[i]);
          if (cv < D8) __stcs(vdst + cv, vt[i]);
        }
      }
      rotate_unit(x1, x2, c, s);
      __stcs(kdst + u, x1);
      __stcs(kdst + half4 + u, x2);
    }
  }
}

struct OccupancyCache {
  std::mutex mu;
  int device = -1;
  int ctas = 0;
};
OccupancyCache g_occ[64];

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
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rotate_qk_cache_kernel, kThreads, 0);
    if (e != cudaSuccess) return e;
    c.device = dev;
    c.ctas = sms * (per_sm > 0 ? per_sm : 1);
  }
  *total = c.ctas;
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_rotate_qk_cache(const CacheArgs& in, const FreqTable& table,
                                   cudaStream_t stream) {
  if (rotate_qk_cache_uses_staged(in.r)) {
    bool launched = false;
    const cudaError_t e = launch_rotate_qk_cache_staged(in, table, stream, &launched);
    if (e != cudaSuccess || launched) return e;
  }
  CacheArgs ca = in;
  RotateArgs& a = ca.r;
  int max_ctas = 0;
  cudaError_t e = resident_ctas(&max_ctas);
  if (e != cudaSuccess) return e;
  const int64_t items_per_cta = kThreads / a.units_per_head;
  // Split a token's rows over several items only when there are too few
  // tokens to fill one wave of resident CTAs.
  const int64_t wave_items = static_cast<int64_t>(max_ctas) * items_per_cta;
  const int64_t want = (wave_items + a.n_tokens - 1) / a.n_tokens;
  auto split = [&](int64_t rows, int32_t* groups, int32_t* per) {
    if (rows == 0) {
      *groups = 0;
      *per = 1;
      return;
    }
    int64_t g = want < 1 ? 1 : (want > rows ? rows : want);
    *per = static_cast<int32_t>((rows + g - 1) / g);
    *groups = static_cast<int32_t>((rows + *per - 1) / *per);
  };
  split(static_cast<int64_t>(a.hq) * a.num_layers, &ca.q_groups, &ca.q_rows_per_group);
  split(static_cast<int64_t>(a.hk) * a.num_layers, &ca.kv_groups, &ca.kv_rows_per_group);
  const int64_t items = a.n_tokens * (ca.q_groups + ca.kv_groups);
  const int64_t needed = (items + items_per_cta - 1) / items_per_cta;
  // One CTA per tile (a one-shot grid): measured on B200 it beats a
  // persistent grid at every layer count for this kernel (64 x 4096 tokens:
  // 5.98 vs 5.86 TB/s at 1 layer, 6.41 vs 5.94 TB/s at 6 layers), the
  // scheduler handing CTAs out as others finish keeps the addresses in flight
  // in one moving window.
  const int64_t ctas = needed;
  rotate_qk_cache_kernel<<<static_cast<unsigned>(ctas), kThreads, 0, stream>>>(ca, table);
  e = cudaGetLastError();
  if (e == cudaSuccess) note_kernel("rotate_qk_cache_kernel");
  return e;
}

}  // namespace cmr
