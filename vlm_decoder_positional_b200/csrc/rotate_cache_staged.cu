// Staged form of the rotate + KV-cache write (rot_dim 64).  Same result, bit
// for bit, as rotate_qk_cache_kernel (rotate_cache.cu): Q rotated in place;
// each token's K rows, rotated, and its V rows written to the cache rows
// [l, slot, h, p, :] of its sequence (the engine's keyCache / valueCache of the
// HF card mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI, "How the VLM rides the
// text-only engine"); planes derived from each sequence's (start, amount) as
// in cmr_rotate_qk_shift.
//
// One CTA per tile of kTileTokens tokens; per layer one ring stage holds
//   - the Q box {64, T, hq, 1} of the Q map {d, t, h, l} (the rotated 128 B of
//     each Q head row, 128-B swizzled, as in rotate_staged.cu),
//   - the K box {head_dim, hk, T, 1} of the K map {d, h, t, l}: whole K rows,
//     token-major ([t][h][d]), so that one token's rows are contiguous,
//   - the V box, likewise.
// A producer thread loads the three boxes per layer; one consumer warp (4
// lanes per token) rotates the Q rows and the first 64 dims of the K rows in
// shared memory; then one thread stores the Q box back and, per token whose
// cache index and slot are in range, its K rows and its V rows as one box each
// of the cache map {d, p, h, slot, l}.  Tokens outside the cache store no K/V
// and set CMR_DEVICE_CACHE_RANGE; tokens past the batch are never stored.
// Waits are bounded as in rotate_staged.cu (CMR_DEVICE_WAIT_TIMEOUT).
#include <mutex>

#include "rotate_common.cuh"
#include "tma.cuh"

namespace cmr {
namespace {

using namespace rot;

constexpr int kRotDim = 64;
constexpr uint32_t kQRowBytes = kRotDim * 2;      // 128 B: one swizzle span
constexpr int kTileTokens = 8;
constexpr int kStages = 3;
constexpr int kConsumers = kTileTokens * (kRotDim / 16);  // 32
constexpr int kThreads = kConsumers + 32;
constexpr uint32_t kMaxStageBytes = 32 * 1024;
constexpr int64_t kMinTiles = 1024;             // as the staged rotate
constexpr int64_t kEvictFirstL2Multiple = 4;    // as the staged rotate

struct CacheStagedArgs {
  CacheArgs c;
  uint32_t q_box_bytes;     // 128 * T * hq
  uint32_t kv_box_bytes;    // 2 * head_dim * hk * T (K or V)
  uint32_t token_kv_bytes;  // 2 * head_dim * hk: one token's K (or V) rows
  uint32_t stage_bytes;     // q_box_bytes + 2 * kv_box_bytes
  int32_t stages;           // min(kStages, num_layers)
  int32_t evict_first;
};

__device__ __forceinline__ void report(int32_t* status, int32_t bit) {
  if (status != nullptr) atomicOr(status, bit);
}

__global__ void __launch_bounds__(kThreads)
    rotate_qk_cache_staged_kernel(const __grid_constant__ CUtensorMap q_map,
                                  const __grid_constant__ CUtensorMap k_map,
                                  const __grid_constant__ CUtensorMap v_map,
                                  const __grid_constant__ CUtensorMap kc_map,
                                  const __grid_constant__ CUtensorMap vc_map,
                                  const CacheStagedArgs args, const FreqTable table) {
  __shared__ double s_inv[kRotDim / 2];
  __shared__ int32_t s_plane[kRotDim / 2];
  __shared__ int32_t s_p[kTileTokens], s_slot[kTileTokens], s_ok[kTileTokens];
  extern __shared__ uint8_t dyn[];
  const uint32_t dyn_addr = tma::smem_addr(dyn);
  const uint32_t ring = (dyn_addr + 1023u) & ~1023u;
  uint8_t* const ring_ptr = dyn + (ring - dyn_addr);
  const int S = args.stages;
  const uint32_t full0 = ring + S * args.stage_bytes;
  const uint32_t empty0 = full0 + 8 * S;

  for (int j = threadIdx.x; j < kRotDim / 2; j += blockDim.x) {
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

  const RotateArgs& a = args.c.r;
  int32_t* const status = args.c.status;
  const int L = a.num_layers;
  const int hq = a.hq, hk = a.hk;
  const int t0 = static_cast<int>(blockIdx.x) * kTileTokens;
  const uint32_t k_off = args.q_box_bytes;                      // K box within a stage
  const uint32_t v_off = args.q_box_bytes + args.kv_box_bytes;  // V box within a stage

  if (threadIdx.x >= kConsumers) {
    if (threadIdx.x != kConsumers) return;
    // ---- producer: layer l goes to stage l % S ----
    int issued = 0, s = 0;
    uint32_t phase = 0;
    for (int l = 0; l < L; ++l) {
      if (!tma::mbar_wait(empty0 + 8 * s, phase ^ 1u)) {
        report(status, CMR_DEVICE_WAIT_TIMEOUT);
        break;
      }
      const uint32_t full = full0 + 8 * s;
      tma::mbar_arrive_expect_tx(full, args.stage_bytes);
      const uint32_t dst = ring + s * args.stage_bytes;
      if (args.evict_first) {
        const uint64_t pol = tma::l2_evict_first_policy();
        if (hq > 0) tma::load_4d_hint(dst, &q_map, full, 0, t0, 0, l, pol);
        tma::load_4d_hint(dst + k_off, &k_map, full, 0, 0, t0, l, pol);
        tma::load_4d_hint(dst + v_off, &v_map, full, 0, 0, t0, l, pol);
      } else {
        if (hq > 0) tma::load_4d(dst, &q_map, full, 0, t0, 0, l);
        tma::load_4d(dst + k_off, &k_map, full, 0, 0, t0, l);
        tma::load_4d(dst + v_off, &v_map, full, 0, 0, t0, l);
      }
      ++issued;
      if (++s == S) {
        s = 0;
        phase ^= 1u;
      }
    }
    for (int l = issued > S ? issued - S : 0; l < issued; ++l)
      if (!tma::mbar_wait(full0 + 8 * (l % S), static_cast<uint32_t>(l / S) & 1u))
        report(status, CMR_DEVICE_WAIT_TIMEOUT);
    return;
  }

  // ---- consumers: thread (token tl, unit u), lanes as in rotate_staged.cu ----
  const int lane = threadIdx.x & 31;
  const int u = lane & 3;
  const int tl = (threadIdx.x >> 5) * 8 + ((lane >> 3) | (((lane >> 2) & 1) << 2));
  const int64_t t = static_cast<int64_t>(t0) + tl;
  int32_t p0 = 0, p1 = 0, p2 = 0;
  int32_t p_cache = 0, slot = 0, ok = 0;
  if (t < a.n_tokens) {
    int32_t b;
    int64_t p;
    token_seq(a, t, b, p);
    const Planes r = canvas_row(p, __ldg(a.start + b), __ldg(a.amount + b));
    p0 = r.t;
    p1 = r.h;
    p2 = r.w;
    slot = args.c.cache_slot ? __ldg(args.c.cache_slot + b) : b;
    ok = p >= 0 && p < args.c.cache_ctx && slot >= 0 && slot < args.c.cache_seqs;
    p_cache = static_cast<int32_t>(ok ? p : 0);
    if (!ok && u == 0) report(status, CMR_DEVICE_CACHE_RANGE);
  }
  if (u == 0) {
    s_p[tl] = p_cache;
    s_slot[tl] = slot;
    s_ok[tl] = ok;
  }
  float c[8], s[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int j = 8 * u + e;
    const int pl = s_plane[j];
    cos_sin(pl == 0 ? p0 : (pl == 1 ? p1 : p2), s_inv[j], c[e], s[e]);
  }
  // Q rows: 16-B chunk c of row r at chunk position c ^ (r & 7), r & 7 = tl & 7.
  const uint32_t sw = static_cast<uint32_t>(tl & 7);
  const uint32_t q_x = (static_cast<uint32_t>(u) ^ sw) * 16u;
  const uint32_t q_y = (static_cast<uint32_t>(u + 4) ^ sw) * 16u;
  // K rows (not swizzled): this token's hk rows of head_dim * 2 bytes.
  const uint32_t row_bytes = static_cast<uint32_t>(a.head_dim) * 2u;
  const uint32_t k_x = 16u * u, k_y = 16u * (u + 4);

  int st = 0, prev = S - 1;
  uint32_t phase = 0;
  for (int l = 0; l < L; ++l) {
    const bool landed = tma::mbar_wait(full0 + 8 * st, phase, tma::kConsumerWaitLimitNs);
    if (tma::named_any(1, kConsumers, !landed)) {
      if (threadIdx.x == 0) report(status, CMR_DEVICE_WAIT_TIMEOUT);
      break;
    }
    uint8_t* const stage = ring_ptr + st * args.stage_bytes;
    uint8_t* row = stage + static_cast<uint32_t>(tl) * kQRowBytes;
#pragma unroll 2
    for (int h = 0; h < hq; ++h, row += kTileTokens * kQRowBytes) {
      uint4* const px = reinterpret_cast<uint4*>(row + q_x);
      uint4* const py = reinterpret_cast<uint4*>(row + q_y);
      uint4 x1 = *px, x2 = *py;
      rotate_unit(x1, x2, c, s);
      *px = x1;
      *py = x2;
    }
    row = stage + k_off + static_cast<uint32_t>(tl) * args.token_kv_bytes;
    for (int h = 0; h < hk; ++h, row += row_bytes) {
      uint4* const px = reinterpret_cast<uint4*>(row + k_x);
      uint4* const py = reinterpret_cast<uint4*>(row + k_y);
      uint4 x1 = *px, x2 = *py;
      rotate_unit(x1, x2, c, s);
      *px = x1;
      *py = x2;
    }
    tma::fence_async_shared();
    tma::named_sync(1, kConsumers);
    if (threadIdx.x == 0) {
      const uint32_t src = ring + st * args.stage_bytes;
      const uint64_t pol = tma::l2_evict_first_policy();
      if (hq > 0) {
        if (args.evict_first)
          tma::store_4d_hint(&q_map, src, 0, t0, 0, l, pol);
        else
          tma::store_4d(&q_map, src, 0, t0, 0, l);
      }
      for (int k = 0; k < kTileTokens; ++k) {
        if (!s_ok[k]) continue;
        const uint32_t off = static_cast<uint32_t>(k) * args.token_kv_bytes;
        if (args.evict_first) {
          tma::store_5d_hint(&kc_map, src + k_off + off, 0, s_p[k], 0, s_slot[k], l, pol);
          tma::store_5d_hint(&vc_map, src + v_off + off, 0, s_p[k], 0, s_slot[k], l, pol);
        } else {
          tma::store_5d(&kc_map, src + k_off + off, 0, s_p[k], 0, s_slot[k], l);
          tma::store_5d(&vc_map, src + v_off + off, 0, s_p[k], 0, s_slot[k], l);
        }
      }
      tma::bulk_commit();
      tma::bulk_wait_read<1>();  // the previous layer's stores have read their stage
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

using CacheStagedFn = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap,
                               CacheStagedArgs, FreqTable);

std::mutex g_mu;
bool g_smem_set[64] = {};

}  // namespace

bool rotate_qk_cache_uses_staged(const RotateArgs& a) {
  if (a.rot_dim != kRotDim || a.hk < 1 || a.hk > 256 || a.hq > 256 || a.head_dim > 256) return false;
  if ((static_cast<int64_t>(a.hk) * a.head_dim) % 64 != 0) return false;  // 128-B token rows
  if (a.n_tokens > INT32_MAX) return false;
  const uint64_t stage = static_cast<uint64_t>(kQRowBytes) * kTileTokens * a.hq +
                         2ull * 2 * a.head_dim * a.hk * kTileTokens;
  if (stage > kMaxStageBytes) return false;
  return (a.n_tokens + kTileTokens - 1) / kTileTokens >= kMinTiles;
}

cudaError_t launch_rotate_qk_cache_staged(const CacheArgs& ca, const FreqTable& table,
                                          cudaStream_t stream, bool* launched) {
  *launched = false;
  const RotateArgs& a = ca.r;
  const uint64_t D = static_cast<uint64_t>(a.head_dim), row = D * 2;
  const uint64_t N = static_cast<uint64_t>(a.n_tokens), hq = a.hq, hk = a.hk;
  const uint64_t L = static_cast<uint64_t>(a.num_layers);
  CUtensorMap q_map{}, k_map{}, v_map{}, kc_map{}, vc_map{};
  if (hq > 0) {
    const uint64_t dims[4] = {D, N, hq, L};
    const uint64_t strides[3] = {row * hq, row, row * hq * N};
    const uint32_t box[4] = {kRotDim, kTileTokens, static_cast<uint32_t>(hq), 1};
    if (!encode_bf16_tensor_map(&q_map, a.q, 4, dims, strides, box, true)) return cudaSuccess;
  }
  {
    const uint64_t dims[4] = {D, hk, N, L};
    const uint64_t strides[3] = {row, row * hk, row * hk * N};
    const uint32_t box[4] = {static_cast<uint32_t>(D), static_cast<uint32_t>(hk), kTileTokens, 1};
    if (!encode_bf16_tensor_map(&k_map, a.k, 4, dims, strides, box, false)) return cudaSuccess;
    if (!encode_bf16_tensor_map(&v_map, const_cast<uint16_t*>(ca.v), 4, dims, strides, box, false))
      return cudaSuccess;
  }
  {
    const uint64_t ctx = static_cast<uint64_t>(ca.cache_ctx);
    const uint64_t seqs = static_cast<uint64_t>(ca.cache_seqs);
    const uint64_t dims[5] = {D, ctx, hk, seqs, L};
    const uint64_t strides[4] = {row, row * ctx, row * ctx * hk, row * ctx * hk * seqs};
    const uint32_t box[5] = {static_cast<uint32_t>(D), 1, static_cast<uint32_t>(hk), 1, 1};
    if (!encode_bf16_tensor_map(&kc_map, ca.k_cache, 5, dims, strides, box, false)) return cudaSuccess;
    if (!encode_bf16_tensor_map(&vc_map, ca.v_cache, 5, dims, strides, box, false)) return cudaSuccess;
  }
  CacheStagedArgs sa;
  sa.c = ca;
  sa.q_box_bytes = kQRowBytes * kTileTokens * static_cast<uint32_t>(hq);
  sa.token_kv_bytes = static_cast<uint32_t>(row * hk);
  sa.kv_box_bytes = sa.token_kv_bytes * kTileTokens;
  sa.stage_bytes = sa.q_box_bytes + 2 * sa.kv_box_bytes;
  sa.stages = a.num_layers < kStages ? a.num_layers : kStages;
  const size_t smem = 1024 + static_cast<size_t>(sa.stages) * (sa.stage_bytes + 16);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (smem > 48 * 1024) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_smem_set[dev & 63]) {
      // The opt-in is an attribute call, which a stream capture may forbid:
      // a first launch inside a capture takes the register kernel instead.
      // The query itself fails on the legacy stream while another stream
      // captures in global mode; that launch takes the register kernel too.
      cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
      if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) {
        cudaGetLastError();
        return cudaSuccess;
      }
      if (cap != cudaStreamCaptureStatusNone) return cudaSuccess;
      e = cudaFuncSetAttribute(rotate_qk_cache_staged_kernel,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(1024 + kStages * (kMaxStageBytes + 16)));
      if (e != cudaSuccess) return e;
      g_smem_set[dev & 63] = true;
    }
  }
  // L2 policy as in the staged rotate: launches of up to 4 L2 sizes stream
  // through with evict-first loads and stores.
  const uint64_t moved = N * L * (2 * kQRowBytes * hq + 4 * row * hk);
  const int64_t l2 = device_l2_bytes();
  sa.evict_first = static_cast<int64_t>(moved) <= kEvictFirstL2Multiple * l2 ? 1 : 0;
  const int64_t ctas = (a.n_tokens + kTileTokens - 1) / kTileTokens;
  rotate_qk_cache_staged_kernel<<<static_cast<unsigned>(ctas), kThreads, smem, stream>>>(
      q_map, k_map, v_map, kc_map, vc_map, sa, table);
  e = cudaGetLastError();
  if (e == cudaSuccess) {
    *launched = true;
    note_kernel("rotate_qk_cache_staged_kernel");
  }
  return e;
}

}  // namespace cmr
