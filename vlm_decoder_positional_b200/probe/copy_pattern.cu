// Ceiling probe for the staged rotation: the same traffic as
// rotate_qk_staged_kernel -- the first 128 B of every 512-B head row of Q and
// K, every layer, HBM -> shared memory -> HBM in TMA boxes of 8 tokens x all
// heads through the same ring of stages -- with no cos/sin and no rotation:
// each box is stored back unchanged.  Its rate is what this access pattern
// can reach on the device, the ceiling the rotation is judged against beside
// the plain-copy peak.  It leaves Q and K bit for bit as they were.  With
// tiles_per_cta > 1 each CTA walks that many consecutive tiles through one
// ring, the staging the rotation measured and did not keep.
//
// A measurement aid, not part of the library: it is built into its own
// libcmr_probe.so and is called only by the benchmark.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../csrc/tma.cuh"

namespace {

constexpr int kRotDim = 64;
constexpr uint32_t kRowBytes = kRotDim * 2;
constexpr int kTileTokens = 8;
constexpr int kStages = 3;
constexpr int kThreads = 64;  // as the rotation: a consumer warp and a producer warp

struct ProbeArgs {
  int32_t num_layers, hq, hk;
  uint32_t q_box_bytes, stage_bytes;
  int32_t stages;
  int32_t tiles_per_cta;  // 1 as the rotation; more: a CTA walks consecutive tiles
  int64_t tiles;          // 8-token tiles in the batch
  int32_t* status;
};

__global__ void __launch_bounds__(kThreads)
    copy_pattern_kernel(const __grid_constant__ CUtensorMap q_map,
                        const __grid_constant__ CUtensorMap k_map, const ProbeArgs args) {
  extern __shared__ uint8_t dyn[];
  const uint32_t dyn_addr = cmr::tma::smem_addr(dyn);
  const uint32_t ring = (dyn_addr + 1023u) & ~1023u;
  const int S = args.stages;
  const uint32_t full0 = ring + S * args.stage_bytes;
  const uint32_t empty0 = full0 + 8 * S;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      cmr::tma::mbar_init(full0 + 8 * s, 1);
      cmr::tma::mbar_init(empty0 + 8 * s, 1);
    }
    cmr::tma::mbar_init_fence();
  }
  __syncthreads();
  const int L = args.num_layers;
  // item i = (tile first + i / L, layer i % L); one tile per CTA in the
  // rotation's own staging, several with tiles_per_cta > 1
  const int64_t first = static_cast<int64_t>(blockIdx.x) * args.tiles_per_cta;
  const int64_t my_tiles =
      args.tiles - first < args.tiles_per_cta ? args.tiles - first : args.tiles_per_cta;
  const int items = static_cast<int>(my_tiles) * L;
  if (threadIdx.x >= 32) {
    if (threadIdx.x != 32) return;
    int issued = 0, s = 0;
    uint32_t phase = 0;
    for (int i = 0; i < items; ++i) {
      const int l = i % L;
      const int t0 = static_cast<int>((first + i / L) * kTileTokens);
      if (!cmr::tma::mbar_wait(empty0 + 8 * s, phase ^ 1u)) {
        if (args.status) atomicOr(args.status, 4);
        break;
      }
      const uint32_t full = full0 + 8 * s;
      cmr::tma::mbar_arrive_expect_tx(full, args.stage_bytes);
      const uint32_t dst = ring + s * args.stage_bytes;
      if (args.hq > 0) cmr::tma::load_4d(dst, &q_map, full, 0, t0, 0, l);
      if (args.hk > 0) cmr::tma::load_4d(dst + args.q_box_bytes, &k_map, full, 0, t0, 0, l);
      ++issued;
      if (++s == S) {
        s = 0;
        phase ^= 1u;
      }
    }
    for (int l = issued > S ? issued - S : 0; l < issued; ++l)
      if (!cmr::tma::mbar_wait(full0 + 8 * (l % S), static_cast<uint32_t>(l / S) & 1u) &&
          args.status)
        atomicOr(args.status, 4);
    return;
  }
  int st = 0, prev = S - 1;
  uint32_t phase = 0;
  for (int i = 0; i < items; ++i) {
    const int l = i % L;
    const int t0 = static_cast<int>((first + i / L) * kTileTokens);
    const bool landed = cmr::tma::mbar_wait(full0 + 8 * st, phase);
    if (cmr::tma::named_any(1, 32, !landed)) {
      if (threadIdx.x == 0 && args.status) atomicOr(args.status, 4);
      break;
    }
    if (threadIdx.x == 0) {
      const uint32_t src = ring + st * args.stage_bytes;
      if (args.hq > 0) cmr::tma::store_4d(&q_map, src, 0, t0, 0, l);
      if (args.hk > 0) cmr::tma::store_4d(&k_map, src + args.q_box_bytes, 0, t0, 0, l);
      cmr::tma::bulk_commit();
      cmr::tma::bulk_wait_read<1>();
      if (i > 0) cmr::tma::mbar_arrive(empty0 + 8 * prev);
    }
    __syncwarp();
    prev = st;
    if (++st == S) {
      st = 0;
      phase ^= 1u;
    }
  }
  if (threadIdx.x == 0) cmr::tma::bulk_wait_read<0>();
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encoder() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

bool encode(CUtensorMap* map, void* base, int64_t n, int heads, int layers, int head_dim) {
  EncodeFn fn = encoder();
  if (fn == nullptr) return false;
  const uint64_t row = static_cast<uint64_t>(head_dim) * 2;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(n),
                              static_cast<cuuint64_t>(heads), static_cast<cuuint64_t>(layers)};
  const cuuint64_t strides[3] = {row * heads, row, row * heads * static_cast<uint64_t>(n)};
  const cuuint32_t box[4] = {kRotDim, kTileTokens, static_cast<cuuint32_t>(heads), 1};
  const cuuint32_t elem[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, elem,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace

// Copies the first 64 dims of every head row of q [L, N, hq, head_dim] and
// k [L, N, hk, head_dim] (bf16, device, 16-byte aligned) onto themselves
// through the staged path, each CTA walking tiles_per_cta consecutive 8-token
// tiles (1: the rotation's own staging; more: the form that overlaps one
// tile's loads with the previous tile's work inside a CTA, through a ring of
// min(3, tiles_per_cta x layers) stages).  Returns 0 when enqueued, 1 for
// arguments it does not take, 2 for a CUDA error.  status (optional, device
// int32) gets bit 4 if a bounded wait gave up.
extern "C" __attribute__((visibility("default"))) int cmr_probe_copy_pattern_tiles(
    void* q, void* k, int64_t n_tokens, int32_t num_layers, int32_t hq, int32_t hk,
    int32_t head_dim, int32_t tiles_per_cta, int32_t* status, cudaStream_t stream) {
  if (n_tokens <= 0 || num_layers <= 0 || hq < 0 || hk < 0 || hq + hk < 1 || head_dim < 64 ||
      head_dim % 8 != 0 || (hq > 0 && !q) || (hk > 0 && !k) || tiles_per_cta < 1 ||
      tiles_per_cta > 64 ||
      (reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k)) % 16 != 0)
    return 1;
  CUtensorMap q_map{}, k_map{};
  if (hq > 0 && !encode(&q_map, q, n_tokens, hq, num_layers, head_dim)) return 1;
  if (hk > 0 && !encode(&k_map, k, n_tokens, hk, num_layers, head_dim)) return 1;
  ProbeArgs a;
  a.num_layers = num_layers;
  a.hq = hq;
  a.hk = hk;
  a.q_box_bytes = kRowBytes * kTileTokens * hq;
  a.stage_bytes = a.q_box_bytes + kRowBytes * kTileTokens * hk;
  const int64_t items = static_cast<int64_t>(num_layers) * tiles_per_cta;
  a.stages = items < kStages ? static_cast<int32_t>(items) : kStages;
  a.tiles_per_cta = tiles_per_cta;
  a.tiles = (n_tokens + kTileTokens - 1) / kTileTokens;
  a.status = status;
  const size_t smem = 1024 + static_cast<size_t>(a.stages) * (a.stage_bytes + 16);
  if (smem > 48 * 1024) return 1;  // the probe serves the ring sizes of 8 + 2 heads
  const int64_t ctas = (a.tiles + tiles_per_cta - 1) / tiles_per_cta;
  copy_pattern_kernel<<<static_cast<unsigned>(ctas), kThreads, smem, stream>>>(q_map, k_map, a);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

// cmr_probe_copy_pattern_tiles with one tile per CTA: the rotation's staging.
extern "C" __attribute__((visibility("default"))) int cmr_probe_copy_pattern(
    void* q, void* k, int64_t n_tokens, int32_t num_layers, int32_t hq, int32_t hk,
    int32_t head_dim, int32_t* status, cudaStream_t stream) {
  return cmr_probe_copy_pattern_tiles(q, k, n_tokens, num_layers, hq, hk, head_dim, 1, status,
                                      stream);
}
