// Fused cos/sin + rotate-half M-RoPE of Q and K, in place, for Q/K held in
// mapped page-locked host memory (cmr_positions_rotate_qk_host), on sm_100a.
//
// Math: as rotate.cu (HF card mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI, "What it
// is": planes T, H, W with interleaved sections [11, 11, 10]): frequency j of
// F = rot_dim/2 reads the position of its plane, a = pos[plane_j][t] *
// theta^(-2j/rot_dim), and turns the pair (x_j, x_{j+F}) of every head.  The
// planes come from each prompt's (start, amount) state, as in the one-call
// path.
//
// Over PCIe the cost is the number and size of the bus transactions, so the
// thread map keeps every load and store instruction on whole rotated parts:
// R = rot_dim/8 consecutive lanes own one head row's rot_dim * 2 bytes, lane
// r holding the 16-byte chunk r (8 dims), so a warp instruction covers the
// rotated parts of 32/R tokens' rows, each contiguous (128 B for rot_dim 64).
// Chunk r < R/2 holds dims x_j of frequencies [8r, 8r + 8) and chunk r + R/2
// their partners x_{j+F}; the two lanes swap their chunks with one shuffle and
// each keeps its own half of the rotation.  Every lane computes the 8 cos/sin
// of its frequency group once per token (fp64 angle and reduction, fp32
// sincos, as the other kernels) and reuses them for all (hq + hk) *
// num_layers rows of the token; kRowBatch rows are loaded before any is
// rotated.  The rotation itself is rot::rotate_unit, the other kernels'
// arithmetic, so the results are the same bits.  Plain loads and stores
// only: no tensor maps over host memory.  rot_dim must make R divide 32 (16,
// 32, 64, 128 or 256).
#include "pdl.cuh"
#include "rotate_common.cuh"

namespace cmr {
namespace {

using namespace rot;

constexpr int kRowsThreads = 256;
constexpr int kRowBatch = 4;  // head rows in flight per lane

__device__ __forceinline__ uint4 shfl_xor4(const uint4& v, int mask) {
  return {__shfl_xor_sync(0xffffffffu, v.x, mask), __shfl_xor_sync(0xffffffffu, v.y, mask),
          __shfl_xor_sync(0xffffffffu, v.z, mask), __shfl_xor_sync(0xffffffffu, v.w, mask)};
}

__global__ void __launch_bounds__(kRowsThreads)
    rotate_qk_rows_kernel(const RotateArgs args, const FreqTable table) {
  __shared__ double s_inv[kMaxFreqs];
  __shared__ int32_t s_plane[kMaxFreqs];
  for (int j = threadIdx.x; j < args.rot_dim / 2; j += blockDim.x) {
    s_inv[j] = table.inv_freq[j];
    s_plane[j] = table.plane[j];
  }
  __syncthreads();  // the only barrier: the tables are read-only from here on
  const int lane = threadIdx.x & 31;
  const int R = args.rot_dim / 8;        // lanes per head row
  const int half = R / 2;                // chunks of x_j; the rest hold x_{j+F}
  const int tokens_per_warp = 32 / R;
  const int slot = lane / R;             // token of the warp's group
  const int chunk = lane - slot * R;     // 16-byte chunk of the row's rotated part
  const int group = chunk % half;        // frequencies [8 group, 8 group + 8)
  const bool first = chunk < half;

  const int64_t N = args.n_tokens;
  const int H = args.hq + args.hk;
  const int J = H * args.num_layers;
  const int64_t D = args.head_dim;
  const int64_t q_layer = N * args.hq * D, k_layer = N * args.hk * D;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (kRowsThreads / 32);
  const int64_t warp = static_cast<int64_t>(blockIdx.x) * (kRowsThreads / 32) + threadIdx.x / 32;
  // every lane of a warp runs the same iterations (the shuffles need them)
  for (int64_t t0 = warp * tokens_per_warp; t0 < N; t0 += warps * tokens_per_warp) {
    const int64_t t = t0 + slot;
    const bool live = t < N;
    int32_t seq = 0;
    int64_t idx = 0;
    if (live) token_seq(args, t, seq, idx);  // cu_seqlens is an input: before the wait
    pdl::wait();  // the origin scan's state is written
    int32_t p0 = 0, p1 = 0, p2 = 0;
    if (live) {
      shift_planes(args, seq, idx, p0, p1, p2);
      if (args.pos_out != nullptr && chunk == 0) store_planes(args, t, p0, p1, p2);
    }
    float c[8], s[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int j = 8 * group + e;
      const int pl = s_plane[j];
      cos_sin(pl == 0 ? p0 : (pl == 1 ? p1 : p2), s_inv[j], c[e], s[e]);
    }
    uint16_t* const q_base = args.q + t * args.hq * D + 8 * chunk;
    uint16_t* const k_base = args.k + t * args.hk * D + 8 * chunk - static_cast<int64_t>(args.hq) * D;
    int h = 0, l = 0;  // the next row: head h of layer l
    for (int j0 = 0; j0 < J; j0 += kRowBatch) {
      uint4 x[kRowBatch];
      uint4* ptr[kRowBatch];
#pragma unroll
      for (int b = 0; b < kRowBatch; ++b) {
        ptr[b] = nullptr;
        x[b] = make_uint4(0, 0, 0, 0);
        if (j0 + b < J) {
          uint16_t* row = (h < args.hq) ? q_base + l * q_layer : k_base + l * k_layer;
          if (live) {
            ptr[b] = reinterpret_cast<uint4*>(row + h * D);
            x[b] = *ptr[b];
          }
          if (++h == H) {
            h = 0;
            ++l;
          }
        }
      }
#pragma unroll
      for (int b = 0; b < kRowBatch; ++b) {
        uint4 other = shfl_xor4(x[b], half);
        uint4 x1 = first ? x[b] : other, x2 = first ? other : x[b];
        rotate_unit(x1, x2, c, s);
        if (ptr[b] != nullptr) *ptr[b] = first ? x1 : x2;
      }
    }
  }
}

}  // namespace

bool rotate_rows_fits(const RotateArgs& a) {
  const int R = a.rot_dim / 8;
  return R >= 2 && R <= 32 && 32 % R == 0;
}

cudaError_t launch_rotate_qk_rows(const RotateArgs& a, const FreqTable& table,
                                  cudaStream_t stream, bool programmatic) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int64_t tokens_per_cta = (kRowsThreads / 32) * (32 / (a.rot_dim / 8));
  int64_t ctas = (a.n_tokens + tokens_per_cta - 1) / tokens_per_cta;
  const int64_t cap = static_cast<int64_t>(sms) * 8;  // enough lanes in flight for PCIe
  if (ctas > cap) ctas = cap;
  if (ctas < 1) ctas = 1;
  e = pdl::launch(rotate_qk_rows_kernel, dim3(static_cast<unsigned>(ctas)), dim3(kRowsThreads),
                  0, stream, programmatic, a, table);
  if (e == cudaSuccess) note_kernel("rotate_qk_rows_kernel");
  return e;
}

}  // namespace cmr
