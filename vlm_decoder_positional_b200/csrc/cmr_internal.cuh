// Internal declarations shared by the kernels and the C-ABI layer of libcmr.
#pragma once

#include <cuda.h>  // CUtensorMap
#include <cuda_runtime.h>
#include <stdint.h>

#include "cmr.h"

namespace cmr {

// ---- canvas geometry of one 448x448 image (HF card "How the VLM rides the
// text-only engine": 64 merged rows on an 8x8 grid, framed by <image> and
// </image>, followed by the template's "\n") ----
constexpr int kGridSide = 8;
constexpr int kGridRows = kGridSide * kGridSide;   // 64
constexpr int kFrameTokens = kGridRows + 3;        // <image>, rows, </image>, "\n" = 67
constexpr int kCanvasSpan = kGridSide + 1;         // max(H, W) + 1 = 9
constexpr int32_t kTextOnlyStart = 1 << 30;

// ---- rotation limits ----
constexpr int kMaxFreqs = 128;  // rot_dim <= 256

// Per-frequency tables, passed by value as a kernel parameter (1.2 KB) and
// staged into shared memory by each CTA.
struct FreqTable {
  double inv_freq[kMaxFreqs];
  int32_t plane[kMaxFreqs];
};

struct RotateArgs {
  uint16_t* q;  // bf16 bits [L, N, hq, D]
  uint16_t* k;  // bf16 bits [L, N, hk, D]
  const int32_t* pos;  // [3, N], or nullptr when the planes come from the shift state
  // shift state (planes derived in the kernel): token t of prompt b sits at
  // absolute index pos_offset[b] + t - cu[b]; cu == nullptr: one token each
  const int32_t* cu;
  const int32_t* pos_offset;
  const int32_t* start;
  const int32_t* amount;
  int32_t num_seqs;
  int64_t n_tokens;
  int32_t num_layers;
  int32_t hq, hk, head_dim, rot_dim;
  int32_t* status;         // optional device status word (staged kernel time-outs)
  // with the shift state: also write each token's planes to pos_out [3, N]
  // (the one-call path, where the rotation replaces the planes kernel)
  int32_t* pos_out;
  int32_t units_per_head;  // rot_dim / 16: threads per token, 8 frequencies each
  int32_t job_groups;       // work items per token (set at launch)
  int32_t jobs_per_group;   // (layer, head) rows per work item
};

// Rotate Q in place and write rotated K and V rows into a KV cache
// [num_layers, cache_seqs, hk, cache_ctx, head_dim]; planes from the shift state.
struct CacheArgs {
  RotateArgs r;           // q, k (read only here), shift state, shape
  const uint16_t* v;      // bf16 bits [L, N, hk, D]
  uint16_t* k_cache;
  uint16_t* v_cache;
  const int32_t* cache_slot;  // [num_seqs] cache row of each sequence, or nullptr: b
  int32_t cache_seqs;
  int32_t cache_ctx;
  int32_t* status;        // optional device status word
  // work split (set at launch): Q rows and KV rows of a token form separate
  // items, each split into groups of (layer, head) rows
  int32_t q_groups, q_rows_per_group;
  int32_t kv_groups, kv_rows_per_group;
};

cudaError_t launch_rotate_qk_cache(const CacheArgs& args, const FreqTable& table,
                                   cudaStream_t stream);

// The TMA-staged rotate + KV-cache write (rot_dim 64, large batches): whether
// launch_rotate_qk_cache hands these shapes to it, and its launch (*launched
// false, nothing enqueued, when tensor maps cannot describe the buffers or the
// first launch falls inside a stream capture).
bool rotate_qk_cache_uses_staged(const RotateArgs& args);
cudaError_t launch_rotate_qk_cache_staged(const CacheArgs& args, const FreqTable& table,
                                          cudaStream_t stream, bool* launched);

// The origin kernel alone: each chunk's outgoing (start, amount), no planes.
cudaError_t launch_positions_origin(const int32_t* ids, const int32_t* cu_seqlens,
                                   int32_t num_seqs, int64_t n_tokens, int32_t image_token_id,
                                   int32_t rule, const int32_t* pos_offset,
                                   const int32_t* in_start, const int32_t* in_amount,
                                   int32_t* out_start, int32_t* out_amount,
                                   int32_t* device_status, cudaStream_t stream);

cudaError_t launch_positions(const int32_t* ids, const int32_t* cu_seqlens, int32_t num_seqs,
                             int64_t n_tokens, int32_t image_token_id, int32_t rule,
                             const int32_t* pos_offset, const int32_t* in_start,
                             const int32_t* in_amount, int32_t* out_pos, int32_t* out_start,
                             int32_t* out_amount, int32_t* device_status, cudaStream_t stream);

// Multi-frame canvas (frames.cu): slices per prompt for a workspace of
// `workspace_bytes` (0 when not even one summary per prompt fits), the bytes of
// one slice summary, and the launch of the summary and planes kernels.
int64_t frames_slices(int32_t num_seqs, int64_t n_tokens, size_t workspace_bytes);
size_t frames_summary_bytes();
cudaError_t launch_positions_frames(const int32_t* ids, const int32_t* cu_seqlens,
                                    int32_t num_seqs, int64_t n_tokens, int32_t image_token_id,
                                    int32_t grid_side, int32_t* out_pos, int32_t* out_start,
                                    int32_t* out_amount, void* workspace,
                                    size_t workspace_bytes, int32_t* device_status,
                                    cudaStream_t stream);

// The built-in scratch of cmr_positions_frames_noalloc: its device address on
// the current device (looked up on the first call per device) and size, and
// the most sequences it serves (one summary each).
cudaError_t frames_static_scratch(void** ptr, size_t* bytes);
int64_t frames_static_max_seqs();

cudaError_t launch_positions_step(const int32_t* cache_len, const int32_t* start,
                                  const int32_t* amount, int32_t num_seqs, int32_t* out_pos,
                                  cudaStream_t stream);

// programmatic: launch with programmatic stream serialization, which only a
// launch that directly follows this library's positions kernels may ask for:
// the staged kernel's Q/K loads start before the wait for pos.
cudaError_t launch_rotate_qk(const RotateArgs& args, const FreqTable& table, cudaStream_t stream,
                             bool programmatic = false);
// The register kernel alone (plain loads and stores, no tensor maps).
cudaError_t launch_rotate_qk_register(const RotateArgs& args, const FreqTable& table,
                                      cudaStream_t stream, bool programmatic = false);
// The row-coalesced kernel for Q/K in mapped host memory (rotate_rows.cu):
// shift-state planes only; rot_dim / 8 must divide 32.
bool rotate_rows_fits(const RotateArgs& args);
cudaError_t launch_rotate_qk_rows(const RotateArgs& args, const FreqTable& table,
                                  cudaStream_t stream, bool programmatic = false);

// TMA tensor map of a bf16 tensor: dims[0] is contiguous, strides_bytes[i] is
// the byte stride of dims[i + 1] (any order), box[i] the box extent per dim.
// False (and *map untouched) when the driver cannot encode it.
bool encode_bf16_tensor_map(CUtensorMap* map, void* base, int rank, const uint64_t* dims,
                            const uint64_t* strides_bytes, const uint32_t* box,
                            bool swizzle_128b);
// Records, per calling thread, the name of the rotate kernel a launch enqueued
// (read back through cmr_last_rotate_kernel).
void note_kernel(const char* name);

// L2 size of the current device in bytes (cached; 0 if it cannot be read).
int64_t device_l2_bytes();

// The TMA-staged rotate (rot_dim 64, one CTA per tile of tokens): whether it
// can take these shapes, its tile count, and its launch (*launched false,
// nothing enqueued, if the buffers cannot be described by tensor maps).
bool staged_rotate_fits(const RotateArgs& args);
// Whether launch_rotate_qk hands these shapes to the staged kernel.
bool rotate_qk_uses_staged(const RotateArgs& args);
int64_t staged_rotate_tiles(int64_t n_tokens);
cudaError_t launch_rotate_qk_staged(const RotateArgs& args, const FreqTable& table,
                                    cudaStream_t stream, bool programmatic, bool* launched);

}  // namespace cmr
