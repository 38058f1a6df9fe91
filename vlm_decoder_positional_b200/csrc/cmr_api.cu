// The C ABI of libcmr (declared in include/cmr.h): host-side argument checks,
// the per-frequency tables, and the kernel launches.  Nothing here allocates
// device memory or synchronises.
#include <cmath>
#include <cstdarg>
#include <climits>
#include <cstdint>
#include <cstdio>

#include "cmr.h"
#include "cmr_internal.cuh"

namespace {

thread_local char g_message[320] = "no error";
thread_local const char* g_last_kernel = nullptr;

cmr_status fail(cmr_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_message, sizeof g_message, fmt, ap);
  va_end(ap);
  return s;
}

cmr_status cuda_fail(cudaError_t e, const char* what) {
  return fail(CMR_ECUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// A pointer the current device can use in a kernel: device or managed memory
// of the current device.  Pageable host memory would fault in a kernel, so it
// is refused here.
cmr_status check_device_ptr(const void* p, const char* name) {
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, p);
  if (e != cudaSuccess) {
    cudaGetLastError();  // clear the error this query may have set
    return fail(CMR_EINVAL, "%s: not a CUDA pointer (%s)", name, cudaGetErrorName(e));
  }
  if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
    return fail(CMR_EINVAL, "%s: not device memory (memory type %d)", name,
                static_cast<int>(attr.type));
  int dev = -1;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (attr.type == cudaMemoryTypeDevice && attr.device != dev)
    return fail(CMR_EINVAL, "%s: lives on device %d but device %d is current", name,
                attr.device, dev);
  return CMR_OK;
}

// Page-locked host memory mapped into the device's address space at the same
// address (cudaHostAlloc'd or cudaHostRegister'd memory on a system with
// unified addressing): a kernel reads and writes it directly over PCIe.
cmr_status check_mapped_host_ptr(const void* p, const char* name) {
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(CMR_EINVAL, "%s: not a CUDA pointer (%s)", name, cudaGetErrorName(e));
  }
  if (attr.type != cudaMemoryTypeHost)
    return fail(CMR_EINVAL, "%s: not page-locked host memory (memory type %d)", name,
                static_cast<int>(attr.type));
  if (attr.devicePointer != p)
    return fail(CMR_EINVAL, "%s: page-locked host memory not mapped at the same address", name);
  return CMR_OK;
}

// Where an entry point's buffers live.
enum class Where { kDevice, kMappedHost };

cmr_status check_ptr(const void* p, const char* name, Where where) {
  return where == Where::kDevice ? check_device_ptr(p, name) : check_mapped_host_ptr(p, name);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool ranges_overlap(const void* a, const void* b, size_t bytes) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + bytes && y < x + bytes;
}

// Checks shared by both rotate entry points; fills the frequency table and the
// shape fields of `a`.  Returns CMR_OK with a.n_tokens == 0 when there is
// nothing to do.
cmr_status check_rotate(void* q, void* k, int64_t n_tokens, int32_t num_layers, int32_t hq,
                        int32_t hk, int32_t head_dim, double theta, const int32_t sections[3],
                        int32_t rot_dim, cmr::RotateArgs* a, cmr::FreqTable* table,
                        Where where = Where::kDevice) {
  if (n_tokens < 0 || num_layers < 0) return fail(CMR_EINVAL, "negative n_tokens or num_layers");
  if (hq < 0 || hk < 0 || hq + hk < 1) return fail(CMR_EINVAL, "need hq, hk >= 0, hq + hk >= 1");
  if (head_dim <= 0 || head_dim % 8 != 0) return fail(CMR_EINVAL, "head_dim must be a positive multiple of 8");
  if (rot_dim < 16 || rot_dim % 16 != 0 || rot_dim > head_dim || rot_dim > 2 * cmr::kMaxFreqs)
    return fail(CMR_EINVAL, "rot_dim must be a multiple of 16 in [16, min(head_dim, 256)]");
  if (!(theta > 0.0) || !std::isfinite(theta)) return fail(CMR_EINVAL, "theta must be finite and > 0");
  if (!sections) return fail(CMR_EINVAL, "sections is required");

  // Frequency -> plane: H takes j = 1, 4, 7, ... (sections[1] of them), W takes
  // j = 2, 5, 8, ... (sections[2]), T keeps the rest and must count sections[0].
  const int F = rot_dim / 2;
  for (int j = 0; j < cmr::kMaxFreqs; ++j) {
    table->plane[j] = 0;
    table->inv_freq[j] = 0.0;
  }
  if (sections[0] < 0 || sections[1] < 0 || sections[2] < 0 ||
      static_cast<int64_t>(sections[0]) + sections[1] + sections[2] != F)
    return fail(CMR_EINVAL, "sections must be >= 0 and sum to rot_dim / 2");
  for (int plane = 1; plane <= 2; ++plane)
    for (int m = 0; m < sections[plane]; ++m) {
      const int j = 3 * m + plane;
      if (j >= F) return fail(CMR_EINVAL, "sections[%d] = %d does not fit the interleave", plane, sections[plane]);
      table->plane[j] = plane;
    }
  for (int j = 0; j < F; ++j) table->inv_freq[j] = std::pow(theta, -2.0 * j / rot_dim);

  const int64_t rows = (static_cast<int64_t>(hq) + hk) * num_layers;  // head rows per token
  if (rows > INT32_MAX)
    return fail(CMR_EUNSUPPORTED, "(hq + hk) * num_layers = %lld exceeds INT32_MAX",
                static_cast<long long>(rows));
  *a = cmr::RotateArgs{};
  a->n_tokens = (num_layers == 0) ? 0 : n_tokens;
  if (a->n_tokens == 0) return CMR_OK;
  if (hq > 0 && !q) return fail(CMR_EINVAL, "q is required when hq > 0");
  if (hk > 0 && !k) return fail(CMR_EINVAL, "k is required when hk > 0");
  if ((hq > 0 && !aligned16(q)) || (hk > 0 && !aligned16(k)))
    return fail(CMR_EINVAL, "q and k must be 16-byte aligned");
  cmr_status s;
  if (hq > 0 && (s = check_ptr(q, "q", where)) != CMR_OK) return s;
  if (hk > 0 && (s = check_ptr(k, "k", where)) != CMR_OK) return s;
  a->q = static_cast<uint16_t*>(q);
  a->k = static_cast<uint16_t*>(k);
  a->num_layers = num_layers;
  a->hq = hq;
  a->hk = hk;
  a->head_dim = head_dim;
  a->rot_dim = rot_dim;
  a->units_per_head = rot_dim / 16;
  return CMR_OK;
}

// Checks of cmr_positions' arguments (num_seqs == 0 with no tokens is valid
// and leaves nothing to do).
cmr_status check_positions(const int32_t* ids, const int32_t* cu_seqlens, int32_t num_seqs,
                           int64_t n_tokens, const int32_t* out_pos, const int32_t* out_start,
                           const int32_t* out_amount, const int32_t* device_status,
                           Where where = Where::kDevice) {
  if (num_seqs < 0 || n_tokens < 0) return fail(CMR_EINVAL, "negative num_seqs or n_tokens");
  if (n_tokens > INT32_MAX) return fail(CMR_EINVAL, "n_tokens exceeds int32 indexing");
  if (num_seqs == 0) {
    if (n_tokens != 0) return fail(CMR_EINVAL, "num_seqs == 0 with n_tokens > 0");
    return CMR_OK;
  }
  if (!cu_seqlens || !out_start || !out_amount)
    return fail(CMR_EINVAL, "cu_seqlens, out_start and out_amount are required");
  if (n_tokens > 0 && (!ids || !out_pos)) return fail(CMR_EINVAL, "ids and out_pos are required");
  cmr_status s;
  if ((s = check_ptr(cu_seqlens, "cu_seqlens", where)) != CMR_OK) return s;
  if ((s = check_ptr(out_start, "out_start", where)) != CMR_OK) return s;
  if ((s = check_ptr(out_amount, "out_amount", where)) != CMR_OK) return s;
  if (n_tokens > 0) {
    if ((s = check_ptr(ids, "ids", where)) != CMR_OK) return s;
    if ((s = check_ptr(out_pos, "out_pos", where)) != CMR_OK) return s;
  }
  // the status word may be device memory or mapped host memory
  if (device_status && check_device_ptr(device_status, "device_status") != CMR_OK &&
      (s = check_mapped_host_ptr(device_status, "device_status")) != CMR_OK)
    return s;
  return CMR_OK;
}

}  // namespace

namespace cmr {
void note_kernel(const char* name) { g_last_kernel = name; }
}  // namespace cmr

extern "C" {

const char* cmr_status_string(cmr_status s) {
  switch (s) {
    case CMR_OK: return "CMR_OK";
    case CMR_EINVAL: return "CMR_EINVAL: invalid argument";
    case CMR_ECUDA: return "CMR_ECUDA: CUDA runtime error";
    case CMR_EUNSUPPORTED: return "CMR_EUNSUPPORTED: shape outside this build's limits";
  }
  return "unknown cmr_status";
}

const char* cmr_last_error_message(void) { return g_message; }

const char* cmr_last_rotate_kernel(void) { return g_last_kernel ? g_last_kernel : ""; }

int32_t cmr_version(void) { return 20200; }  // 2.2.0

cmr_status cmr_positions(const int32_t* ids, const int32_t* cu_seqlens, int32_t num_seqs,
                         int64_t n_tokens, int32_t image_token_id, int32_t* out_pos,
                         int32_t* out_start, int32_t* out_amount, int32_t* device_status,
                         cmr_stream_t stream) {
  cmr_status s = check_positions(ids, cu_seqlens, num_seqs, n_tokens, out_pos, out_start,
                                 out_amount, device_status);
  if (s != CMR_OK || num_seqs == 0) return s;
  cudaError_t e = cmr::launch_positions(ids, cu_seqlens, num_seqs, n_tokens, image_token_id,
                                        CMR_RULE_CANVAS, nullptr, nullptr, nullptr, out_pos,
                                        out_start, out_amount, device_status,
                                        reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "positions launch");
  return CMR_OK;
}

cmr_status cmr_positions_chunk(const int32_t* ids, const int32_t* cu_seqlens, int32_t num_seqs,
                               int64_t n_tokens, int32_t image_token_id, int32_t rule,
                               const int32_t* pos_offset, const int32_t* in_start,
                               const int32_t* in_amount, int32_t* out_pos, int32_t* out_start,
                               int32_t* out_amount, int32_t* device_status, cmr_stream_t stream) {
  if (rule != CMR_RULE_CANVAS && rule != CMR_RULE_QWEN_VL && rule != CMR_RULE_PLANES_1D)
    return fail(CMR_EINVAL, "unknown rule %d", rule);
  if (num_seqs < 0 || n_tokens < 0) return fail(CMR_EINVAL, "negative num_seqs or n_tokens");
  if (n_tokens > INT32_MAX) return fail(CMR_EINVAL, "n_tokens exceeds int32 indexing");
  if (num_seqs == 0) {
    if (n_tokens != 0) return fail(CMR_EINVAL, "num_seqs == 0 with n_tokens > 0");
    return CMR_OK;
  }
  if (!cu_seqlens || !out_start || !out_amount)
    return fail(CMR_EINVAL, "cu_seqlens, out_start and out_amount are required");
  if (n_tokens > 0 && (!ids || !out_pos)) return fail(CMR_EINVAL, "ids and out_pos are required");
  // Every CTA of a chunk reads the incoming state while slice 0 writes the
  // outgoing one, so the two must not share memory.
  const size_t bytes = static_cast<size_t>(num_seqs) * sizeof(int32_t);
  for (const int32_t* in : {in_start, in_amount})
    for (const int32_t* out : {out_start, out_amount})
      if (in && ranges_overlap(in, out, bytes))
        return fail(CMR_EINVAL, "incoming and outgoing state must not overlap");
  cmr_status s;
  if ((s = check_device_ptr(cu_seqlens, "cu_seqlens")) != CMR_OK) return s;
  if ((s = check_device_ptr(out_start, "out_start")) != CMR_OK) return s;
  if ((s = check_device_ptr(out_amount, "out_amount")) != CMR_OK) return s;
  if (n_tokens > 0) {
    if ((s = check_device_ptr(ids, "ids")) != CMR_OK) return s;
    if ((s = check_device_ptr(out_pos, "out_pos")) != CMR_OK) return s;
  }
  if (pos_offset && (s = check_device_ptr(pos_offset, "pos_offset")) != CMR_OK) return s;
  if (in_start && (s = check_device_ptr(in_start, "in_start")) != CMR_OK) return s;
  if (in_amount && (s = check_device_ptr(in_amount, "in_amount")) != CMR_OK) return s;
  if (device_status && (s = check_device_ptr(device_status, "device_status")) != CMR_OK) return s;
  cudaError_t e = cmr::launch_positions(ids, cu_seqlens, num_seqs, n_tokens, image_token_id, rule,
                                        pos_offset, in_start, in_amount, out_pos, out_start,
                                        out_amount, device_status,
                                        reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "positions_chunk launch");
  return CMR_OK;
}

size_t cmr_positions_frames_workspace_bytes(int32_t num_seqs, int64_t n_tokens) {
  if (num_seqs <= 0 || n_tokens < 0) return 0;
  return static_cast<size_t>(cmr::frames_slices(num_seqs, n_tokens, SIZE_MAX)) *
         cmr::frames_summary_bytes() * static_cast<size_t>(num_seqs);
}

cmr_status cmr_positions_frames(const int32_t* ids, const int32_t* cu_seqlens, int32_t num_seqs,
                                int64_t n_tokens, int32_t image_token_id, int32_t grid_side,
                                int32_t* out_pos, int32_t* out_start, int32_t* out_amount,
                                void* workspace, size_t workspace_bytes,
                                int32_t* device_status, cmr_stream_t stream) {
  if (grid_side < 1 || grid_side > 128) return fail(CMR_EINVAL, "grid_side must be in 1 .. 128");
  cmr_status s = check_positions(ids, cu_seqlens, num_seqs, n_tokens, out_pos, out_start,
                                 out_amount, device_status);
  if (s != CMR_OK || num_seqs == 0) return s;
  const size_t one = cmr::frames_summary_bytes() * static_cast<size_t>(num_seqs);
  if (!workspace || workspace_bytes < one)
    return fail(CMR_EINVAL, "workspace must hold at least %zu bytes (16 per sequence)", one);
  if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0)
    return fail(CMR_EINVAL, "workspace must be 16-byte aligned");
  if ((s = check_device_ptr(workspace, "workspace")) != CMR_OK) return s;
  cudaError_t e = cmr::launch_positions_frames(ids, cu_seqlens, num_seqs, n_tokens,
                                               image_token_id, grid_side, out_pos, out_start,
                                               out_amount, workspace, workspace_bytes,
                                               device_status,
                                               reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "positions_frames launch");
  return CMR_OK;
}

cmr_status cmr_positions_frames_noalloc(const int32_t* ids, const int32_t* cu_seqlens,
                                        int32_t num_seqs, int64_t n_tokens,
                                        int32_t image_token_id, int32_t grid_side,
                                        int32_t* out_pos, int32_t* out_start,
                                        int32_t* out_amount, int32_t* device_status,
                                        cmr_stream_t stream) {
  if (grid_side < 1 || grid_side > 128) return fail(CMR_EINVAL, "grid_side must be in 1 .. 128");
  if (num_seqs > cmr::frames_static_max_seqs())
    return fail(CMR_EINVAL,
                "num_seqs = %d exceeds the %lld sequences the built-in scratch serves; "
                "use cmr_positions_frames with a workspace",
                num_seqs, static_cast<long long>(cmr::frames_static_max_seqs()));
  cmr_status s = check_positions(ids, cu_seqlens, num_seqs, n_tokens, out_pos, out_start,
                                 out_amount, device_status);
  if (s != CMR_OK || num_seqs == 0) return s;
  void* scratch = nullptr;
  size_t scratch_bytes = 0;
  cudaError_t e = cmr::frames_static_scratch(&scratch, &scratch_bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the built-in scratch");
  e = cmr::launch_positions_frames(ids, cu_seqlens, num_seqs, n_tokens, image_token_id,
                                   grid_side, out_pos, out_start, out_amount, scratch,
                                   scratch_bytes, device_status,
                                   reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "positions_frames_noalloc launch");
  return CMR_OK;
}

cmr_status cmr_positions_step(const int32_t* cache_len, const int32_t* start,
                              const int32_t* amount, int32_t num_seqs, int32_t* out_pos,
                              cmr_stream_t stream) {
  if (num_seqs < 0) return fail(CMR_EINVAL, "negative num_seqs");
  if (num_seqs == 0) return CMR_OK;
  if (!cache_len || !start || !amount || !out_pos)
    return fail(CMR_EINVAL, "cache_len, start, amount and out_pos are required");
  cmr_status s;
  if ((s = check_device_ptr(cache_len, "cache_len")) != CMR_OK) return s;
  if ((s = check_device_ptr(start, "start")) != CMR_OK) return s;
  if ((s = check_device_ptr(amount, "amount")) != CMR_OK) return s;
  if ((s = check_device_ptr(out_pos, "out_pos")) != CMR_OK) return s;
  cudaError_t e = cmr::launch_positions_step(cache_len, start, amount, num_seqs, out_pos,
                                             reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "positions_step launch");
  return CMR_OK;
}

cmr_status cmr_rotate_qk(void* q, void* k, const int32_t* pos, int64_t n_tokens,
                         int32_t num_layers, int32_t hq, int32_t hk, int32_t head_dim,
                         double theta, const int32_t sections[3], int32_t rot_dim,
                         int32_t* device_status, cmr_stream_t stream) {
  cmr::RotateArgs a;
  cmr::FreqTable table;
  cmr_status s = check_rotate(q, k, n_tokens, num_layers, hq, hk, head_dim, theta, sections,
                              rot_dim, &a, &table);
  if (s != CMR_OK || a.n_tokens == 0) return s;
  if (!pos) return fail(CMR_EINVAL, "pos is required");
  if ((s = check_device_ptr(pos, "pos")) != CMR_OK) return s;
  if (device_status && (s = check_device_ptr(device_status, "device_status")) != CMR_OK) return s;
  a.pos = pos;
  a.status = device_status;
  cudaError_t e = cmr::launch_rotate_qk(a, table, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "rotate_qk launch");
  return CMR_OK;
}

cmr_status cmr_positions_rotate_qk(const int32_t* ids, const int32_t* cu_seqlens,
                                   int32_t num_seqs, int64_t n_tokens, int32_t image_token_id,
                                   int32_t* out_pos, int32_t* out_start, int32_t* out_amount,
                                   void* q, void* k, int32_t num_layers, int32_t hq, int32_t hk,
                                   int32_t head_dim, double theta, const int32_t sections[3],
                                   int32_t rot_dim, int32_t* device_status,
                                   cmr_stream_t stream) {
  // Every check of both steps runs before anything is enqueued.
  cmr::RotateArgs a;
  cmr::FreqTable table;
  cmr_status s = check_positions(ids, cu_seqlens, num_seqs, n_tokens, out_pos, out_start,
                                 out_amount, device_status);
  if (s != CMR_OK) return s;
  s = check_rotate(q, k, n_tokens, num_layers, hq, hk, head_dim, theta, sections, rot_dim, &a,
                   &table);
  if (s != CMR_OK) return s;
  if (num_seqs == 0) return CMR_OK;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (a.n_tokens == 0) {  // no rotation (no layers): the planes kernel writes pos
    cudaError_t e = cmr::launch_positions(ids, cu_seqlens, num_seqs, n_tokens, image_token_id,
                                          CMR_RULE_CANVAS, nullptr, nullptr, nullptr, out_pos,
                                          out_start, out_amount, device_status, st);
    return e == cudaSuccess ? CMR_OK : cuda_fail(e, "positions launch");
  }
  // The origin scan writes each prompt's (start, amount); the rotation,
  // launched to start while the scan runs (its Q/K loads do not depend on it),
  // derives each token's planes from that state, writes them to out_pos and
  // rotates -- the planes kernel is not needed.
  cudaError_t e = cmr::launch_positions_origin(ids, cu_seqlens, num_seqs, n_tokens,
                                               image_token_id, CMR_RULE_CANVAS, nullptr, nullptr,
                                               nullptr, out_start, out_amount, device_status, st);
  if (e != cudaSuccess) return cuda_fail(e, "positions launch");
  a.pos = nullptr;
  a.cu = cu_seqlens;
  a.num_seqs = num_seqs;
  a.pos_offset = nullptr;
  a.start = out_start;
  a.amount = out_amount;
  a.pos_out = out_pos;
  a.status = device_status;
  e = cmr::launch_rotate_qk(a, table, st, /*programmatic=*/true);
  if (e != cudaSuccess) return cuda_fail(e, "rotate_qk launch");
  return CMR_OK;
}

cmr_status cmr_positions_rotate_qk_host(const int32_t* ids, const int32_t* cu_seqlens,
                                        int32_t num_seqs, int64_t n_tokens,
                                        int32_t image_token_id, int32_t* out_pos,
                                        int32_t* out_start, int32_t* out_amount, void* q, void* k,
                                        int32_t num_layers, int32_t hq, int32_t hk,
                                        int32_t head_dim, double theta,
                                        const int32_t sections[3], int32_t rot_dim,
                                        int32_t* device_status, cmr_stream_t stream) {
  // The checks of cmr_positions_rotate_qk, with every buffer in mapped host
  // memory (the status word may be either).
  cmr::RotateArgs a;
  cmr::FreqTable table;
  cmr_status s = check_positions(ids, cu_seqlens, num_seqs, n_tokens, out_pos, out_start,
                                 out_amount, device_status, Where::kMappedHost);
  if (s != CMR_OK) return s;
  s = check_rotate(q, k, n_tokens, num_layers, hq, hk, head_dim, theta, sections, rot_dim, &a,
                   &table, Where::kMappedHost);
  if (s != CMR_OK) return s;
  if (num_seqs == 0) return CMR_OK;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (a.n_tokens == 0) {  // no rotation: the planes kernel writes pos
    cudaError_t e = cmr::launch_positions(ids, cu_seqlens, num_seqs, n_tokens, image_token_id,
                                          CMR_RULE_CANVAS, nullptr, nullptr, nullptr, out_pos,
                                          out_start, out_amount, device_status, st);
    return e == cudaSuccess ? CMR_OK : cuda_fail(e, "positions launch");
  }
  // The origin scan reads the ids over PCIe and writes the state; the
  // row-coalesced kernel (whole rotated parts per instruction, plain loads
  // and stores: no tensor maps over host memory; the register kernel for
  // rot_dims it does not take) then derives, writes and uses each token's
  // planes, moving only the rotated dims of each head row across the bus.
  cudaError_t e = cmr::launch_positions_origin(ids, cu_seqlens, num_seqs, n_tokens,
                                               image_token_id, CMR_RULE_CANVAS, nullptr, nullptr,
                                               nullptr, out_start, out_amount, device_status, st);
  if (e != cudaSuccess) return cuda_fail(e, "positions launch");
  a.pos = nullptr;
  a.cu = cu_seqlens;
  a.num_seqs = num_seqs;
  a.pos_offset = nullptr;
  a.start = out_start;
  a.amount = out_amount;
  a.pos_out = out_pos;
  a.status = device_status;
  e = cmr::rotate_rows_fits(a) ? cmr::launch_rotate_qk_rows(a, table, st, /*programmatic=*/true)
                               : cmr::launch_rotate_qk_register(a, table, st,
                                                                /*programmatic=*/true);
  if (e != cudaSuccess) return cuda_fail(e, "rotate_qk launch");
  return CMR_OK;
}

cmr_status cmr_rotate_qk_shift(void* q, void* k, const int32_t* cu_seqlens, int32_t num_seqs,
                               const int32_t* pos_offset, const int32_t* start,
                               const int32_t* amount, int64_t n_tokens, int32_t num_layers,
                               int32_t hq, int32_t hk, int32_t head_dim, double theta,
                               const int32_t sections[3], int32_t rot_dim,
                               int32_t* device_status, cmr_stream_t stream) {
  cmr::RotateArgs a;
  cmr::FreqTable table;
  cmr_status s = check_rotate(q, k, n_tokens, num_layers, hq, hk, head_dim, theta, sections,
                              rot_dim, &a, &table);
  if (s != CMR_OK || a.n_tokens == 0) return s;
  if (num_seqs <= 0) return fail(CMR_EINVAL, "num_seqs must be > 0 when there are tokens");
  if (!cu_seqlens && num_seqs != n_tokens)
    return fail(CMR_EINVAL, "without cu_seqlens every sequence holds one token (num_seqs == n_tokens)");
  if (!start || !amount) return fail(CMR_EINVAL, "start and amount are required");
  if (cu_seqlens && (s = check_device_ptr(cu_seqlens, "cu_seqlens")) != CMR_OK) return s;
  if (pos_offset && (s = check_device_ptr(pos_offset, "pos_offset")) != CMR_OK) return s;
  if ((s = check_device_ptr(start, "start")) != CMR_OK) return s;
  if ((s = check_device_ptr(amount, "amount")) != CMR_OK) return s;
  if (device_status && (s = check_device_ptr(device_status, "device_status")) != CMR_OK) return s;
  a.status = device_status;
  a.cu = cu_seqlens;
  a.num_seqs = num_seqs;
  a.pos_offset = pos_offset;
  a.start = start;
  a.amount = amount;
  cudaError_t e = cmr::launch_rotate_qk(a, table, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "rotate_qk_shift launch");
  return CMR_OK;
}

const char* cmr_rotate_qk_kernel(int64_t n_tokens, int32_t num_layers, int32_t hq, int32_t hk,
                                 int32_t head_dim, int32_t rot_dim) {
  if (n_tokens <= 0 || num_layers <= 0 || hq < 0 || hk < 0 || hq + hk < 1) return nullptr;
  if (head_dim <= 0 || head_dim % 8 != 0) return nullptr;
  if (rot_dim < 16 || rot_dim % 16 != 0 || rot_dim > head_dim || rot_dim > 2 * cmr::kMaxFreqs)
    return nullptr;
  if ((static_cast<int64_t>(hq) + hk) * num_layers > INT32_MAX) return nullptr;
  cmr::RotateArgs a{};
  a.n_tokens = n_tokens;
  a.num_layers = num_layers;
  a.hq = hq;
  a.hk = hk;
  a.head_dim = head_dim;
  a.rot_dim = rot_dim;
  return cmr::rotate_qk_uses_staged(a) ? "rotate_qk_staged_kernel" : "rotate_qk_kernel";
}

const char* cmr_rotate_qk_cache_kernel(int64_t n_tokens, int32_t num_layers, int32_t hq,
                                       int32_t hk, int32_t head_dim, int32_t rot_dim) {
  if (cmr_rotate_qk_kernel(n_tokens, num_layers, hq, hk, head_dim, rot_dim) == nullptr)
    return nullptr;
  cmr::RotateArgs a{};
  a.n_tokens = n_tokens;
  a.num_layers = num_layers;
  a.hq = hq;
  a.hk = hk;
  a.head_dim = head_dim;
  a.rot_dim = rot_dim;
  return cmr::rotate_qk_cache_uses_staged(a) ? "rotate_qk_cache_staged_kernel"
                                             : "rotate_qk_cache_kernel";
}

cmr_status cmr_rotate_qk_cache(void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                               int32_t num_seqs, const int32_t* pos_offset, const int32_t* start,
                               const int32_t* amount, int64_t n_tokens, int32_t num_layers,
                               int32_t hq, int32_t hk, int32_t head_dim, double theta,
                               const int32_t sections[3], int32_t rot_dim, void* k_cache,
                               void* v_cache, int32_t cache_seqs, int32_t cache_ctx,
                               const int32_t* cache_slot, int32_t* device_status,
                               cmr_stream_t stream) {
  cmr::CacheArgs ca{};
  cmr::FreqTable table;
  cmr_status s = check_rotate(q, const_cast<void*>(k), n_tokens, num_layers, hq, hk, head_dim,
                              theta, sections, rot_dim, &ca.r, &table);
  if (s != CMR_OK || ca.r.n_tokens == 0) return s;
  if (num_seqs <= 0) return fail(CMR_EINVAL, "num_seqs must be > 0 when there are tokens");
  if (!cu_seqlens && num_seqs != n_tokens)
    return fail(CMR_EINVAL, "without cu_seqlens every sequence holds one token (num_seqs == n_tokens)");
  if (!start || !amount) return fail(CMR_EINVAL, "start and amount are required");
  if (hk > 0) {
    if (!v || !k_cache || !v_cache) return fail(CMR_EINVAL, "v, k_cache and v_cache are required");
    if (!aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
      return fail(CMR_EINVAL, "v, k_cache and v_cache must be 16-byte aligned");
    if (cache_seqs <= 0 || cache_ctx <= 0) return fail(CMR_EINVAL, "cache sizes must be > 0");
    if ((s = check_device_ptr(v, "v")) != CMR_OK) return s;
    if ((s = check_device_ptr(k_cache, "k_cache")) != CMR_OK) return s;
    if ((s = check_device_ptr(v_cache, "v_cache")) != CMR_OK) return s;
  }
  if (cu_seqlens && (s = check_device_ptr(cu_seqlens, "cu_seqlens")) != CMR_OK) return s;
  if (pos_offset && (s = check_device_ptr(pos_offset, "pos_offset")) != CMR_OK) return s;
  if (cache_slot && (s = check_device_ptr(cache_slot, "cache_slot")) != CMR_OK) return s;
  if ((s = check_device_ptr(start, "start")) != CMR_OK) return s;
  if ((s = check_device_ptr(amount, "amount")) != CMR_OK) return s;
  if (device_status && (s = check_device_ptr(device_status, "device_status")) != CMR_OK) return s;
  ca.r.cu = cu_seqlens;
  ca.r.num_seqs = num_seqs;
  ca.r.pos_offset = pos_offset;
  ca.r.start = start;
  ca.r.amount = amount;
  ca.v = static_cast<const uint16_t*>(v);
  ca.k_cache = static_cast<uint16_t*>(k_cache);
  ca.v_cache = static_cast<uint16_t*>(v_cache);
  ca.cache_slot = cache_slot;
  ca.cache_seqs = cache_seqs;
  ca.cache_ctx = cache_ctx;
  ca.status = device_status;
  cudaError_t e = cmr::launch_rotate_qk_cache(ca, table, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "rotate_qk_cache launch");
  return CMR_OK;
}

cmr_status cmr_copy_rotated_dims(void* dst, const void* src, int64_t rows, int32_t head_dim,
                                 int32_t rot_dim, int32_t direction, cmr_stream_t stream) {
  if (rows < 0 || head_dim <= 0 || rot_dim <= 0 || rot_dim > head_dim)
    return fail(CMR_EINVAL, "need rows >= 0 and 0 < rot_dim <= head_dim");
  if (direction != 0 && direction != 1) return fail(CMR_EINVAL, "direction must be 0 or 1");
  if (rows == 0) return CMR_OK;
  if (!dst || !src) return fail(CMR_EINVAL, "dst and src are required");
  const size_t pitch = static_cast<size_t>(head_dim) * 2;
  const size_t width = static_cast<size_t>(rot_dim) * 2;
  cudaError_t e = cudaMemcpy2DAsync(dst, pitch, src, pitch, width, static_cast<size_t>(rows),
                                    direction == 0 ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToHost,
                                    reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy2DAsync");
  return CMR_OK;
}

}  // extern "C"
