/*
 * cmr.h -- canvas M-RoPE for the Qwen3.5-hybrid decoder of MiniCPM-V-4.7-1B,
 * as a C ABI over hand-written sm_100a (B200) CUDA kernels.
 *
 * Two steps (HF card mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI, "How the VLM rides
 * the text-only engine"; Core AI model zoo port notes, "The canvas rule and
 * why the gate is on the planes"):
 *   1. positions: the three position planes (T, H, W) of every token, derived
 *      from the token ids by the canvas rule;
 *   2. rotate: rotate-half M-RoPE of the Q and K heads of the full-attention
 *      layers, in place, with cos/sin built per frequency from the plane that
 *      the interleaved sections (e.g. [11, 11, 10]) assign to it.
 *
 * Conventions for every entry point:
 *   - Pointers named "device" must point to memory the current CUDA device can
 *     read/write (cudaMalloc, torch CUDA tensors, managed memory).  Host
 *     pointers are rejected with CMR_EINVAL where the runtime can tell.  The
 *     one exception, cmr_positions_rotate_qk_host, takes mapped page-locked
 *     host memory instead (and rejects device memory).
 *   - The caller owns every buffer.  The library never allocates, frees or
 *     synchronises; all work is enqueued on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream) and runs asynchronously.
 *   - Arguments are validated on the host before anything is enqueued; on any
 *     non-CMR_OK return nothing was enqueued, except CMR_ECUDA from a launch,
 *     which means the launch itself failed.  cmr_last_error_message() then
 *     gives a one-line reason (per calling thread).
 *   - Kernels never trap.  Malformed device-side data (cu_seqlens, cache
 *     indices) and a staged copy that never arrived are reported through an
 *     optional device status word; every wait inside a kernel is bounded.
 */
#ifndef CMR_H_
#define CMR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define CMR_API __attribute__((visibility("default")))
#else
#define CMR_API
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* cmr_stream_t;

typedef enum cmr_status {
  CMR_OK = 0,
  CMR_EINVAL = 1,       /* an argument is out of range, misaligned or null */
  CMR_ECUDA = 2,        /* a CUDA runtime call or a kernel launch failed */
  CMR_EUNSUPPORTED = 3  /* valid, but outside the shapes this build handles */
} cmr_status;

/* Bits a kernel ORs into the optional device status word. */
#define CMR_DEVICE_BAD_CU_SEQLENS 1 /* cu_seqlens not 0 .. n_tokens, non-decreasing */
#define CMR_DEVICE_CACHE_RANGE 2    /* a token's cache index or slot outside the cache */
#define CMR_DEVICE_WAIT_TIMEOUT 4   /* a staged kernel waited over 1 s for one of its own
                                       copies and gave up: the call's results are not to be
                                       trusted (rows of the tiles involved may be unrotated
                                       or half written) */

/* Position rules for cmr_positions_chunk. */
#define CMR_RULE_CANVAS 0    /* this model's canvas rule: start = O + 67, amount 58 */
#define CMR_RULE_QWEN_VL 1   /* Qwen-VL's shift: start = O + 65, amount 56 */
#define CMR_RULE_PLANES_1D 2 /* plain 1-D positions: (p, p, p), state (2^30, 0) */

/* Planes of a packed batch of prompts (the canvas table, HF card
 * mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI, "How the VLM rides the text-only
 * engine").  For prompt b, O = the first local index whose id equals
 * image_token_id (the <image> marker, 248078 for this model).  Then, for each
 * local index p:
 *   p <  O                 -> (p, p, p)
 *   p == O                 -> (O, O-1, O-1)
 *   p == O + 1 + k, k < 64 -> (O, O + k/8, O + k%8)   (8x8 grid, row-major)
 *   p == O + 65            -> (O, O+8, O+8)
 *   O + 65 < p < start     -> (O, O, O)
 *   p >= start             -> (p - amount) on all three planes
 * with start = O + 67 and amount = start - (O + 9) = 58 (the port notes give
 * start as i0 + 67 and amount as 58).  A prompt with no marker is text-only: start =
 * 2^30, amount = 0, every token (p, p, p).  Later markers in a prompt are
 * ordinary tokens.  Frames cut off by the end of a prompt keep the rows that
 * exist; start still reads O + 67.
 *
 *   ids          device int32 [n_tokens], prompts packed back to back
 *   cu_seqlens   device int32 [num_seqs + 1]: cu[0] = 0, non-decreasing,
 *                cu[num_seqs] = n_tokens; prompt b is ids[cu[b] .. cu[b+1])
 *   num_seqs     >= 0 (0 requires n_tokens == 0)
 *   n_tokens     0 .. INT32_MAX
 *   out_pos      device int32 [3, n_tokens], plane-major: T row, H row, W row
 *   out_start, out_amount   device int32 [num_seqs]
 *   device_status  optional device int32 [1] (may be NULL).  If cu_seqlens is
 *                malformed, the kernels OR CMR_DEVICE_BAD_CU_SEQLENS into it
 *                and write no planes for the prompts whose bounds are invalid
 *                (their out_start / out_amount entries are then unspecified).
 *                The library never clears it.
 * Two kernels: one CTA per prompt (a cluster of up to 16 CTAs when prompts
 * average more than 65,536 tokens) scans its ids up to the first marker (no
 * id is read twice) and writes the state; then CTAs over slices of 2,048
 * tokens (8,192 where the batch still fills three waves of CTAs) write the
 * planes, reading the state back from out_start / out_amount.
 * Errors: CMR_EINVAL for null required pointers, negative sizes, num_seqs = 0
 * with n_tokens > 0, or n_tokens > INT32_MAX. */
CMR_API cmr_status cmr_positions(const int32_t* ids, const int32_t* cu_seqlens,
                         int32_t num_seqs, int64_t n_tokens,
                         int32_t image_token_id, int32_t* out_pos,
                         int32_t* out_start, int32_t* out_amount,
                         int32_t* device_status, cmr_stream_t stream);

/* Planes of a batch of prompt CHUNKS: chunked prefill, and later turns that
 * append to a kept state (port notes, "Prefill in chunks and a second turn":
 * S = 16 prefill answers as the one-token order; a second question reuses
 * the state after turn 1).  Chunk b is ids[cu[b] .. cu[b+1]) and holds the
 * absolute indices pos_offset[b] + 0, 1, ... of its sequence.  The sequence's
 * state before the chunk is (in_start[b], in_amount[b]) -- (2^30, 0) while no
 * <image> has been seen, the value cmr_positions / an earlier chunk returned
 * otherwise.  If a frame is known, its origin follows from amount = start -
 * (O + 9); if not, the chunk's first marker at local index m sets O =
 * pos_offset[b] + m and
 *   CMR_RULE_CANVAS:    start = O + 67, amount = 58 (as cmr_positions);
 *   CMR_RULE_QWEN_VL:   start = O + 65, amount = 56 (port notes, CoreAIKit:
 *                       Qwen-VL's rule shifts by 64 from the pads and by 56;
 *                       </image> and "\n" then count as text after the
 *                       frame);
 *   CMR_RULE_PLANES_1D: no shift at all, state (2^30, 0) (the LiteRT card:
 *                       the runtime feeds plain 1-D positions).
 * Each token gets the canvas table's row at its absolute index.  With all
 * offsets 0, no incoming state and CMR_RULE_CANVAS this is cmr_positions.
 *
 *   ids, cu_seqlens, num_seqs, n_tokens, image_token_id, out_pos,
 *   device_status   as in cmr_positions
 *   rule            one of CMR_RULE_*
 *   pos_offset      device int32 [num_seqs], or NULL for all zeros
 *   in_start, in_amount   device int32 [num_seqs], or NULL for (2^30, 0)
 *   out_start, out_amount device int32 [num_seqs]: the state after the chunk.
 *                   Must not overlap in_start / in_amount (use two buffers and
 *                   swap them between chunks).
 * Absolute indices (pos_offset[b] plus the chunk's length) must stay below
 * 2^30 - 67: a start of 2^30 or more reads as "no frame seen".
 * Errors: as cmr_positions, plus CMR_EINVAL for an unknown rule or
 * overlapping incoming and outgoing state. */
CMR_API cmr_status cmr_positions_chunk(const int32_t* ids, const int32_t* cu_seqlens,
                                       int32_t num_seqs, int64_t n_tokens,
                                       int32_t image_token_id, int32_t rule,
                                       const int32_t* pos_offset,
                                       const int32_t* in_start,
                                       const int32_t* in_amount, int32_t* out_pos,
                                       int32_t* out_start, int32_t* out_amount,
                                       int32_t* device_status, cmr_stream_t stream);

/* Planes of prompts holding several image frames, on an s x s grid of any
 * side (s = grid_side: 8 for the 448x448 thumbnail's 64 rows, 16 for a grid
 * of 256).  The pages print the canvas for one thumbnail only (HF card
 * mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI, "How the VLM rides the text-only
 * engine"); the MNN card ("Validation") says sliced and multi-image prompts
 * were checked too, without values.  The reading implemented: a running
 * counter c gives each text token (c, c, c) and advances by 1; EVERY marker
 * opens a frame of s*s + 3 tokens anchored at the counter's value f:
 *   <image> (f, f-1, f-1); row k < s*s (f, f + k/s, f + k%s) (row-major);
 *   </image> (f, f+s, f+s); the "\n" after it (f, f, f);
 * and the counter then stands at f + s + 1, one past the frame's largest
 * coordinate (the card's 9 = max(H, W) + 1), also when the next marker or the
 * end of the prompt cuts the frame short.  With one marker and s = 8 this is
 * cmr_positions.  The state is start = (last marker) + s*s + 3 and amount with
 * every later text token at p - amount, so cmr_positions_step and the shift
 * forms continue a prompt after its last frame; text-only (2^30, 0).
 *
 *   ids, cu_seqlens, num_seqs, n_tokens, image_token_id, out_pos, out_start,
 *   out_amount, device_status   as in cmr_positions
 *   grid_side      1 .. 128
 *   workspace      device memory, 16-byte aligned, of workspace_bytes >= 16 *
 *                  num_seqs; cmr_positions_frames_workspace_bytes gives the
 *                  size for full parallelism (16 B per sequence per slice of
 *                  about 4,096 tokens); a smaller one works with fewer,
 *                  longer slices.  It holds one summary per slice between the
 *                  call's two kernels; its contents before and after a call
 *                  do not matter, but calls that overlap on the device must
 *                  not share it.
 * Every coordinate must fit in int32.  Two kernels: a per-slice summary (marker
 * count, first and last marker, text between frames), then the planes, the
 * second launched to overlap the first.
 * Errors: as cmr_positions, plus CMR_EINVAL for grid_side outside 1 .. 128 and a
 * missing, misaligned or too small workspace. */
CMR_API cmr_status cmr_positions_frames(const int32_t* ids, const int32_t* cu_seqlens,
                                        int32_t num_seqs, int64_t n_tokens,
                                        int32_t image_token_id, int32_t grid_side,
                                        int32_t* out_pos, int32_t* out_start,
                                        int32_t* out_amount, void* workspace,
                                        size_t workspace_bytes, int32_t* device_status,
                                        cmr_stream_t stream);

/* Workspace bytes for cmr_positions_frames at full parallelism (0 for no
 * sequences).  No CUDA call is made. */
CMR_API size_t cmr_positions_frames_workspace_bytes(int32_t num_seqs, int64_t n_tokens);

/* cmr_positions_frames for callers that cannot allocate device memory and so
 * cannot hand over a workspace: code running while a CUDA graph is being
 * captured (cudaMalloc is refused there), serving loops that forbid
 * allocation on the hot path (cudaMalloc may synchronise the device and its
 * latency is unbounded), and plug-ins whose host application owns all device
 * memory through its own allocator.  Same arguments, results and errors as
 * cmr_positions_frames, without the workspace: the slice summaries live in a
 * scratch array built into the library, 256 KB (16,384 summaries of 16
 * bytes) that every device loading the library holds until the process
 * exits.  It serves up to 16,384 sequences per call (more: CMR_EINVAL, and
 * cmr_positions_frames with a workspace is the way); the more sequences, the
 * fewer and longer the slices each prompt is split into.
 *   - The first call on each device looks up the scratch's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before capturing any stream into a CUDA graph.
 *   - Every call on a device shares the one scratch: calls that overlap on
 *     the device (other streams, other host threads) race and must be
 *     serialised by the caller.  A call writes every summary it reads, so
 *     nothing is left to clear between calls.
 *   - It allocates nothing: no cudaMalloc, no cudaFree, no library allocator.
 * The paper has no counterpart: this is an interface for such callers only. */
CMR_API cmr_status cmr_positions_frames_noalloc(const int32_t* ids, const int32_t* cu_seqlens,
                                                int32_t num_seqs, int64_t n_tokens,
                                                int32_t image_token_id, int32_t grid_side,
                                                int32_t* out_pos, int32_t* out_start,
                                                int32_t* out_amount, int32_t* device_status,
                                                cmr_stream_t stream);

/* Planes of one new token per sequence, for decode and continuation (port
 * notes: generated tokens sit at p - amount; the canvas table's last row,
 * after the frame, covers generated tokens too).  Token b sits at absolute
 * index p = cache_len[b] of its sequence, whose start / amount came from
 * cmr_positions.  As in the engine, which binds only start and amount, the
 * origin follows from amount = start - (O + 9); the token then gets the row of
 * the canvas table above for index p (p >= start -> (p - amount) x 3; the
 * text-only pair (2^30, 0) gives (p, p, p)).
 *
 *   cache_len, start, amount   device int32 [num_seqs]
 *   out_pos      device int32 [3, num_seqs], plane-major
 * Errors: CMR_EINVAL for null pointers or num_seqs < 0. */
CMR_API cmr_status cmr_positions_step(const int32_t* cache_len, const int32_t* start,
                              const int32_t* amount, int32_t num_seqs,
                              int32_t* out_pos, cmr_stream_t stream);

/* Rotate Q and K in place with interleaved M-RoPE (HF card "What it is":
 * three planes T, H, W with interleaved sections [11, 11, 10]; port notes:
 * `_mrope_freq_masks`, `forward_stateful_core(cos_sin=...)`).
 * With F = rot_dim / 2 frequencies, frequency j belongs to plane
 *   H if j % 3 == 1 and j < 3 * sections[1],
 *   W if j % 3 == 2 and j < 3 * sections[2],
 *   T otherwise,
 * has inv_freq_j = theta^(-2j / rot_dim), and at token t turns the pair
 * (x_j, x_{j+F}) of every head by a = pos[plane_j][t] * inv_freq_j:
 *   x_j     <- x_j cos a - x_{j+F} sin a
 *   x_{j+F} <- x_{j+F} cos a + x_j sin a
 * Dims rot_dim .. head_dim-1 are not read or written.  The angle is formed and
 * reduced modulo 2*pi in fp64, cos/sin and the rotation run in fp32, and the
 * result is rounded to bf16 (nearest-even).  Large batches with rot_dim 64 run
 * a TMA-staged kernel; the result is the same bit for bit either way.
 *
 *   q      device bf16 [num_layers, n_tokens, hq, head_dim], 16-byte aligned
 *   k      device bf16 [num_layers, n_tokens, hk, head_dim], 16-byte aligned
 *          (either may be NULL when its head count is 0)
 *   pos    device int32 [3, n_tokens] (plane-major), shared by every layer
 *   n_tokens >= 0, num_layers >= 0 (either 0: nothing to do, CMR_OK)
 *   hq, hk >= 0 with hq + hk >= 1
 *   head_dim  multiple of 8
 *   theta  > 0 and finite (1e7 for this model)
 *   sections  host int32 [3] = {T, H, W} frequency counts, summing to
 *          rot_dim / 2, each realisable by the interleave above
 *   rot_dim   multiple of 16, 16 .. min(head_dim, 256)  (64 for this model)
 *   device_status  optional device int32 [1] (may be NULL): receives
 *          CMR_DEVICE_WAIT_TIMEOUT if a staged copy timed out.  Never cleared.
 * Errors: CMR_EINVAL for any violation above; CMR_EUNSUPPORTED when
 * (hq + hk) * num_layers > INT32_MAX. */
CMR_API cmr_status cmr_rotate_qk(void* q, void* k, const int32_t* pos, int64_t n_tokens,
                         int32_t num_layers, int32_t hq, int32_t hk,
                         int32_t head_dim, double theta,
                         const int32_t sections[3], int32_t rot_dim,
                         int32_t* device_status, cmr_stream_t stream);

/* The whole path in one call: the results of cmr_positions and then
 * cmr_rotate_qk with those planes (same arguments, same results, bit for
 * bit).  Two kernels: the origin scan writes each prompt's (start, amount);
 * the rotation is launched with programmatic stream serialization behind it,
 * so its CTAs start while the scan runs and the TMA loads of Q and K (which
 * the scan never touches) go out at once; it then derives each token's planes
 * from its prompt's state, writes them to out_pos and rotates with them.
 * Launching the two calls separately cannot overlap them, because a caller's
 * kernel before a plain cmr_rotate_qk may still be writing Q/K when it
 * signals.  With no layers to rotate, the planes kernel of cmr_positions
 * writes out_pos instead.  With malformed cu_seqlens the planes and rows of
 * the prompts involved are unspecified (CMR_DEVICE_BAD_CU_SEQLENS is set).
 *
 *   ids, cu_seqlens, num_seqs, n_tokens, image_token_id, out_pos, out_start,
 *   out_amount     as in cmr_positions (out_pos is also the rotation's pos)
 *   q, k, num_layers, hq, hk, head_dim, theta, sections, rot_dim
 *                  as in cmr_rotate_qk (n_tokens tokens)
 *   device_status  optional, receives the bits of both steps
 * Errors: every check of both calls runs before anything is enqueued. */
CMR_API cmr_status cmr_positions_rotate_qk(const int32_t* ids, const int32_t* cu_seqlens,
                                           int32_t num_seqs, int64_t n_tokens,
                                           int32_t image_token_id, int32_t* out_pos,
                                           int32_t* out_start, int32_t* out_amount, void* q,
                                           void* k, int32_t num_layers, int32_t hq, int32_t hk,
                                           int32_t head_dim, double theta,
                                           const int32_t sections[3], int32_t rot_dim,
                                           int32_t* device_status, cmr_stream_t stream);

/* cmr_positions_rotate_qk on a batch that lives in host memory: the same
 * arguments, results and errors, with ids, cu_seqlens, out_pos, out_start,
 * out_amount, q and k all page-locked host memory mapped into the device's
 * address space at the same address (cudaHostAlloc / cudaMallocHost, or
 * cudaHostRegister with cudaHostRegisterMapped, on a system with unified
 * addressing; PyTorch's pin_memory() tensors qualify).  The kernels read and
 * write those buffers directly over PCIe (zero-copy): each id once, the
 * rotated dims of each head row (rot_dim * 2 bytes of every head_dim * 2)
 * read and written once, the planes and the state written once; the other
 * dims of Q/K never cross the bus.  Nothing is staged in device memory and
 * no copy engine is used, so a caller whose batch is on the host needs no
 * device buffers and no copies of its own.  The rotation runs on the
 * register kernel (plain loads and stores; tensor maps are never built over
 * host memory).  Calls are asynchronous: the host may read the results, and
 * must not touch the buffers, until the stream has been synchronised.
 * device_status may be device memory or mapped host memory.
 * Errors: as cmr_positions_rotate_qk, plus CMR_EINVAL for a buffer that is
 * not mapped page-locked host memory (device memory and pageable host memory
 * are refused). */
CMR_API cmr_status cmr_positions_rotate_qk_host(const int32_t* ids, const int32_t* cu_seqlens,
                                                int32_t num_seqs, int64_t n_tokens,
                                                int32_t image_token_id, int32_t* out_pos,
                                                int32_t* out_start, int32_t* out_amount, void* q,
                                                void* k, int32_t num_layers, int32_t hq,
                                                int32_t hk, int32_t head_dim, double theta,
                                                const int32_t sections[3], int32_t rot_dim,
                                                int32_t* device_status, cmr_stream_t stream);

/* cmr_rotate_qk with the planes derived inside the kernel instead of read
 * from pos [3, n_tokens]: token t of prompt b (cu[b] <= t < cu[b+1]) sits at
 * absolute index p = pos_offset[b] + t - cu[b] and gets the canvas table's
 * row for p under its sequence's (start[b], amount[b]), exactly as
 * cmr_positions_step would give it.  One launch then covers a decode step
 * (cu_seqlens = NULL: token b is sequence b, p = pos_offset[b]) or a prefill
 * chunk whose state is known, and the 24 B/token pos round trip disappears.
 *
 *   q, k, n_tokens, num_layers, hq, hk, head_dim, theta, sections, rot_dim,
 *   device_status as in cmr_rotate_qk
 *   cu_seqlens    device int32 [num_seqs + 1] as in cmr_positions (it must be
 *                 well formed: it is not checked on the device), or NULL when
 *                 num_seqs == n_tokens and each sequence holds one token
 *   pos_offset    device int32 [num_seqs], or NULL for all zeros
 *   start, amount device int32 [num_seqs]
 * Errors: as cmr_rotate_qk, plus CMR_EINVAL for num_seqs <= 0 with tokens,
 * missing start/amount, or cu_seqlens == NULL with num_seqs != n_tokens. */
CMR_API cmr_status cmr_rotate_qk_shift(void* q, void* k, const int32_t* cu_seqlens,
                                       int32_t num_seqs, const int32_t* pos_offset,
                                       const int32_t* start, const int32_t* amount,
                                       int64_t n_tokens, int32_t num_layers, int32_t hq,
                                       int32_t hk, int32_t head_dim, double theta,
                                       const int32_t sections[3], int32_t rot_dim,
                                       int32_t* device_status, cmr_stream_t stream);

/* Name of the kernel that cmr_rotate_qk / cmr_rotate_qk_shift /
 * cmr_positions_rotate_qk launch for these shapes: "rotate_qk_staged_kernel"
 * (TMA-staged, rot_dim 64, large batches) or "rotate_qk_kernel"
 * (register-resident rows, every other case).  It is a prediction from the
 * shapes alone; a call still takes rotate_qk_kernel when
 *   - the driver cannot encode tensor maps for the buffers (any driver for
 *     sm_100a can, for contiguous 16-byte aligned Q/K of under 1 TB per layer);
 *   - the staged ring needs more than 48 KB of shared memory (more than 24
 *     head rows of Q and K per token: not this model's 8 + 2), the process has
 *     not launched that form on this device before, and the call is being
 *     captured into a CUDA graph (or its stream cannot be queried).
 * cmr_last_rotate_kernel names the kernel a call actually launched.
 * Returns NULL when the shapes are invalid or there is nothing to launch.
 * Static strings; no CUDA call is made. */
CMR_API const char* cmr_rotate_qk_kernel(int64_t n_tokens, int32_t num_layers, int32_t hq,
                                         int32_t hk, int32_t head_dim, int32_t rot_dim);

/* The same for cmr_rotate_qk_cache: "rotate_qk_cache_staged_kernel" (TMA-staged,
 * rot_dim 64, large batches, head_dim <= 256, K/V token rows a multiple of
 * 128 B) or "rotate_qk_cache_kernel".  A call still takes
 * rotate_qk_cache_kernel when the driver cannot encode tensor maps for the
 * buffers, or when the staged kernel's ring needs more than 48 KB of shared
 * memory (this model's 8 + 2 heads: 73 KB), the process has not launched it
 * on this device before, and the call is being captured into a CUDA graph (or
 * its stream cannot be queried).  NULL when the shapes are invalid or there is
 * nothing to launch. */
CMR_API const char* cmr_rotate_qk_cache_kernel(int64_t n_tokens, int32_t num_layers,
                                               int32_t hq, int32_t hk, int32_t head_dim,
                                               int32_t rot_dim);

/* Rotate Q in place and write each token's rotated K row and its V row into
 * a KV cache, in one pass: the step after the rotation in the full-attention
 * layers (HF card mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI, "How the VLM rides
 * the text-only engine": keyCache / valueCache [6, 1, 2, -1, 256], the 6
 * full-attention layers, context up to 4,096).  Token t of prompt b sits at
 * absolute index p = pos_offset[b] + t - cu[b]; its planes are the canvas rows
 * at p under (start[b], amount[b]) as in cmr_rotate_qk_shift; its rows land at
 *   k_cache[l, slot, h, p, :] = K[l, t, h, :] rotated (all head_dim dims)
 *   v_cache[l, slot, h, p, :] = V[l, t, h, :]
 * with slot = cache_slot[b] (or b when cache_slot is NULL).  K and V are not
 * modified.  A token whose p or slot falls outside the cache writes no K/V row
 * and ORs CMR_DEVICE_CACHE_RANGE into device_status.  Large batches with
 * rot_dim 64 run a TMA-staged kernel (cmr_rotate_qk_cache_kernel says which);
 * the result is the same bit for bit either way.
 *
 *   q                  device bf16 [num_layers, n_tokens, hq, head_dim], rotated in place
 *   k, v               device bf16 [num_layers, n_tokens, hk, head_dim], read only
 *   k_cache, v_cache   device bf16 [num_layers, cache_seqs, hk, cache_ctx, head_dim]
 *   cache_slot         device int32 [num_seqs], or NULL
 *   cache_seqs, cache_ctx  > 0
 *   cu_seqlens, num_seqs, pos_offset, start, amount   as in cmr_rotate_qk_shift
 *   the rest           as in cmr_rotate_qk
 * All of q, k, v, k_cache, v_cache 16-byte aligned; the caches must not
 * overlap q, k or v.  Two tokens that land on the same (slot, position) --
 * sequences sharing a slot, or repeated indices -- race; give each sequence
 * its own slot.
 * Errors: as cmr_rotate_qk_shift, plus CMR_EINVAL for missing or misaligned
 * v / caches or non-positive cache sizes. */
CMR_API cmr_status cmr_rotate_qk_cache(void* q, const void* k, const void* v,
                                       const int32_t* cu_seqlens, int32_t num_seqs,
                                       const int32_t* pos_offset, const int32_t* start,
                                       const int32_t* amount, int64_t n_tokens,
                                       int32_t num_layers, int32_t hq, int32_t hk,
                                       int32_t head_dim, double theta,
                                       const int32_t sections[3], int32_t rot_dim,
                                       void* k_cache, void* v_cache, int32_t cache_seqs,
                                       int32_t cache_ctx, const int32_t* cache_slot,
                                       int32_t* device_status, cmr_stream_t stream);

/* Copy only the rotated dims of head rows between host and device memory: the
 * first rot_dim of every head_dim-wide bf16 row (a pitched copy of rot_dim * 2
 * bytes out of every head_dim * 2), for `rows` consecutive rows, on `stream`.
 * For callers whose Q/K live in host memory: the rotation reads and writes
 * only these dims, so moving the rest over PCIe is wasted; rows copied back
 * keep their untouched dims on the host side.
 *
 *   dst, src    host (pinned for asynchrony) or device memory, one of each
 *   rows        >= 0 rows of head_dim bf16 elements each
 *   direction   0: host -> device, 1: device -> host
 * Errors: CMR_EINVAL for null pointers, rot_dim > head_dim or non-positive
 * sizes, an unknown direction; CMR_ECUDA if the copy cannot be enqueued. */
CMR_API cmr_status cmr_copy_rotated_dims(void* dst, const void* src, int64_t rows,
                                         int32_t head_dim, int32_t rot_dim,
                                         int32_t direction, cmr_stream_t stream);

/* Static, never-null description of a status code. */
CMR_API const char* cmr_status_string(cmr_status s);

/* One-line reason for the last non-CMR_OK return on the calling thread. */
CMR_API const char* cmr_last_error_message(void);

/* Name of the rotate kernel that the calling thread's last successful rotate
 * call enqueued ("rotate_qk_staged_kernel", "rotate_qk_kernel",
 * "rotate_qk_cache_staged_kernel" or "rotate_qk_cache_kernel"); "" before the
 * first.  Static strings; no CUDA call is made. */
CMR_API const char* cmr_last_rotate_kernel(void);

/* ABI version: major * 10000 + minor * 100 + patch. */
CMR_API int32_t cmr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CMR_H_ */
