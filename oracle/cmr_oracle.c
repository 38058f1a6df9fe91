/*
 * cmr_oracle.c -- the oracle for canvas M-RoPE.  TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct fp64 CPU restatement of what the hot path
 * computes.  Only the tests, the package's smoke check and the bench's CPU
 * baseline / reference arm load it.  It shares no code, header, table or
 * constant generator with the CUDA library, and the product path never calls it.
 *
 * Sources (web pages on MiniCPM-V-4.7-1B):
 *   [P1] Core AI model zoo, "MiniCPM-V-4.7-1B: canvas M-RoPE on the Qwen3.5
 *        hybrid, on Core AI", section "The canvas rule and why the gate is on
 *        the planes".
 *   [P2] Hugging Face card mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI, section
 *        "How the VLM rides the text-only engine" (engine I/O table and the
 *        canvas table), and "What it is" (interleaved sections [11, 11, 10]).
 * The pages do not print the rotation's own parameters.  The oracle takes the
 * reading fixed for this model: rotate-half on the first rot_dim (64) dims of
 * each 256-dim head, pairs (d, d + rot_dim/2), one frequency per pair with
 * inv_freq = theta^(-2j/rot_dim), theta = 1e7, and the interleave that gives
 * frequency j to H when j % 3 == 1 and j < 33, to W when j % 3 == 2 and
 * j < 30, and to T otherwise.
 *
 * Every loop follows the rule in the pages' order; there is no blocking,
 * fusion or reordering.  Pins for every function live in tests/ (-m "not gpu").
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORC_OK 0
#define ORC_EINVAL 1

/* One 448x448 image = an 8x8 merged grid of 64 rows ([P2] canvas table). */
#define GRID_SIDE 8
#define GRID_ROWS 64
/* <image> + 64 rows + </image> + "\n" with this chat template: start = O + 67
 * ([P1] writes it as i0 + 67; [P2] start = 73 for O = 6). */
#define FRAME_TOKENS 67
/* 9 = max(H, W) + 1 on the 8x8 grid ([P2] defines amount as start minus O + 9). */
#define CANVAS_SPAN 9
/* Text-only prompts send start = 2^30 and amount = 0 ([P1], [P2]). */
#define TEXT_ONLY_START (1 << 30)

/* Rules the oracle can evaluate: the canvas rule and the pages' two red arms
 * ([P1]: in torch, amount + 1 and 1-D planes each fail all four prompts). */
#define RULE_CANVAS 0
#define RULE_AMOUNT_PLUS_ONE 1
#define RULE_PLANES_1D 2

/* ------------------------------------------------------------------------ */
/* Planes of one position                                                     */
/* ------------------------------------------------------------------------ */

/* The canvas table of [P2] for position p, canvas origin O (the index of
 * <image>) and the host's start / amount:
 *   p <  O                 -> (p, p, p)          text before the frame
 *   p == O                 -> (O, O-1, O-1)      <image>
 *   p == O + 1 + k, k < 64 -> (O, O+k/8, O+k%8)  image row k
 *   p == O + 65            -> (O, O+8, O+8)      </image>
 *   O + 65 < p < start     -> (O, O, O)          the "\n" after </image>
 *   p >= start             -> (p - amount) x 3   everything after the frame
 * The last row is tested first, so that arbitrary (start, amount) pairs, as
 * the red arm and the decode form pass them, still give one answer. */
static void canvas_planes(int64_t p, int64_t O, int64_t start, int64_t amount,
                          int64_t out[3]) {
  if (p >= start) {
    out[0] = out[1] = out[2] = p - amount;
  } else if (p < O) {
    out[0] = out[1] = out[2] = p;
  } else if (p == O) {
    out[0] = O;
    out[1] = O - 1;
    out[2] = O - 1;
  } else if (p <= O + GRID_ROWS) {
    int64_t k = p - O - 1;
    out[0] = O;
    out[1] = O + k / GRID_SIDE;
    out[2] = O + k % GRID_SIDE;
  } else if (p == O + GRID_ROWS + 1) {
    out[0] = O;
    out[1] = O + GRID_SIDE;
    out[2] = O + GRID_SIDE;
  } else {
    out[0] = out[1] = out[2] = O;
  }
}

/* The graph form: the engine binds only start and amount ([P2] engine table:
 * rope_shift_start, rope_shift_amount), so the origin follows from the
 * definition amount = start - (O + 9), i.e. O = start - amount - 9.  With the
 * text-only sentinel (2^30, 0) every realistic p lies below O -> (p, p, p). */
static void planes_from_shift(int64_t p, int64_t start, int64_t amount,
                              int64_t out[3]) {
  int64_t O = start - amount - CANVAS_SPAN;
  canvas_planes(p, O, start, amount, out);
}

/* ------------------------------------------------------------------------ */
/* Positions of a packed batch of prompts                                    */
/* ------------------------------------------------------------------------ */

/* ids: [n_tokens] int32; cu_seqlens: [num_seqs + 1] with cu[0] = 0,
 * non-decreasing, cu[num_seqs] = n_tokens.  pos: [3, n_tokens] (T, H, W planes),
 * start / amount: [num_seqs].  rule: RULE_CANVAS or one of the red arms. */
int oracle_positions(const int32_t* ids, const int32_t* cu_seqlens,
                     int32_t num_seqs, int64_t n_tokens, int32_t image_token_id,
                     int32_t rule, int32_t* pos, int32_t* start_out,
                     int32_t* amount_out) {
  if (num_seqs < 0 || n_tokens < 0) return ORC_EINVAL;
  if (num_seqs == 0) return n_tokens == 0 ? ORC_OK : ORC_EINVAL;
  if (cu_seqlens[0] != 0 || (int64_t)cu_seqlens[num_seqs] != n_tokens)
    return ORC_EINVAL;
  for (int32_t b = 0; b < num_seqs; ++b)
    if (cu_seqlens[b + 1] < cu_seqlens[b]) return ORC_EINVAL;

  for (int32_t b = 0; b < num_seqs; ++b) {
    const int64_t first = cu_seqlens[b];
    const int64_t len = (int64_t)cu_seqlens[b + 1] - first;

    /* O = the index of <image>, the canvas origin; the first one wins. */
    int64_t O = -1;
    for (int64_t p = 0; p < len; ++p) {
      if (ids[first + p] == image_token_id) {
        O = p;
        break;
      }
    }

    int64_t start, amount;
    if (O < 0) {
      start = TEXT_ONLY_START;
      amount = 0;
    } else {
      start = O + FRAME_TOKENS;
      amount = start - (O + CANVAS_SPAN);
    }
    start_out[b] = (int32_t)start;
    amount_out[b] = (int32_t)amount;

    for (int64_t p = 0; p < len; ++p) {
      int64_t v[3];
      if (rule == RULE_PLANES_1D || O < 0) {
        v[0] = v[1] = v[2] = p;
      } else if (rule == RULE_AMOUNT_PLUS_ONE) {
        planes_from_shift(p, start, amount + 1, v);
      } else {
        canvas_planes(p, O, start, amount, v);
      }
      for (int r = 0; r < 3; ++r) pos[r * n_tokens + first + p] = (int32_t)v[r];
    }
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Chunks of prompts: chunked prefill and later turns                         */
/* ------------------------------------------------------------------------ */

/* Rules for the chunked form: the canvas rule; Qwen-VL's shift, which the
 * port notes' CoreAIKit section gives as 64 and 56 from the index where the
 * pads begin (start = O + 65, so </image> and "\n" count as text after the
 * frame, amount = start - (O + 9) = 56); and plain 1-D positions (the LiteRT
 * card: the runtime feeds plain 1-D positions). */
#define CHUNK_RULE_CANVAS 0
#define CHUNK_RULE_QWEN_VL 1
#define CHUNK_RULE_PLANES_1D 2
#define QWEN_VL_FRAME_SHIFT 65

/* Chunk b holds the absolute indices pos_offset[b] + [0, len_b) of its
 * sequence (a prefill chunk, or the next turn appended to a kept state).
 * in_start / in_amount (either may be NULL: no state yet) carry what earlier
 * chunks established: (2^30, 0) while no <image> has been seen, else the
 * sequence's start and amount.  With a frame already seen, its origin follows
 * from amount = start - (O + 9).  Otherwise the chunk's first marker, if any,
 * sets O (absolute) and start / amount by the rule.  Every token then gets the
 * canvas table's row at its absolute index.  out_start / out_amount receive
 * the sequence's state after the chunk. */
int oracle_positions_chunk(const int32_t* ids, const int32_t* cu_seqlens,
                           int32_t num_seqs, int64_t n_tokens,
                           int32_t image_token_id, int32_t rule,
                           const int32_t* pos_offset, const int32_t* in_start,
                           const int32_t* in_amount, int32_t* pos,
                           int32_t* start_out, int32_t* amount_out) {
  if (num_seqs < 0 || n_tokens < 0) return ORC_EINVAL;
  if (rule < CHUNK_RULE_CANVAS || rule > CHUNK_RULE_PLANES_1D) return ORC_EINVAL;
  if (num_seqs == 0) return n_tokens == 0 ? ORC_OK : ORC_EINVAL;
  if (cu_seqlens[0] != 0 || (int64_t)cu_seqlens[num_seqs] != n_tokens)
    return ORC_EINVAL;
  for (int32_t b = 0; b < num_seqs; ++b)
    if (cu_seqlens[b + 1] < cu_seqlens[b]) return ORC_EINVAL;

  for (int32_t b = 0; b < num_seqs; ++b) {
    const int64_t first = cu_seqlens[b];
    const int64_t len = (int64_t)cu_seqlens[b + 1] - first;
    const int64_t offset = pos_offset ? pos_offset[b] : 0;
    int64_t start = in_start ? in_start[b] : TEXT_ONLY_START;
    int64_t amount = in_amount ? in_amount[b] : 0;

    if (rule == CHUNK_RULE_PLANES_1D) {
      start = TEXT_ONLY_START;
      amount = 0;
    } else if (start >= TEXT_ONLY_START) {
      /* no frame yet: the chunk's first <image>, if any, is the origin */
      for (int64_t p = 0; p < len; ++p) {
        if (ids[first + p] == image_token_id) {
          const int64_t O = offset + p;
          start = O + (rule == CHUNK_RULE_QWEN_VL ? QWEN_VL_FRAME_SHIFT : FRAME_TOKENS);
          amount = start - (O + CANVAS_SPAN);
          break;
        }
      }
    }
    start_out[b] = (int32_t)start;
    amount_out[b] = (int32_t)amount;

    for (int64_t p = 0; p < len; ++p) {
      int64_t v[3];
      planes_from_shift(offset + p, start, amount, v);
      for (int r = 0; r < 3; ++r) pos[r * n_tokens + first + p] = (int32_t)v[r];
    }
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Several frames per prompt, any grid side                                   */
/* ------------------------------------------------------------------------ */

/* The pages print the canvas only for one 448x448 thumbnail per prompt (an
 * 8x8 grid); the MNN card says its canvas positions were also checked on
 * sliced and multi-image prompts, and the thumbnail's own numbers fix the
 * structure: a frame lies on a canvas anchored at the text position where it
 * starts, and the text after it resumes one past the largest coordinate the
 * frame used ([P2]: 9 = max(H, W) + 1).  The reading taken here, for a grid of
 * side s (8 for the thumbnail, 16 for a 4x-larger grid):
 *   - a running counter c starts at 0; a text token gets (c, c, c) and c
 *     advances by 1;
 *   - every <image> marker opens a frame of s*s + 3 tokens laid at the
 *     counter's value f: <image> (f, f-1, f-1); image row k (k < s*s, row-
 *     major on the s x s grid) (f, f + k/s, f + k%s); </image> (f, f+s, f+s);
 *     the "\n" (f, f, f); the counter moves to f + s + 1, one past the
 *     frame's largest coordinate;
 *   - a frame cut short by the next marker or by the end of the prompt keeps
 *     the rows that exist, and the counter still stands at f + s + 1 after it
 *     (as a truncated thumbnail keeps start = O + 67).
 * With one marker and s = 8 this is the canvas rule (oracle_positions).
 * State after the prompt: start = (index of the last marker) + s*s + 3, and
 * amount such that the text from start on sits at p - amount; text-only
 * prompts (2^30, 0).  Parity with the pages is unpinned beyond the one-frame
 * case: they print no multi-frame values. */
int oracle_positions_frames(const int32_t* ids, const int32_t* cu_seqlens,
                            int32_t num_seqs, int64_t n_tokens,
                            int32_t image_token_id, int32_t grid_side,
                            int32_t* pos, int32_t* start_out,
                            int32_t* amount_out) {
  if (num_seqs < 0 || n_tokens < 0 || grid_side < 1 || grid_side > 128)
    return ORC_EINVAL;
  if (num_seqs == 0) return n_tokens == 0 ? ORC_OK : ORC_EINVAL;
  if (cu_seqlens[0] != 0 || (int64_t)cu_seqlens[num_seqs] != n_tokens)
    return ORC_EINVAL;
  for (int32_t b = 0; b < num_seqs; ++b)
    if (cu_seqlens[b + 1] < cu_seqlens[b]) return ORC_EINVAL;

  const int64_t s = grid_side;
  const int64_t frame_len = s * s + 3;
  for (int32_t b = 0; b < num_seqs; ++b) {
    const int64_t first = cu_seqlens[b];
    const int64_t len = (int64_t)cu_seqlens[b + 1] - first;
    int64_t c = 0;           /* the running counter */
    int64_t d = frame_len;   /* offset into the open frame; frame_len: none */
    int64_t f = 0;           /* the open frame's anchor */
    int64_t last_marker = -1;
    for (int64_t p = 0; p < len; ++p) {
      int64_t v[3];
      if (ids[first + p] == image_token_id) { /* a new frame */
        f = c;
        c = f + s + 1;
        d = 0;
        last_marker = p;
      }
      if (d < frame_len) {
        if (d == 0) {                /* <image> */
          v[0] = f;
          v[1] = v[2] = f - 1;
        } else if (d <= s * s) {     /* image row k */
          const int64_t k = d - 1;
          v[0] = f;
          v[1] = f + k / s;
          v[2] = f + k % s;
        } else if (d == s * s + 1) { /* </image> */
          v[0] = f;
          v[1] = v[2] = f + s;
        } else {                     /* the "\n" */
          v[0] = v[1] = v[2] = f;
        }
        ++d;
      } else {                       /* text */
        v[0] = v[1] = v[2] = c;
        ++c;
      }
      for (int r = 0; r < 3; ++r) pos[r * n_tokens + first + p] = (int32_t)v[r];
    }
    if (last_marker < 0) {
      start_out[b] = TEXT_ONLY_START;
      amount_out[b] = 0;
    } else {
      /* the counter after the last frame is that frame's anchor + s + 1, and
       * the text at index start takes it */
      const int64_t start = last_marker + frame_len;
      const int64_t last_anchor_next = f + s + 1;
      start_out[b] = (int32_t)start;
      amount_out[b] = (int32_t)(start - last_anchor_next);
    }
  }
  return ORC_OK;
}

/* Decode / continuation: the token at absolute index p = cache_len[b] of
 * sequence b, with that sequence's start and amount.  Generated tokens sit at
 * p - amount on all three planes ([P1]; [P2]'s canvas table counts generated
 * tokens in its last row). */
int oracle_positions_step(const int32_t* cache_len, const int32_t* start,
                          const int32_t* amount, int32_t num_seqs,
                          int32_t* pos) {
  if (num_seqs < 0) return ORC_EINVAL;
  for (int32_t b = 0; b < num_seqs; ++b) {
    int64_t v[3];
    planes_from_shift(cache_len[b], start[b], amount[b], v);
    for (int r = 0; r < 3; ++r) pos[(int64_t)r * num_seqs + b] = (int32_t)v[r];
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Frequencies                                                                */
/* ------------------------------------------------------------------------ */

/* Interleaved sections {T, H, W} ([P2], "What it is": sections [11, 11, 10]):
 * frequency j belongs to H when j % 3 == 1 and j < 3*s_H, to W when
 * j % 3 == 2 and j < 3*s_W, and to T otherwise.  For {11, 11, 10} and 32
 * frequencies that is H if j%3==1 and j<33, W if j%3==2 and j<30.
 * Returns ORC_EINVAL unless the map gives exactly s_T, s_H, s_W frequencies. */
int oracle_freq_planes(int32_t rot_dim, const int32_t sections[3],
                       int32_t* plane) {
  if (rot_dim <= 0 || rot_dim % 2 != 0) return ORC_EINVAL;
  const int32_t nfreq = rot_dim / 2;
  if (sections[0] < 0 || sections[1] < 0 || sections[2] < 0) return ORC_EINVAL;
  if (sections[0] + sections[1] + sections[2] != nfreq) return ORC_EINVAL;
  int32_t count[3] = {0, 0, 0};
  for (int32_t j = 0; j < nfreq; ++j) {
    int32_t r = 0;
    if (j % 3 == 1 && j < 3 * sections[1])
      r = 1;
    else if (j % 3 == 2 && j < 3 * sections[2])
      r = 2;
    plane[j] = r;
    count[r]++;
  }
  for (int r = 0; r < 3; ++r)
    if (count[r] != sections[r]) return ORC_EINVAL;
  return ORC_OK;
}

/* inv_freq_j = theta^(-2j / rot_dim), one frequency per rotated pair. */
static double inv_freq(double theta, int32_t j, int32_t rot_dim) {
  return pow(theta, -2.0 * (double)j / (double)rot_dim);
}

/* ------------------------------------------------------------------------ */
/* Rotation                                                                   */
/* ------------------------------------------------------------------------ */

/* Rotate-half on one head row, in fp64: for d < rot_dim/2 the pair
 * (x_d, x_{d + rot_dim/2}) turns by the angle of frequency d at the position
 * of that frequency's plane.  Dims >= rot_dim are left alone. */
static void rotate_row(double* x, const int32_t* plane, const int32_t* pos,
                       int64_t n_tokens, int64_t t, double theta,
                       int32_t rot_dim) {
  const int32_t half = rot_dim / 2;
  for (int32_t d = 0; d < half; ++d) {
    double a = (double)pos[(int64_t)plane[d] * n_tokens + t] *
               inv_freq(theta, d, rot_dim);
    double c = cos(a), s = sin(a);
    double x1 = x[d], x2 = x[d + half];
    x[d] = x1 * c - x2 * s;
    x[d + half] = x2 * c + x1 * s;
  }
}

static int check_rotate_args(int64_t n_tokens, int32_t num_layers,
                             int32_t heads, int32_t head_dim, double theta,
                             int32_t rot_dim) {
  if (n_tokens < 0 || num_layers < 0 || heads < 0) return ORC_EINVAL;
  if (head_dim <= 0 || rot_dim <= 0 || rot_dim % 2 != 0 || rot_dim > head_dim)
    return ORC_EINVAL;
  if (!(theta > 0.0) || !isfinite(theta)) return ORC_EINVAL;
  return ORC_OK;
}

/* x: [num_layers, n_tokens, heads, head_dim] doubles, rotated in place.
 * pos: [3, n_tokens], shared by every layer and head. */
int oracle_rotate_f64(double* x, const int32_t* pos, int64_t n_tokens,
                      int32_t num_layers, int32_t heads, int32_t head_dim,
                      double theta, const int32_t sections[3],
                      int32_t rot_dim) {
  int32_t plane[512];
  if (check_rotate_args(n_tokens, num_layers, heads, head_dim, theta,
                        rot_dim) != ORC_OK || rot_dim > 1024)
    return ORC_EINVAL;
  if (oracle_freq_planes(rot_dim, sections, plane) != ORC_OK) return ORC_EINVAL;
  for (int32_t l = 0; l < num_layers; ++l)
    for (int64_t t = 0; t < n_tokens; ++t)
      for (int32_t h = 0; h < heads; ++h) {
        double* row = x + (((int64_t)l * n_tokens + t) * heads + h) * head_dim;
        rotate_row(row, plane, pos, n_tokens, t, theta, rot_dim);
      }
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* bfloat16                                                                   */
/* ------------------------------------------------------------------------ */

/* bf16 is the top half of an IEEE binary32: the value is exact in double. */
double oracle_bf16_to_f64(uint16_t bits) {
  uint32_t w = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &w, sizeof f);
  return (double)f;
}

/* Round a double to the nearest bf16, ties to even, in one step (never via
 * binary32, which would round twice).  bf16: 8 exponent bits, 7 fraction bits,
 * normals 2^-126 .. (2 - 2^-7) 2^127, subnormal spacing 2^-133. */
uint16_t oracle_f64_to_bf16(double x) {
  if (isnan(x)) return 0x7FC0;
  const uint16_t sign = signbit(x) ? 0x8000 : 0;
  double m = fabs(x);
  if (m == 0.0) return sign;
  if (isinf(m)) return sign | 0x7F80;
  int e;
  frexp(m, &e);            /* m = f * 2^e, f in [0.5, 1): binade exponent e-1 */
  int E = e - 1;
  if (E < -126) E = -126;  /* subnormal range shares the spacing of 2^-126 */
  const double ulp = ldexp(1.0, E - 7);
  const double q = rint(m / ulp); /* exact division; rint = ties to even */
  const double r = q * ulp;
  const double max_bf16 = ldexp(255.0, 127 - 7); /* (2 - 2^-7) * 2^127 */
  if (r > max_bf16) return sign | 0x7F80;
  float f = (float)r; /* exact: r has at most 8 significant bits */
  uint32_t w;
  memcpy(&w, &f, sizeof w);
  return sign | (uint16_t)((w >> 16) & 0x7FFF);
}

/* x: [num_layers, n_tokens, heads, head_dim] bf16 bit patterns, rotated in
 * place: each head row goes to fp64, is rotated by rotate_row and comes back
 * through oracle_f64_to_bf16.  Dims >= rot_dim keep their bits.  If f64_out is
 * not NULL it receives the unrounded rotated rows, same layout as x. */
int oracle_rotate_bf16(uint16_t* x, const int32_t* pos, int64_t n_tokens,
                       int32_t num_layers, int32_t heads, int32_t head_dim,
                       double theta, const int32_t sections[3], int32_t rot_dim,
                       double* f64_out) {
  int32_t plane[512];
  double row[1024];
  if (check_rotate_args(n_tokens, num_layers, heads, head_dim, theta,
                        rot_dim) != ORC_OK || head_dim > 1024)
    return ORC_EINVAL;
  if (oracle_freq_planes(rot_dim, sections, plane) != ORC_OK) return ORC_EINVAL;
  for (int32_t l = 0; l < num_layers; ++l)
    for (int64_t t = 0; t < n_tokens; ++t)
      for (int32_t h = 0; h < heads; ++h) {
        const int64_t off = (((int64_t)l * n_tokens + t) * heads + h) * head_dim;
        for (int32_t d = 0; d < head_dim; ++d)
          row[d] = oracle_bf16_to_f64(x[off + d]);
        rotate_row(row, plane, pos, n_tokens, t, theta, rot_dim);
        for (int32_t d = 0; d < rot_dim; ++d) x[off + d] = oracle_f64_to_bf16(row[d]);
        if (f64_out)
          for (int32_t d = 0; d < head_dim; ++d) f64_out[off + d] = row[d];
      }
  return ORC_OK;
}
