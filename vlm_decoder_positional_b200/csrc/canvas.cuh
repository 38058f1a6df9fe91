// The canvas table as device code, shared by the positions and rotate kernels.
//
// HF card mlboydaisuke/MiniCPM-V-4.7-1B-CoreAI, "How the VLM rides the
// text-only engine": with O the index of <image> and the host's start/amount,
// position p gets
//   p <  O                 -> (p, p, p)
//   p == O                 -> (O, O-1, O-1)        <image>
//   p == O + 1 + k, k < 64 -> (O, O+k/8, O+k%8)    image row k (8x8 grid)
//   p == O + 65            -> (O, O+8, O+8)        </image>
//   O + 65 < p < start     -> (O, O, O)            the "\n"
//   p >= start             -> (p - amount) x 3     everything after the frame
// Since amount = start - (O + 9), the pair (start, amount) alone fixes O; the
// text-only pair (2^30, 0) puts every realistic p below O.
#pragma once

#include "cmr_internal.cuh"

namespace cmr {

struct Planes {
  int32_t t, h, w;
};

// Row for absolute index p.  "After the frame" is tested first, so any
// (start, amount) pair gives one answer.
__device__ __forceinline__ Planes canvas_row(int64_t p, int64_t start, int64_t amount) {
  if (p >= start) {
    const int32_t v = static_cast<int32_t>(p - amount);
    return {v, v, v};
  }
  const int64_t origin = start - amount - kCanvasSpan;
  const int64_t d = p - origin;  // offset into the frame
  const int32_t o = static_cast<int32_t>(origin);
  if (d < 0) {
    const int32_t v = static_cast<int32_t>(p);
    return {v, v, v};
  }
  if (d == 0) return {o, o - 1, o - 1};  // <image>
  if (d <= kGridRows) {                  // image row k = d - 1
    const int32_t k = static_cast<int32_t>(d - 1);
    return {o, o + k / kGridSide, o + k % kGridSide};
  }
  if (d == kGridRows + 1) return {o, o + kGridSide, o + kGridSide};  // </image>
  return {o, o, o};  // the "\n" after </image>
}

}  // namespace cmr
