// tc_order.cuh -- column orders of the tensor-core (tcgen05) path.
//
// The expansion of a 128-column code group into tensor memory produces its fp16 values in a
// per-format order of positions; the B operand rows (x for gate/up, the hidden h for down)
// are stored in the same order, so that position p of A meets position p of B:
//   PQ2_0 : inside every 16 columns, position 2s+h holds column s + 8h (s < 8, h < 2)
//   PTQ1_0: each 64-column half of a 128-column group is self-contained: quintets 12h..12h+11
//           in pairs, then remainder trits 4h..4h+3 (see perm_pos).
#pragma once

#include "scion_internal.cuh"

namespace scion {
namespace {

__device__ __forceinline__ int perm_pos(int fmt, int col) {  // physical column -> position
  if (fmt == SCION_PQ2_0) {
    int c16 = col & 15;
    return (col & ~15) | (2 * (c16 & 7) + (c16 >> 3));
  }
  // PTQ1_0: half h of the group (positions 64h .. 64h+63) holds quintets 12h .. 12h+11 as
  // pairs (2i, 2i+1) -- position 10i + 2j + u <-> column 5(12h + 2i + u) + j -- and then
  // remainder trits 4h .. 4h+3 (columns 120 + 4h ..) in natural order.
  const int g = col & ~127, k = col & 127;
  if (k >= 120) return g | (64 * ((k - 120) >> 2) + 60 + ((k - 120) & 3));
  const int q = k / 5, j = k % 5, half = q / 12, i = (q % 12) >> 1, u = q & 1;
  return g | (64 * half + 10 * i + 2 * j + u);
}

// PQ2_0 B-operand factor of position p for the tensor-core decode: positions (2s, 2s+1) of
// every 16 hold the pair of columns (s, s + 8) that its subnormal expansion builds with the field
// at bits 2f..2f+1 of a 16-bit code half (f = s < 5 ? s : s - 5), i.e. scaled by 4^f; its B
// operands (x and h) carry 4^-f, an exact power-of-two scaling.  The prefill expansion shifts
// each field down first and needs no factor.
__device__ __forceinline__ float pq2_pos_scale(int p) {
  const int s = (p & 15) >> 1;
  return 1.0f / float(1 << (2 * (s < 5 ? s : s - 5)));
}

// Column held by position p of a 128-column group (the inverse of perm_pos).
__device__ __forceinline__ int pos_col(int fmt, int p) {
  if (fmt == SCION_PQ2_0) return (p & ~15) | (((p & 15) >> 1) + 8 * (p & 1));
  const int half = p >> 6, r = p & 63;
  if (r >= 60) return 120 + 4 * half + (r - 60);
  const int i = r / 10, rem = r % 10;
  return 5 * (12 * half + 2 * i + (rem & 1)) + (rem >> 1);
}

}  // namespace
}  // namespace scion
