// topk_warp.cuh -- top-k gating for one token by one warp (logits held in registers).
//
// The k largest router logits ("Scion-35B-A3B" model card, Model Overview: top-8 of 256;
// "Scion-FlashNext-176B-A6B", Model Overview: top-10 of 512), ties to the lower expert id,
// then the gates: softmax over the selected logits (norm_topk = 1) or the selected entries
// of a softmax over all E logits (norm_topk = 0).  VPL = logits per lane (E <= 32 * VPL).
#pragma once

#include <float.h>
#include <math.h>

namespace scion {

template <int VPL>
__device__ __forceinline__ void warp_topk(const float* __restrict__ row, int E, int k, int norm_topk, int lane,
                                          int32_t* __restrict__ ids_out, float* __restrict__ gates_out) {
  float v[VPL];
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    float x = e < E ? row[e] : -INFINITY;
    if (e < E && !(x >= -FLT_MAX)) x = -FLT_MAX;  // NaN / -inf rank below every finite logit
    v[i] = x;
    mx = fmaxf(mx, x);
  }
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float zall = 0.f;
  if (!norm_topk) {
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if (lane + 32 * i < E) zall += expf(v[i] - mx);
    for (int o = 16; o; o >>= 1) zall += __shfl_xor_sync(0xffffffffu, zall, o);
  }
  static_assert(VPL <= 64, "at most 2048 experts");
  // Order-preserving 32-bit keys of the logits (larger logit <-> larger key; -0 is taken as +0,
  // so equal logits stay ties); entries past E get key 0, below every logit's key (-FLT_MAX maps
  // to 0x00800000).
  uint32_t key[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const uint32_t b = v[i] == 0.f ? 0u : __float_as_uint(v[i]);
    key[i] = lane + 32 * i < E ? ((b >> 31) ? ~b : (b | 0x80000000u)) : 0u;
  }
  // Each lane keeps its L best entries in (key descending, slot ascending) order: the slot order
  // is the id order inside a lane, so strict comparisons in ascending slot order keep ties on the
  // lower id.  A lane whose list runs dry refills it from the entries after the last one taken.
  constexpr int L = VPL < 4 ? VPL : 4;
  uint32_t lk[L];
  int ls[L];
  auto fill = [&](uint32_t after_key, int after_slot) {
#pragma unroll
    for (int j = 0; j < L; ++j) lk[j] = 0u, ls[j] = VPL;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const uint32_t x = key[i];
      if (x == 0u || x > after_key || (x == after_key && i <= after_slot)) continue;
      bool c[L];
#pragma unroll
      for (int j = 0; j < L; ++j) c[j] = x > lk[j];
#pragma unroll
      for (int j = L - 1; j > 0; --j) {
        lk[j] = c[j - 1] ? lk[j - 1] : (c[j] ? x : lk[j]);
        ls[j] = c[j - 1] ? ls[j - 1] : (c[j] ? i : ls[j]);
      }
      if (c[0]) lk[0] = x, ls[0] = i;
    }
  };
  fill(0xffffffffu, -1);
  float my_v = -INFINITY;
  int my_id = -1;
  for (int j = 0; j < k; ++j) {
    // the best head of the warp, then the lowest id among the lanes holding that key
    const uint32_t m = __reduce_max_sync(0xffffffffu, lk[0]);
    const unsigned cand = lk[0] == m ? unsigned(lane + 32 * ls[0]) : 0xffffffffu;
    const int bi = int(__reduce_min_sync(0xffffffffu, cand));
    if (lane == j) my_v = __uint_as_float((m >> 31) ? (m & 0x7fffffffu) : ~m), my_id = bi;
    if ((bi & 31) == lane) {
      const uint32_t tk = lk[0];
      const int ts = ls[0];
#pragma unroll
      for (int q = 0; q + 1 < L; ++q) lk[q] = lk[q + 1], ls[q] = ls[q + 1];
      lk[L - 1] = 0u, ls[L - 1] = VPL;
      if (lk[0] == 0u) fill(tk, ts);
    }
  }
  const float top = __shfl_sync(0xffffffffu, my_v, 0);
  float ex = 0.f;
  if (lane < k) ex = norm_topk ? expf(my_v - top) : expf(my_v - mx);
  float z = ex;
  for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  if (!norm_topk) z = zall;
  if (lane < k) {
    ids_out[lane] = my_id;
    gates_out[lane] = ex / z;
  }
}

}  // namespace scion
