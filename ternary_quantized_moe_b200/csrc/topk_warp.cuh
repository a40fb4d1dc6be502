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
  float my_v = -INFINITY;
  int my_id = -1;
  if constexpr (VPL <= 16) {
    // each lane sorts its values (descending, lower id first on ties) ...
    int id[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      id[i] = lane + 32 * i;
      if (id[i] >= E) v[i] = -INFINITY, id[i] = 0x7fffffff;
    }
#pragma unroll
    for (int r = 0; r < VPL; ++r)
#pragma unroll
      for (int i = r & 1; i + 1 < VPL; i += 2)
        if (v[i + 1] > v[i] || (v[i + 1] == v[i] && id[i + 1] < id[i])) {
          const float tv = v[i];
          const int ti = id[i];
          v[i] = v[i + 1], id[i] = id[i + 1], v[i + 1] = tv, id[i + 1] = ti;
        }
    // ... then every round the warp takes the best lane head and that lane pops it
    for (int j = 0; j < k; ++j) {
      float bv = v[0];
      int bi = id[0];
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        const float v2 = __shfl_xor_sync(0xffffffffu, bv, o);
        const int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
        if (v2 > bv || (v2 == bv && i2 < bi)) bv = v2, bi = i2;
      }
      if (lane == j) my_v = bv, my_id = bi;
      if ((bi & 31) == lane) {
#pragma unroll
        for (int i = 0; i + 1 < VPL; ++i) v[i] = v[i + 1], id[i] = id[i + 1];
        v[VPL - 1] = -INFINITY, id[VPL - 1] = 0x7fffffff;
      }
    }
  } else {
    // many logits per lane: each round scans the lane's untaken entries
    unsigned long long taken = 0;
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !((taken >> i) & 1ull) && (bi == 0x7fffffff || v[i] > bv)) bv = v[i], bi = e;
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        const float v2 = __shfl_xor_sync(0xffffffffu, bv, o);
        const int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
        if (v2 > bv || (v2 == bv && i2 < bi)) bv = v2, bi = i2;
      }
      if (lane == j) my_v = bv, my_id = bi;
      if ((bi & 31) == lane) taken |= 1ull << (bi >> 5);
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
