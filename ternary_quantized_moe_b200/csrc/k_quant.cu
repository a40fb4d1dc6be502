// k_quant.cu -- float -> ternary quantizers of groups of 128 weights (absmean, Lloyd).
//
// "Scion: ternary MoE quantization with trained corrections", Findings: the deployable Lloyd
// quantizer beats one-shot absmean on MoE experts; "Scion-35B-A3B" model card, Highlights: the
// deployed quantizer is ternary Lloyd over groups of 128.  Each group of 128 consecutive fp32
// weights gets codes in {-1, 0, +1} and one fp16 scale s (w ~ code * s):
//   absmean: s = mean |w|; code = sign(w) where 2|w| >= s (w / s rounded half away from zero
//            and clamped to [-1, 1]), else 0.
//   Lloyd:   from the absmean codes, alternately s = mean |w| over the nonzero codes (the
//            centroid of the +-s cells) and re-partition to the nearest level by the same rule,
//            until no code changes or `iters` rounds ran; s is the centroid of the final codes.
// One warp per group, four weights per lane; sums and decisions in fp64.  The group sums are
// exact in fp64 whenever the group's nonzero magnitudes span less than 2^29, so the order of
// summation does not change them.
#include <cuda_fp16.h>

#include "scion_internal.cuh"

namespace scion {
namespace {

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int8_t ternary_code(float w, double s) {
  return (w != 0.0f && 2.0 * fabs(double(w)) >= s) ? (w > 0.0f ? 1 : -1) : 0;
}

__global__ void __launch_bounds__(256) quantize_kernel(int method, const float* __restrict__ w, int64_t n_groups,
                                                       int iters, int8_t* __restrict__ codes,
                                                       uint16_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  for (int64_t g = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); g < n_groups; g += warps) {
    const float4 v4 = __ldg(reinterpret_cast<const float4*>(w + g * 128) + lane);
    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
    double s = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i) s += fabs(double(v[i]));
    s = warp_sum_f64(s) / 128.0;
    int8_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = ternary_code(v[i], s);
    if (method == SCION_QUANT_LLOYD) {
      auto centroid = [&]() {
        double sum = 0.0;
        int n = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (c[i]) sum += fabs(double(v[i])), ++n;
        sum = warp_sum_f64(sum);
#pragma unroll
        for (int o = 16; o; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
        return n ? sum / n : 0.0;
      };
      for (int it = 0; it < iters; ++it) {
        s = centroid();
        bool changed = false;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int8_t cn = ternary_code(v[i], s);
          changed |= cn != c[i];
          c[i] = cn;
        }
        if (!__any_sync(0xffffffffu, changed)) break;
      }
      s = centroid();
    }
    char4 out;
    out.x = c[0], out.y = c[1], out.z = c[2], out.w = c[3];
    reinterpret_cast<char4*>(codes + g * 128)[lane] = out;
    if (lane == 0) scales[g] = __half_as_ushort(__double2half(s));
  }
}

}  // namespace
}  // namespace scion

extern "C" int scion_quantize_device(int method, const float* w, int64_t n_groups, int iters, int8_t* codes,
                                     uint16_t* scale_f16, void* stream) {
  if ((method != SCION_QUANT_ABSMEAN && method != SCION_QUANT_LLOYD) || n_groups < 0 || iters < 0 || iters > 1000)
    return SCION_EINVAL;
  if (n_groups == 0) return SCION_OK;
  if (!w || !codes || !scale_f16) return SCION_EINVAL;
  if ((reinterpret_cast<uintptr_t>(w) & 15) || (reinterpret_cast<uintptr_t>(codes) & 3)) return SCION_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t blocks = (n_groups + 7) / 8;
  const unsigned grid = unsigned(blocks < 148 * 16 ? blocks : 148 * 16);
  scion::quantize_kernel<<<grid, 256, 0, s>>>(method, w, n_groups, iters, codes, scale_f16);
  return cudaGetLastError() == cudaSuccess ? SCION_OK : SCION_ECUDA;
}
