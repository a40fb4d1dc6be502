// k_static.cu -- router logits without any device allocation.
//
// Who needs this: code that cannot call cudaMalloc -- for instance a host runtime
// whose device memory is owned by another allocator, a thread that must not take the
// allocator's locks, or an embedding whose memory budget was fixed in advance.  Such a
// caller still provides x, the router weights and the output, but cannot provide the
// split-K scratch that the router GEMV needs.  This entry point keeps that scratch in a
// file-scope device array that is part of the library image: every GPU that loads the
// library holds it (kStaticScratchBytes + counters) until the process exits.
//
// The computation is the router part of the x-projection kernel: logits[t][e] =
// x_t . W_r[e] + x_t . D[e] in fp32 on the tensor cores (mma.sync bf16), K split over
// 512-column chunks whose partial sums are reduced by the last CTA of each 16-row unit.
#include <mutex>

#include "scion_internal.cuh"

namespace {

constexpr int kMaxTokens = 64;          // tokens per call
constexpr int kMaxExperts = 512;        // router rows
constexpr int kMaxHidden = 4096;        // d
constexpr int kChunk = 512;             // K columns per CTA (4 warps x 128)
constexpr int kMaxUnits = kMaxExperts / 16;
constexpr int kMaxChunks = kMaxHidden / kChunk;
constexpr size_t kPartialFloats = size_t(kMaxUnits) * kMaxChunks * 16 * kMaxTokens;  // 1 MiB of fp32

// The scratch: split-K partial sums, then one arrival counter per 16-row unit.
static __device__ __align__(256) float g_router_scratch[kPartialFloats + kMaxUnits];

std::mutex g_mu;
void* g_scratch_ptr[128];  // per device, resolved once with that device current

__device__ __forceinline__ uint4 ldg_nc(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// One CTA = (16 router rows, one 512-column chunk); NT token tiles of 8.
template <int NT>
__global__ void __launch_bounds__(128) router_static_kernel(const __nv_bfloat16* __restrict__ x, int T, int d, int E,
                                                            const __nv_bfloat16* __restrict__ wr,
                                                            const __nv_bfloat16* __restrict__ wd, float* scratch,
                                                            int n_chunks, float* __restrict__ logits) {
  __shared__ float red[4][NT][32][4];
  __shared__ int last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g8 = lane >> 2, c = lane & 3;
  const int unit = blockIdx.x, chunk = blockIdx.y;
  const int row0 = unit * 16, kw = chunk * kChunk + warp * 128;
  float* partial = scratch;
  unsigned* count = reinterpret_cast<unsigned*>(scratch + kPartialFloats);

  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
  if (kw < d) {
    const int ra = row0 + g8, rb = row0 + g8 + 8;
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const __nv_bfloat16* W = m ? wd : wr;
      uint4 wa[4], wb[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int kk = kw + 32 * q + 8 * c;
        wa[q] = ra < E ? ldg_nc(W + int64_t(ra) * d + kk) : make_uint4(0, 0, 0, 0);
        wb[q] = rb < E ? ldg_nc(W + int64_t(rb) * d + kk) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int tok = nt * 8 + g8;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 xb = tok < T ? *reinterpret_cast<const uint4*>(x + int64_t(tok) * d + kw + 32 * q + 8 * c)
                                   : make_uint4(0, 0, 0, 0);
          const uint32_t fa0[4] = {wa[q].x, wb[q].x, wa[q].y, wb[q].y};
          const uint32_t fa1[4] = {wa[q].z, wb[q].z, wa[q].w, wb[q].w};
          scion::mma_bf16_16816(acc[nt], fa0, xb.x, xb.y);
          scion::mma_bf16_16816(acc[nt], fa1, xb.z, xb.w);
        }
      }
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) red[warp][nt][lane][i] = acc[nt][i];
  __syncthreads();
  float* part = partial + (size_t(unit) * kMaxChunks + chunk) * 16 * kMaxTokens;
  for (int p = threadIdx.x; p < NT * 32; p += blockDim.x) {
    const int nt = p >> 5, ln = p & 31;
    for (int i = 0; i < 4; ++i) {
      const float v = red[0][nt][ln][i] + red[1][nt][ln][i] + red[2][nt][ln][i] + red[3][nt][ln][i];
      const int row = (ln >> 2) + 8 * (i >> 1), tok = nt * 8 + 2 * (ln & 3) + (i & 1);
      part[row * kMaxTokens + tok] = v;
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = (atomicAdd(&count[unit], 1u) == unsigned(n_chunks - 1));
  __syncthreads();
  if (!last) return;
  __threadfence();
  for (int p = threadIdx.x; p < 16 * T; p += blockDim.x) {
    const int row = p / T, tok = p % T;
    if (row0 + row >= E) continue;
    float v = 0.f;
    for (int ch = 0; ch < n_chunks; ++ch)
      v += __ldcg(&partial[(size_t(unit) * kMaxChunks + ch) * 16 * kMaxTokens + row * kMaxTokens + tok]);
    logits[int64_t(tok) * E + row0 + row] = v;
  }
  if (threadIdx.x == 0) count[unit] = 0;
}

// Device address of the scratch array for the current device (looked up once per device).
int scratch_for_current_device(float** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return SCION_ECUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_router_scratch) != cudaSuccess || !p) return SCION_ECUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = static_cast<float*>(g_scratch_ptr[dev]);
  return SCION_OK;
}

}  // namespace

extern "C" int scion_router_logits_static(const void* x, int T, const void* w_router, const void* w_router_delta,
                                          int n_experts, int d, float* logits, void* stream) {
  if (T < 0 || T > kMaxTokens || n_experts < 1 || n_experts > kMaxExperts || d < 128 || d > kMaxHidden || d % 128)
    return SCION_EINVAL;
  if (T == 0) return SCION_OK;
  if (!x || !w_router || !w_router_delta || !logits) return SCION_EINVAL;
  // x and both router matrices are read with 16-byte loads, logits written as fp32
  if (((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(w_router) |
        reinterpret_cast<uintptr_t>(w_router_delta)) & 15) || (reinterpret_cast<uintptr_t>(logits) & 3))
    return SCION_EINVAL;
  float* scratch = nullptr;
  int st = scratch_for_current_device(&scratch);
  if (st != SCION_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the arrival counters must start at zero (a kernel that did not finish could have left them set)
  if (cudaMemsetAsync(scratch + kPartialFloats, 0, sizeof(unsigned) * kMaxUnits, s) != cudaSuccess)
    return SCION_ECUDA;
  const int n_chunks = (d + kChunk - 1) / kChunk;
  dim3 grid((n_experts + 15) / 16, n_chunks);
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  const auto* wr = static_cast<const __nv_bfloat16*>(w_router);
  const auto* wd = static_cast<const __nv_bfloat16*>(w_router_delta);
  const int nt = (T + 7) / 8;
  if (nt == 1)
    router_static_kernel<1><<<grid, 128, 0, s>>>(xb, T, d, n_experts, wr, wd, scratch, n_chunks, logits);
  else if (nt == 2)
    router_static_kernel<2><<<grid, 128, 0, s>>>(xb, T, d, n_experts, wr, wd, scratch, n_chunks, logits);
  else if (nt <= 4)
    router_static_kernel<4><<<grid, 128, 0, s>>>(xb, T, d, n_experts, wr, wd, scratch, n_chunks, logits);
  else
    router_static_kernel<8><<<grid, 128, 0, s>>>(xb, T, d, n_experts, wr, wd, scratch, n_chunks, logits);
  return cudaGetLastError() == cudaSuccess ? SCION_OK : SCION_ECUDA;
}
