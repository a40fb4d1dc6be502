// k_selftest.cu -- the bounded-wait failure path, exercised without a GPU fault.
//
// Every wait of the tensor-core and ring kernels goes through mbar_wait: a try_wait loop with
// a time limit after which the waiting thread raises the CTA's abort flag, writes SCION_ETIMEOUT
// into the device status word and returns false, so that every role unwinds and the context
// stays usable.  This kernel waits on a barrier phase that nothing completes, with a short
// limit, and a second warp waits on another such phase with a longer one: the first gives up
// on its own clock, the second on the abort flag.
#include "tc_common.cuh"

namespace scion {
namespace {

using namespace tc;

__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns, int* status, unsigned long long* elapsed_ns) {
  __shared__ uint64_t never0, never1;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&never0, 1);
    mbar_init(&never1, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const uint64_t t0 = globaltimer();
  bool ok = true;
  if (threadIdx.x == 0) ok = mbar_wait(&never0, 0, &abort_flag, status, limit_ns);
  if (threadIdx.x == 32) ok = mbar_wait(&never1, 0, &abort_flag, nullptr, 10 * limit_ns);
  __syncthreads();
  if (threadIdx.x == 0) status[1] = ok, *elapsed_ns = globaltimer() - t0;
  if (threadIdx.x == 32) status[2] = ok;
}

}  // namespace
}  // namespace scion

extern "C" int scion_selftest_bounded_wait(int limit_us, int* result, double* elapsed_ms, void* stream) {
  if (limit_us < 1 || limit_us > 1000000 || !result || !elapsed_ms) return SCION_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = nullptr;
  unsigned long long* el = nullptr;
  int st = SCION_OK;
  if (cudaMalloc(&status, 3 * sizeof(int)) != cudaSuccess || cudaMalloc(&el, sizeof(unsigned long long)) != cudaSuccess) {
    st = SCION_ENOMEM;
  } else {
    unsigned long long el_host = 0;
    cudaError_t e = cudaMemsetAsync(status, 0, 3 * sizeof(int), s);
    if (e == cudaSuccess) {
      scion::bounded_wait_selftest_kernel<<<1, 64, 0, s>>>(uint64_t(limit_us) * 1000ull, status, el);
      e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaMemcpyAsync(result, status, 3 * sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(&el_host, el, sizeof(el_host), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) st = SCION_ECUDA;
    *elapsed_ms = double(el_host) * 1e-6;
  }
  if (status) cudaFree(status);
  if (el) cudaFree(el);
  return st;
}
