// Self-test of the bounded waits every pipeline kernel relies on: a wait on
// an mbarrier phase that nothing completes must give up after its limit
// (~1 s), report DEV_TIMEOUT to the host and leave the CUDA context usable.
// The waiting kernel is one warp; it holds no TMEM and issues no copies.
#include "../../include/looped_spec.h"
#include "tc.cuh"

namespace lt {

static __device__ int g_selftest_status;
static __device__ int g_selftest_alive;

__global__ void k_selftest_wait() {
  __shared__ __align__(8) unsigned long long bar;
  const uint32_t b = (uint32_t)__cvta_generic_to_shared(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);  // one arrival completes phase 0; none is made
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    int abort_flag = 0;
    const bool done = mbar_wait(b, 0, &abort_flag);
    g_selftest_status = done ? 0 : DEV_TIMEOUT;
  }
}

__global__ void k_selftest_alive() { g_selftest_alive = 1; }

}  // namespace lt

using namespace lt;

extern "C" int lt_selftest_wait(int32_t* h_out, void* stream) {
  if (!h_out) return LT_ERR_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const int zero = 0;
  cudaEvent_t e0, e1;
  if (cudaMemcpyToSymbolAsync(g_selftest_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) ||
      cudaMemcpyToSymbolAsync(g_selftest_alive, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) ||
      cudaEventCreate(&e0) || cudaEventCreate(&e1))
    return LT_ERR_CUDA;
  cudaEventRecord(e0, st);
  k_selftest_wait<<<1, 32, 0, st>>>();
  cudaEventRecord(e1, st);
  k_selftest_alive<<<1, 1, 0, st>>>();
  int status = -1, alive = 0;
  float ms = 0.f;
  const bool ok = cudaGetLastError() == cudaSuccess &&
                  cudaMemcpyFromSymbolAsync(&status, g_selftest_status, sizeof(int), 0,
                                            cudaMemcpyDeviceToHost, st) == cudaSuccess &&
                  cudaMemcpyFromSymbolAsync(&alive, g_selftest_alive, sizeof(int), 0,
                                            cudaMemcpyDeviceToHost, st) == cudaSuccess &&
                  cudaStreamSynchronize(st) == cudaSuccess &&
                  cudaEventElapsedTime(&ms, e0, e1) == cudaSuccess;
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  if (!ok) return LT_ERR_CUDA;
  h_out[0] = status;
  h_out[1] = alive;
  h_out[2] = (int32_t)ms;
  return LT_OK;
}
