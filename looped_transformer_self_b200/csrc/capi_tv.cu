// Total variation between two readouts of the same positions, for depth
// selection (LoopSpec page, section 2.4, Eq. 7: the mean TV(p_r, p_R) over
// positions bounds the rejection rate of a depth-r draft; section 3.1, Fig. 3
// measures it at T = 1, top-p 0.7, and the share of positions whose argmax
// agrees at T = 0).
#include "../../include/looped_spec.h"
#include "readout.cuh"

namespace lt {

// One block of 1024 threads per row (grid-stride over rows).  Both rows are
// turned in place into their readout distributions with the decode step's own
// processing (readout_dist), then tv[i] = 1/2 sum_j |p_a(j) - p_b(j)|.  At
// T = 0 the readouts are one-hot at the argmax (lowest index on ties) and
// tv[i] is 1 where the two argmaxes differ, else 0; the rows are left as they
// are.
__global__ void __launch_bounds__(1024)
    k_readout_tv(float* za, long long sa, float* zb, long long sb, int n,
                 int V, float T, float top_p, float* __restrict__ tv) {
  __shared__ float sk[33];
  __shared__ int si[33];
  __shared__ DistSmem ds;
  for (int i = blockIdx.x; i < n; i += gridDim.x) {
    float* a = za + (size_t)i * sa;
    float* b = zb + (size_t)i * sb;
    int arg[2];
    for (int k = 0; k < 2; ++k) {
      const float* z = k ? b : a;
      float best = -INFINITY;
      int bi = 0x7fffffff;
      for (int j = threadIdx.x; j < V; j += blockDim.x) {
        const float v = z[j];
        if (better_max(v, j, best, bi)) {
          best = v;
          bi = j;
        }
      }
      arg[k] = block_arg<false>(best, bi, sk, si);
    }
    if (T == 0.f) {
      if (threadIdx.x == 0) tv[i] = arg[0] != arg[1] ? 1.f : 0.f;
      continue;
    }
    readout_dist(a, a, V, arg[0], T, top_p, ds);
    readout_dist(b, b, V, arg[1], T, top_p, ds);
    float s = 0.f;
    for (int j = threadIdx.x; j < V; j += blockDim.x) s += fabsf(a[j] - b[j]);
    const float t = block_sum(s, ds.red);
    if (threadIdx.x == 0) tv[i] = 0.5f * t;
    __syncthreads();  // ds and the rows are reused by the next row
  }
}

}  // namespace lt

using namespace lt;

extern "C" int lt_readout_tv(float* d_za, long long stride_a, float* d_zb, long long stride_b,
                             int n, int V, float T, float top_p, float* d_tv, void* stream) {
  if (n < 0 || V <= 0 || !(T >= 0.f) || !(top_p > 0.f)) return LT_ERR_ARG;
  if (n == 0) return LT_OK;
  if (!d_za || !d_zb || !d_tv || stride_a < V || stride_b < V) return LT_ERR_ARG;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = n < 2 * sms ? n : 2 * sms;
  k_readout_tv<<<grid, 1024, 0, (cudaStream_t)stream>>>(d_za, stride_a, d_zb, stride_b, n, V, T,
                                                         top_p, d_tv);
  return cudaGetLastError() == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}
