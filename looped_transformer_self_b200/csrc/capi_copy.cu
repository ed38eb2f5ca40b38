// Calibration of the copy screen on a committed text (CopyLoop card,
// kongchang.com: copied continuations are scored at a shallow loop depth and
// only those above a threshold from a light calibration go on to the
// full-depth verification).  For every position of the text this computes, on
// the device, the first token the decoder's copy lookup would propose there,
// its depth-d1 screen score and the probability that full depth accepts it;
// the caller picks the threshold from those three arrays.
#include "../../include/looped_spec.h"
#include "readout.cuh"

namespace lt {

// One block of 1024 threads per position t (grid-stride over positions).
//  1. lookup: over end positions e in [k-1, t-1] (each followed by a committed
//     token), the backward match m(e) = #{j = 0, 1, ... : j < cap, j <= e,
//     tok[e-j] == tok[t-j]} up to the first mismatch; the largest m(e) >= k
//     wins, the largest e on ties; the proposal's first token is tok[e+1];
//  2. screen score: softmax of z1 row t at T = 1, at that token (copy_score,
//     the decode step's own screen);
//  3. acceptance of a one-hot draft at full depth: T = 0, whether it is the
//     argmax of zR row t (lowest index on ties); T > 0, its probability under
//     the readout processing of zR row t (readout_dist, in place).
__global__ void __launch_bounds__(1024)
    k_copy_screen(const int* __restrict__ tok, int n, int k, int cap, const float* z1,
                  long long s1, float* zR, long long sR, int V, float T, float top_p,
                  int* __restrict__ out_tok, float* __restrict__ score,
                  float* __restrict__ accept) {
  __shared__ float sk[33];
  __shared__ int si[33];
  __shared__ DistSmem ds;
  for (int t = blockIdx.x; t < n; t += gridDim.x) {
    // 1. the longest, then most recent, earlier match (key m, index t - e)
    float best = -1.f;
    int bi = 0x7fffffff;
    for (int e = k - 1 + (int)threadIdx.x; e <= t - 1; e += blockDim.x) {
      int m = 0;
      while (m < cap && m <= e && tok[e - m] == tok[t - m]) ++m;
      if (m >= k && better_max((float)m, t - e, best, bi)) {
        best = (float)m;
        bi = t - e;
      }
    }
    const int w = block_arg<false>(best, bi, sk, si);
    if (w == 0x7fffffff) {  // no proposal at t
      if (threadIdx.x == 0) {
        out_tok[t] = -1;
        score[t] = -1.f;
        accept[t] = 0.f;
      }
      __syncthreads();
      continue;
    }
    const int s = tok[t - w + 1];
    // 2. screen score at depth d1
    const float* a1 = z1 + (size_t)t * s1;
    float b1 = -INFINITY;
    int i1 = 0x7fffffff;
    for (int j = threadIdx.x; j < V; j += blockDim.x)
      if (better_max(a1[j], j, b1, i1)) {
        b1 = a1[j];
        i1 = j;
      }
    const int arg1 = block_arg<false>(b1, i1, sk, si);
    const float sc = copy_score(a1, V, arg1, s, ds.red);
    // 3. full-depth acceptance of the one-hot draft s
    float* aR = zR + (size_t)t * sR;
    float bR = -INFINITY;
    int iR = 0x7fffffff;
    for (int j = threadIdx.x; j < V; j += blockDim.x)
      if (better_max(aR[j], j, bR, iR)) {
        bR = aR[j];
        iR = j;
      }
    const int argR = block_arg<false>(bR, iR, sk, si);
    float acc;
    if (T == 0.f) {
      acc = argR == s ? 1.f : 0.f;
    } else {
      readout_dist(aR, aR, V, argR, T, top_p, ds);
      __syncthreads();
      acc = aR[s];
    }
    if (threadIdx.x == 0) {
      out_tok[t] = s;
      score[t] = sc;
      accept[t] = acc;
    }
    __syncthreads();  // shared reductions and the rows are reused by the next position
  }
}

}  // namespace lt

using namespace lt;

extern "C" int lt_copy_screen_scores(const int32_t* d_tokens, int n, int k, int match_cap,
                                     const float* d_z1, long long stride1, float* d_zR,
                                     long long strideR, int V, float T, float top_p,
                                     int32_t* d_tok, float* d_score, float* d_accept,
                                     void* stream) {
  if (n < 0 || V <= 0 || k < 1 || match_cap < k || !(T >= 0.f) || !(top_p > 0.f) ||
      top_p > 1.f)
    return LT_ERR_ARG;
  if (n == 0) return LT_OK;
  if (!d_tokens || !d_z1 || !d_zR || !d_tok || !d_score || !d_accept || stride1 < V ||
      strideR < V)
    return LT_ERR_ARG;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = n < 2 * sms ? n : 2 * sms;
  k_copy_screen<<<grid, 1024, 0, (cudaStream_t)stream>>>(d_tokens, n, k, match_cap, d_z1, stride1,
                                                          d_zR, strideR, V, T, top_p, d_tok,
                                                          d_score, d_accept);
  return cudaGetLastError() == cudaSuccess ? LT_OK : LT_ERR_CUDA;
}
