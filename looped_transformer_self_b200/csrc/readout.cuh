// Block-wide helpers and the readout processing shared by the decode step's
// readouts (decide.cuh) and the depth-wise total-variation measurement
// (capi_tv.cu).
//
// Readout processing follows "LoopSpec: Pipelined Self-Speculative Decoding
// for Looped Transformers" (liuzhao09.github.io/papers/loopspec.html),
// section 2.1: temperature, optional top-p truncation, normalisation, the
// same at every depth.  Reading where the page is silent: top-p keeps every
// token with p >= theta*, theta* the largest probability value whose upper set
// holds >= top_p of the mass (ties at the boundary are kept).
#pragma once

#include "common.cuh"

namespace lt {

// ---------------------------------------------------------------------------
// block helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool better_min(float k, int i, float bk, int bi) {
  return k < bk || (k == bk && i < bi);
}
__device__ __forceinline__ bool better_max(float k, int i, float bk, int bi) {
  return k > bk || (k == bk && i < bi);
}

// Block-wide arg-min (MIN=true) or arg-max of (key, index), lowest index on ties.
template <bool MIN>
__device__ __forceinline__ int block_arg(float k, int idx, float* sk, int* si) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float k2 = __shfl_xor_sync(0xffffffffu, k, o);
    const int i2 = __shfl_xor_sync(0xffffffffu, idx, o);
    if (MIN ? better_min(k2, i2, k, idx) : better_max(k2, i2, k, idx)) {
      k = k2;
      idx = i2;
    }
  }
  __syncthreads();
  if (lane == 0) {
    sk[w] = k;
    si[w] = idx;
  }
  __syncthreads();
  if (w == 0) {
    k = lane < nw ? sk[lane] : (MIN ? INFINITY : -INFINITY);
    idx = lane < nw ? si[lane] : 0x7fffffff;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float k2 = __shfl_xor_sync(0xffffffffu, k, o);
      const int i2 = __shfl_xor_sync(0xffffffffu, idx, o);
      if (MIN ? better_min(k2, i2, k, idx) : better_max(k2, i2, k, idx)) {
        k = k2;
        idx = i2;
      }
    }
    if (lane == 0) si[32] = idx;
  }
  __syncthreads();
  return si[32];
}

// Inclusive suffix sums of 1024 u64 bins held one per thread (blockDim 1024).
__device__ __forceinline__ unsigned long long suffix_scan_1024(unsigned long long v,
                                                              unsigned long long* wsum) {
  // prefix scan over reversed order: thread t holds bin 1023 - t
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  __syncthreads();
  if (lane == 31) wsum[w] = v;
  __syncthreads();
  if (w == 0) {
    unsigned long long s = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long t = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += t;
    }
    wsum[lane] = s;
  }
  __syncthreads();
  return v + (w > 0 ? wsum[w - 1] : 0ull);
}


// Shared memory of readout_dist.
struct DistSmem {
  float red[33];
  unsigned long long hist[1024];
  unsigned long long wsum[32];
  int sel[2];
  unsigned long long sel_above;
};

// p = top-p(softmax(z / T)) of one readout row (one block of 1024 threads).
// a: the row's argmax (block_arg), so exp never overflows.  p may alias z.
// The top-p threshold is an exact 3-level radix select over the float bits of
// p with integer (2^-40) mass, so the sums do not depend on thread order.
__device__ __forceinline__ void readout_dist(const float* z, float* p, int V, int a, float T,
                                             float top_p, DistSmem& sm) {
  const float zmax = z[a];
  __syncthreads();  // every thread holds zmax before p (possibly z) is written
  const float invT = 1.f / T;
  float ssum = 0.f;
  for (int j = threadIdx.x; j < V; j += blockDim.x) {
    const float e = expf((z[j] - zmax) * invT);
    p[j] = e;
    ssum += e;
  }
  const float Z = block_sum(ssum, sm.red);
  const float invZ = 1.f / Z;
  if (!(top_p < 1.f)) {
    for (int j = threadIdx.x; j < V; j += blockDim.x) p[j] *= invZ;
    return;
  }
  const double SCALE = 1099511627776.0;  // 2^40
  const unsigned long long target = (unsigned long long)((double)top_p * SCALE + 0.5);
  unsigned long long above = 0ull;
  uint32_t prefix = 0u;
  const int shifts[3] = {20, 10, 0};
  bool all = false;
  for (int lvl = 0; lvl < 3; ++lvl) {
    sm.hist[threadIdx.x] = 0ull;
    __syncthreads();
    const int sh = shifts[lvl];
    for (int j = threadIdx.x; j < V; j += blockDim.x) {
      const float pj = (lvl == 0) ? p[j] * invZ : p[j];
      if (lvl == 0) p[j] = pj;
      const uint32_t b = __float_as_uint(pj);
      if (lvl == 0 || (b >> (sh + 10)) == prefix) {
        const unsigned long long m = (unsigned long long)((double)pj * SCALE + 0.5);
        atomicAdd(&sm.hist[(b >> sh) & 1023u], m);
      }
    }
    __syncthreads();
    const int bin = 1023 - threadIdx.x;
    const unsigned long long hv = sm.hist[bin];
    const unsigned long long cum = suffix_scan_1024(hv, sm.wsum);  // mass of bins >= bin
    if (threadIdx.x == 0) sm.sel[0] = -1;
    __syncthreads();
    if (above + cum >= target && above + cum - hv < target) {
      sm.sel[0] = bin;
      sm.sel_above = above + cum - hv;
    }
    __syncthreads();
    if (sm.sel[0] < 0) {
      all = true;
      break;
    }
    above = sm.sel_above;
    prefix = (prefix << 10) | (uint32_t)sm.sel[0];
    __syncthreads();
  }
  const uint32_t theta = all ? 0u : prefix;
  float ks = 0.f;
  for (int j = threadIdx.x; j < V; j += blockDim.x) {
    const float pj = p[j];
    if (__float_as_uint(pj) >= theta) ks += pj;
  }
  const float Z2 = block_sum(ks, sm.red);
  const float inv2 = 1.f / Z2;
  for (int j = threadIdx.x; j < V; j += blockDim.x) {
    const float pj = p[j];
    p[j] = __float_as_uint(pj) >= theta ? pj * inv2 : 0.f;
  }
}

// Screen score of a copied token s (CopyLoop card: copied continuations are
// scored at a shallow depth): softmax of the row's logits at T = 1, taken at
// s.  a: the row's argmax.  One block; `red` holds >= 33 floats.  The decode
// step's screen and the calibration call both use this.
__device__ __forceinline__ float copy_score(const float* __restrict__ z, int V, int a, int s,
                                            float* red) {
  const float zmax = z[a];
  float acc = 0.f;
  for (int j = threadIdx.x; j < V; j += blockDim.x) acc += expf(z[j] - zmax);
  const float Z = block_sum(acc, red);
  return expf(z[s] - zmax) / Z;
}

}  // namespace lt
