// Shared device helpers for the looped-Transformer decoding library (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lt {

// Device error word: the first failure wins (atomicCAS from 0).  The host
// reads it after a step and reports LT_ERR_DEVICE_CHECK / LT_ERR_CAPACITY.
enum DevErr : int {
  DEV_OK = 0,
  DEV_TIMEOUT = 1,        // a bounded wait gave up
  DEV_TABLE_FULL = 2,     // no free branch-table entry
  DEV_SLOTS_FULL = 3,     // no free KV slot
  DEV_BAD_INDEX = 4,      // a slot / token / position out of range
  DEV_NO_ROOT = 5,        // no branch holds the committed prefix
  DEV_CHAIN = 6,          // a branch's uncommitted span exceeds the chain window
  DEV_STATE = 7,          // state machine invariant broken
};

__device__ __forceinline__ void set_err(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// ---- bf16 / f32 element access ---------------------------------------------
template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// ---- block reductions (fixed order: deterministic) --------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Sum over the block; every thread gets the result.  `red` holds >= 33 floats.
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  if (w == 0) {
    float t = lane < nw ? red[lane] : 0.f;
    t = warp_sum(t);
    if (lane == 0) red[32] = t;
  }
  __syncthreads();
  return red[32];
}
__device__ __forceinline__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  if (w == 0) {
    float t = lane < nw ? red[lane] : -INFINITY;
    t = warp_max(t);
    if (lane == 0) red[32] = t;
  }
  __syncthreads();
  return red[32];
}

// ---- Philox-4x32-10 (Salmon et al., SC'11) ------------------------------------
// Counter (c0, c1, c2, c3) = (element index, uid or position, purpose, 0), key
// = (seed lo, seed hi); the first output word is used.
__device__ __forceinline__ uint32_t philox_word0(uint32_t c0, uint32_t c1, uint32_t c2,
                                                 uint32_t c3, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c0, hi0 = __umulhi(0xD2511F53u, c0);
    const uint32_t lo1 = 0xCD9E8D57u * c2, hi1 = __umulhi(0xCD9E8D57u, c2);
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return c0;
}

enum Purpose : uint32_t { P_PROP1 = 1, P_PROP2 = 2, P_ACC1 = 3, P_ACC2 = 4, P_RES = 5, P_AR = 6 };

__device__ __forceinline__ float uniform01(uint64_t seed, uint32_t stream, uint32_t purpose) {
  uint32_t b = philox_word0(0u, stream, purpose, 0u, (uint32_t)seed, (uint32_t)(seed >> 32));
  return (float)(b >> 8) * 5.9604644775390625e-08f;  // * 2^-24, exact
}

// Exponential-race key E_i / w_i of element i (E_i = -ln v_i, v_i in (0,1)).
__device__ __forceinline__ float race_key(uint64_t seed, uint32_t stream, uint32_t purpose,
                                          uint32_t i, float w) {
  uint32_t b = philox_word0(i, stream, purpose, 0u, (uint32_t)seed, (uint32_t)(seed >> 32));
  float v = ((float)(b >> 8) + 0.5f) * 5.9604644775390625e-08f;
  return -logf(v) / w;
}

// ---- stream-K partition shared by the GEMM and its reducers ------------------
// Work units are (tile, k-chunk) pairs linearised tile-major; CTA c of G owns
// units [u0(c), u0(c+1)).  A tile is covered by consecutive CTAs; each CTA
// writes one fp32 partial per tile it touches, at index c * jmax + j where j
// counts the tiles of that CTA.  Reducers sum a tile's partials in CTA order.
__host__ __device__ __forceinline__ int sk_u0(int c, int U, int G) {
  return (int)(((long long)c * U) / G);
}
__host__ __device__ __forceinline__ int sk_cta_of(int u, int U, int G) {
  int c = (int)(((long long)u * G) / U);
  if (c >= G) c = G - 1;
  while (c > 0 && sk_u0(c, U, G) > u) --c;
  while (c + 1 < G && sk_u0(c + 1, U, G) <= u) ++c;
  return c;
}

struct GemmShape {
  int n_out;     // output features (MMA M side, tiled by 128)
  int k;         // reduction length
  int kch;       // stream-K units per tile (groups of kc k-chunks)
  int kc;        // k-chunks (128 bytes of K each) per unit: one TMA request per operand
  int l2_own;    // weight bytes per CTA of its own range requested into L2 beyond the ring
  int l2_next;   // weight bytes per CTA of the next GEMM's slice requested into L2
  int prewait;   // ring stages of weights requested before the dependency wait
  int nch;       // k-chunks per tile, ceil(K / chunk)
  int nfull;     // k-chunks that lie wholly inside K (units within them load as one 3-D box)
  int tiles;     // ceil(n_out / 128)
  int units;     // tiles * kch
  int grid;      // CTAs (<= units)
  int jmax;      // max tiles one CTA touches
  const int* tile_c;   // device [2*tiles]: first and last CTA covering tile t
  const int* cta_t0;   // device [grid]: first tile of CTA c
  const int4* tinfo;   // device [tiles]: (first CTA, last CTA, segment index of the first CTA, 0)
};

// Sum of the partials of output feature n for row i (fixed CTA order).
// Partial layout: part[((c * jmax + j) * ncols + i) * 128 + (n % 128)]: CTA c's
// j-th tile.  A tile's first CTA may have started in an earlier tile (segment
// j_lo); every later CTA of the tile starts in it (segment 0).  One table load,
// then up to 16 partials issued as independent loads: two L2 round trips.
__device__ __forceinline__ float sk_reduce(const float* __restrict__ part, const GemmShape& s,
                                           int ncols, int i, int n) {
  constexpr int PB = 16;
  const int t = n >> 7, r = n & 127;
  const int4 ti = __ldg(s.tinfo + t);
  const size_t row = (size_t)i * 128 + r;
  const size_t cstride = (size_t)s.jmax * ncols * 128;
  float v[PB];
#pragma unroll
  for (int k = 0; k < PB; ++k) {
    const int c = ti.x + k;
    const size_t off = k == 0 ? ((size_t)ti.x * s.jmax + ti.z) * ncols * 128 : (size_t)c * cstride;
    v[k] = c <= ti.y ? __ldcg(part + off + row) : 0.f;
  }
  float acc = 0.f;
#pragma unroll
  for (int k = 0; k < PB; ++k) acc += v[k];
  for (int c = ti.x + PB; c <= ti.y; ++c) acc += __ldcg(part + (size_t)c * cstride + row);
  return acc;
}

// Same sum with the tile's table entry already in hand (loaded ahead of time).
__device__ __forceinline__ float sk_reduce_ti(const float* __restrict__ part, const GemmShape& s,
                                              int4 ti, int ncols, int i, int n) {
  constexpr int PB = 16;
  const int r = n & 127;
  const size_t row = (size_t)i * 128 + r;
  const size_t cstride = (size_t)s.jmax * ncols * 128;
  float v[PB];
#pragma unroll
  for (int k = 0; k < PB; ++k) {
    const int c = ti.x + k;
    const size_t off = k == 0 ? ((size_t)ti.x * s.jmax + ti.z) * ncols * 128 : (size_t)c * cstride;
    v[k] = c <= ti.y ? __ldcg(part + off + row) : 0.f;
  }
  float acc = 0.f;
#pragma unroll
  for (int k = 0; k < PB; ++k) acc += v[k];
  for (int c = ti.x + PB; c <= ti.y; ++c) acc += __ldcg(part + (size_t)c * cstride + row);
  return acc;
}

// Sums of one tile's partials for up to four rows at once (each in fixed CTA
// order): all loads of a round are independent.
template <int PB>
__device__ __forceinline__ void tile_sum4(const float* __restrict__ part, const GemmShape& s,
                                          int4 ti, int ncols, const int* rows4, int nr, int r,
                                          float out[4]) {
  const size_t cstride = (size_t)s.jmax * ncols * 128;
  const size_t base0 = ((size_t)ti.x * s.jmax + ti.z) * ncols * 128 + r;
  float v[4][PB];
#pragma unroll
  for (int k = 0; k < PB; ++k) {
    const int c = ti.x + k;
    const size_t off = k == 0 ? base0 : (size_t)c * cstride + r;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      v[u][k] = (c <= ti.y && u < nr) ? __ldcg(part + off + (size_t)rows4[u] * 128) : 0.f;
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < PB; ++k) acc += v[u][k];
    out[u] = acc;
  }
  for (int c = ti.x + PB; c <= ti.y; ++c)
    for (int u = 0; u < nr; ++u) out[u] += __ldcg(part + (size_t)c * cstride + r + (size_t)rows4[u] * 128);
}

// ---- in-GEMM epilogues --------------------------------------------------------------
// The CTA whose segment completes a group of output tiles (the last to arrive
// on the group's counter) reduces the group's partials in fixed CTA order and
// applies the epilogue, so no separate epilogue kernel is needed.
//
// RMSNorm is applied by its consumers: a GEMM operand row is X = g (.) h
// (unnormalised) and the per-row factor r = 1 / sqrt(mean(h^2) + eps) -- which
// commutes with the matmul -- multiplies the GEMM's reduced output.  Sums of
// squares come as per-128-feature tile parts ssq[t][row], added in tile order.
enum EpiKind : int { EPI_NONE = 0, EPI_RESID = 1, EPI_SWIGLU = 2 };

struct GemmEpi {
  int kind;
  unsigned long long* counters;  // [groups] segment arrivals, monotonic over launches (a
                                // launch's arrivals take a group from k*need to (k+1)*need)
  const int* need;     // [groups] segments that complete a group
  const int* mask;     // [ncols] rows taking part
  // EPI_RESID (group = one tile of h's features):
  //   h[i][n] += scale * y;  X[i][n] = g[n] * h[i][n] (if g);  ssq_out[t][i] = sum_n h[i][n]^2
  float* h;
  float scale;
  const void* g;
  void* X;
  size_t lo;           // lo-plane offset of X (split tf32), 0 otherwise
  float* ssq_out;
  // EPI_SWIGLU (group = gate tile t with up tile t + ffn/128):
  //   X[i][n] = SiLU(r_i * gate) * (r_i * up), r_i from ssq_in
  const float* ssq_in;
  int ssq_tiles;       // tiles of the normalised row (ceil(d / 128))
  float eps;
  int d;               // features of h (RESID) / of the normalised row (SWIGLU)
  int ffn;
};

// 1 / sqrt(mean(h_i^2) + eps) from per-tile sum-of-squares parts (fixed order).
__device__ __forceinline__ float inv_rms_parts(const float* __restrict__ ssq, int tiles,
                                               int ncols, int i, int d, float eps) {
  float s = 0.f;
  for (int t0 = 0; t0 < tiles; t0 += 16) {  // 16 independent loads per round
    float v[16];
#pragma unroll
    for (int k = 0; k < 16; ++k)
      v[k] = t0 + k < tiles ? __ldcg(ssq + (size_t)(t0 + k) * ncols + i) : 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) s += v[k];
  }
  return rsqrtf(s / d + eps);
}

// ---- programmatic dependent launch ---------------------------------------------
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace lt
