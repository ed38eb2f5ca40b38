// Group epilogues of the weight-streaming GEMM, run by the four drain warps
// (128 threads) of a CTA: residual (h += s*y, X = g (.) h, sum-of-squares
// part) and SwiGLU, for a share of the active rows of one tile group.
#pragma once

#include "tc.cuh"

namespace lt {

// ---------------------------------------------------------------------------
// in-GEMM epilogues (run by the 4 drain warps of the CTA completing a group)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void drain_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <typename TX>
__device__ __forceinline__ void store_x(TX* X, size_t idx, float v, size_t lo);
template <>
__device__ __forceinline__ void store_x<__nv_bfloat16>(__nv_bfloat16* X, size_t idx, float v,
                                                       size_t) {
  X[idx] = __float2bfloat16_rn(v);
}
template <>
__device__ __forceinline__ void store_x<float>(float* X, size_t idx, float v, size_t lo) {
  if (lo) {  // split tf32 pair
    const float hi = __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
    X[idx] = hi;
    X[lo + idx] = v - hi;
  } else {
    X[idx] = v;
  }
}
template <typename TX>
__device__ __forceinline__ float load_g(const void* g, int n) {
  return (float)(reinterpret_cast<const TX*>(g)[n]);
}

struct EpiSmem {
  int rows[64];      // active rows of this launch
  int nact;
  int last;          // group completed by this CTA, or -1
  float inv[64];     // per active row: 1 / rms (SwiGLU)
  float wsum[4][64]; // per warp, per active row: partial sum of squares
  int4 ti[8][2];     // per segment of this CTA: table entries of its group's tiles
  unsigned long long target[GEMM_MAX_SEGS];  // per segment: arrival count completing its group
  int ok;            // thread 0's last continue / stop decision, shared with the drain warps
  int okb[2];        // the same for the segment loop (alternating slots)
};

// Residual epilogue of one tile for active rows r0 .. r1-1 (indices into
// sm.rows): h += scale * y; X = g (.) h; sum-of-squares part of those rows.
template <typename TX>
__device__ void epi_resid(const GemmEpi& ep, const float* __restrict__ part, const GemmShape& s,
                          int ncols, int t, int4 ti, int r0, int r1, int et, EpiSmem& sm) {
  const int n = t * 128 + et;
  const bool valid = n < s.n_out;
  const int lane = et & 31, w = et >> 5;
  for (int k0 = r0; k0 < r1; k0 += 4) {
    const int nr = min(4, r1 - k0);
    float y[4], h0[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)  // h rows first: their loads overlap the partials'
      h0[u] = (valid && u < nr) ? __ldcg(ep.h + (size_t)sm.rows[k0 + u] * ep.d + n) : 0.f;
    tile_sum4<12>(part, s, ti, ncols, sm.rows + k0, nr, n & 127, y);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (u >= nr) break;
      const int i = sm.rows[k0 + u];
      float hv = 0.f;
      if (valid) {
        hv = h0[u] + ep.scale * y[u];
        ep.h[(size_t)i * ep.d + n] = hv;
        if (ep.g)
          store_x<TX>(reinterpret_cast<TX*>(ep.X), (size_t)i * ep.d + n, load_g<TX>(ep.g, n) * hv,
                      ep.lo);
      }
      float sq = hv * hv;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
      if (lane == 0) sm.wsum[w][k0 + u] = sq;
    }
  }
  drain_sync();
  if (et >= r0 && et < r1) {
    const float v = sm.wsum[0][et] + sm.wsum[1][et] + sm.wsum[2][et] + sm.wsum[3][et];
    ep.ssq_out[(size_t)t * ncols + sm.rows[et]] = v;
  }
}

// SwiGLU epilogue of one (gate tile g, up tile g + ffn/128) pair for active
// rows r0 .. r1-1; sm.inv was filled during the mainloop.
template <typename TX>
__device__ void epi_swiglu(const GemmEpi& ep, const float* __restrict__ part, const GemmShape& s,
                           int ncols, int g, int4 tg, int4 tu, int r0, int r1, int et,
                           EpiSmem& sm) {
  const int n = g * 128 + et;
  if (n >= ep.ffn) return;
  for (int k0 = r0; k0 < r1; k0 += 4) {
    const int nr = min(4, r1 - k0);
    float gv[4], uv[4];
    tile_sum4<4>(part, s, tg, ncols, sm.rows + k0, nr, n & 127, gv);
    tile_sum4<4>(part, s, tu, ncols, sm.rows + k0, nr, n & 127, uv);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (u >= nr) break;
      const float r = sm.inv[k0 + u];
      const float g = r * gv[u], up = r * uv[u];
      store_x<TX>(reinterpret_cast<TX*>(ep.X), (size_t)sm.rows[k0 + u] * ep.ffn + n,
                  g / (1.f + __expf(-g)) * up, ep.lo);
    }
  }
}


}  // namespace lt
