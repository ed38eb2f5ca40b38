// Per-layer kernels of the batched mixed-depth pass (CUDA cores, HBM/L2-bound).
//
// One decode step runs every shared-block layer once over all active rows;
// each row sits at its own loop depth and reads/writes only the KV cache of
// that depth ("LoopSpec", liuzhao09.github.io/papers/loopspec.html, section
// 2.1 and Fig. 2: shared weights, but states and KV of different depths are
// never mixed).  Layer (a reading; the pages give only Eq. 1): pre-norm,
// RMSNorm -> QKV -> RoPE -> causal attention -> O (+ s * residual) -> RMSNorm ->
// SwiGLU MLP (+ s * residual).
//
// Row bookkeeping arrays (length C = table capacity = GEMM columns):
//   mask[i]     row takes part in this pass (else its columns are zero and its
//               hidden state and caches are untouched)
//   r_pos[i]    position of the row's token; r_slot[i] its KV slot
//   tag[i]      cache plane of the row within the layer (loop depth - 1 for
//               shared-block layers, readout index for coda layers, 0 for prelude)
//   slot of position j < r_pos[i]:  j < r_blen[i] ? lists[r_boff[i] + j]
//                                   : chain[i * W + j % W]
// KV pool: kv[((plane * S + slot) * 2 + {0: K, 1: V}) * d + feature].
#pragma once

#include "common.cuh"

namespace lt {

constexpr int ATT_CH = 128;       // positions per attention split (fixed: batch invariant)
constexpr int EPI_THREADS = 1024;  // epilogues: many partial reductions in flight per row

// Writes a GEMM operand element.  bf16: rounded.  fp32 with lo != 0: the value
// is stored as a tf32 pair, hi (low 13 mantissa bits cleared) at X[i] and the
// exact remainder at X[lo + i], for the split-tf32 tensor-core GEMM.
template <typename T>
__device__ __forceinline__ void store_act(T* X, size_t i, float v, size_t lo);
template <>
__device__ __forceinline__ void store_act<__nv_bfloat16>(__nv_bfloat16* X, size_t i, float v,
                                                         size_t) {
  X[i] = __float2bfloat16_rn(v);
}
template <>
__device__ __forceinline__ void store_act<float>(float* X, size_t i, float v, size_t lo) {
  if (lo) {
    const float h = __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
    X[i] = h;
    X[lo + i] = v - h;
  } else {
    X[i] = v;
  }
}

template <typename T>
__device__ __forceinline__ size_t kv_off(int plane, int slot, int which, int S, int d) {
  return (((size_t)plane * S + slot) * 2 + which) * (size_t)d;
}

// ---- embedding: H^(0) of new rows (prelude P starts from the token's embedding)
template <typename T>
__global__ void k_embed(const T* __restrict__ E, const int* __restrict__ tok,
                        const int* __restrict__ mask, int d, int V, float* __restrict__ h,
                        int* err) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x;
  if (!mask[i]) return;
  const int t = tok[i];
  if (t < 0 || t >= V) {
    if (threadIdx.x == 0) set_err(err, DEV_BAD_INDEX);
    return;
  }
  for (int n = threadIdx.x; n < d; n += blockDim.x)
    h[(size_t)i * d + n] = to_f<T>(E[(size_t)t * d + n]);
}

// ---- GEMM operand X = g (.) h for masked rows, plus the per-128-feature tile
// parts of sum(h^2) that the consumers turn into the RMSNorm factor -------------
// (RMSNorm's per-row factor commutes with the matmul, so the GEMM consumers
// apply it; masked rows keep whatever X held -- their columns are ignored.)
template <typename T>
__global__ void k_stage_norm(const float* __restrict__ h, const int* __restrict__ mask,
                             const T* __restrict__ g, int d, int C, T* __restrict__ X, size_t lo,
                             float* __restrict__ ssq) {
  __shared__ float wsum[32];
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x;
  if (!mask[i]) return;
  const float* hr = h + (size_t)i * d;
  T* xr = X + (size_t)i * d;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int base = 0; base < d; base += blockDim.x) {
    const int n = base + threadIdx.x;
    float sq = 0.f;
    if (n < d) {
      const float v = hr[n];
      store_act<T>(xr, n, to_f<T>(g[n]) * v, lo);
      sq = v * v;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (lane == 0) wsum[w] = sq;
    __syncthreads();
    if (threadIdx.x < blockDim.x / 128) {
      const int t = base / 128 + threadIdx.x;
      if (t * 128 < d) {
        const int w0 = 4 * threadIdx.x;
        ssq[(size_t)t * C + i] = wsum[w0] + wsum[w0 + 1] + wsum[w0 + 2] + wsum[w0 + 3];
      }
    }
    __syncthreads();
  }
}

template <typename T>
__global__ void k_copy_rows(const float* __restrict__ src, const int* __restrict__ mask, int d,
                            float* __restrict__ dst) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x;
  if (!mask[i]) return;
  for (int n = threadIdx.x; n < d; n += blockDim.x) dst[(size_t)i * d + n] = src[(size_t)i * d + n];
}

// ---- QKV epilogue: reduce partials, RoPE(q, k), scatter K/V to the row's plane --
template <typename T>
__global__ void k_qkv_epi(const float* __restrict__ part, const GemmShape s, int C,
                          const int* __restrict__ mask, const int* __restrict__ r_pos,
                          const int* __restrict__ r_slot, const int* __restrict__ tagsrc,
                          int tag_off, int plane_base, int S, int d, int hd,
                          const float2* __restrict__ rope, T* __restrict__ kv,
                          float* __restrict__ q, const float* __restrict__ ssq, int ssq_tiles,
                          float eps, int* err) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x;
  if (!mask[i]) return;
  const float r = inv_rms_parts(ssq, ssq_tiles, C, i, d, eps);
  const int pos = r_pos[i], slot = r_slot[i];
  const int tag = (tagsrc ? tagsrc[i] : 0) + tag_off;
  if (slot < 0 || slot >= S) {
    if (threadIdx.x == 0) set_err(err, DEV_BAD_INDEX);
    return;
  }
  const int plane = plane_base + tag;
  T* krow = kv + kv_off<T>(plane, slot, 0, S, d);
  T* vrow = kv + kv_off<T>(plane, slot, 1, S, d);
  const int half = hd / 2;
  for (int p = threadIdx.x; p < d / 2; p += blockDim.x) {
    const int head = p / half, e = p - head * half;
    const int n1 = head * hd + e, n2 = n1 + half;
    const float2 cs = rope[(size_t)pos * half + e];
    const float q1 = r * sk_reduce(part, s, C, i, n1), q2 = r * sk_reduce(part, s, C, i, n2);
    q[(size_t)i * d + n1] = q1 * cs.x - q2 * cs.y;
    q[(size_t)i * d + n2] = q2 * cs.x + q1 * cs.y;
    const float k1 = r * sk_reduce(part, s, C, i, d + n1);
    const float k2 = r * sk_reduce(part, s, C, i, d + n2);
    krow[n1] = from_f<T>(k1 * cs.x - k2 * cs.y);
    krow[n2] = from_f<T>(k2 * cs.x + k1 * cs.y);
  }
  for (int n = threadIdx.x; n < d; n += blockDim.x)
    vrow[n] = from_f<T>(r * sk_reduce(part, s, C, i, 2 * d + n));
}

// ---- vector loads of EPL consecutive cache elements ------------------------------
// Loads go through L2 (ld.global.cg): a fused attention block may read back a
// cache row it wrote itself, which the non-coherent read-only path would not see.
template <typename T, int EPL>
__device__ __forceinline__ void load_vec(const T* __restrict__ p, float* out) {
  constexpr int BYTES = EPL * (int)sizeof(T);
  if constexpr (sizeof(T) == 2) {
    if constexpr (BYTES % 16 == 0) {
#pragma unroll
      for (int c = 0; c < BYTES / 16; ++c) {
        uint4 u = __ldcg(reinterpret_cast<const uint4*>(p) + c);
        const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float2 f = __bfloat1622float2(b[j]);
          out[c * 8 + 2 * j] = f.x;
          out[c * 8 + 2 * j + 1] = f.y;
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < BYTES / 4; ++c) {
        uint32_t u = __ldcg(reinterpret_cast<const unsigned int*>(p) + c);
        float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
        out[2 * c] = f.x;
        out[2 * c + 1] = f.y;
      }
    }
  } else {
    if constexpr (BYTES % 16 == 0) {
#pragma unroll
      for (int c = 0; c < BYTES / 16; ++c) {
        float4 f = __ldcg(reinterpret_cast<const float4*>(p) + c);
        out[4 * c] = f.x;
        out[4 * c + 1] = f.y;
        out[4 * c + 2] = f.z;
        out[4 * c + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int c = 0; c < BYTES / 8; ++c) {
        float2 f = __ldcg(reinterpret_cast<const float2*>(p) + c);
        out[2 * c] = f.x;
        out[2 * c + 1] = f.y;
      }
    }
  }
}

// ---- raw cache words: loaded now, converted when used (keeps 8 positions of K
// and V in flight per lane without 128 float registers) -----------------------------
template <typename T, int EPL>
struct RawVec {
  static constexpr int BYTES = EPL * (int)sizeof(T);
  static constexpr int WORDS = BYTES / 4;
  uint32_t w[WORDS];
  __device__ __forceinline__ void load(const T* p) {
    if constexpr (BYTES % 16 == 0) {
#pragma unroll
      for (int c = 0; c < BYTES / 16; ++c) {
        const uint4 u = __ldcg(reinterpret_cast<const uint4*>(p) + c);
        w[4 * c] = u.x;
        w[4 * c + 1] = u.y;
        w[4 * c + 2] = u.z;
        w[4 * c + 3] = u.w;
      }
    } else if constexpr (BYTES % 8 == 0) {
#pragma unroll
      for (int c = 0; c < BYTES / 8; ++c) {
        const uint2 u = __ldcg(reinterpret_cast<const uint2*>(p) + c);
        w[2 * c] = u.x;
        w[2 * c + 1] = u.y;
      }
    } else {
#pragma unroll
      for (int c = 0; c < WORDS; ++c) w[c] = __ldcg(reinterpret_cast<const unsigned int*>(p) + c);
    }
  }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int c = 0; c < WORDS; ++c) w[c] = 0u;
  }
  __device__ __forceinline__ float get(int e) const {
    if constexpr (sizeof(T) == 2)
      return __uint_as_float((e & 1) ? (w[e >> 1] & 0xFFFF0000u) : (w[e >> 1] << 16));
    else
      return __uint_as_float(w[e]);
  }
};

// ---- paged, per-depth, branch-aware decode attention ------------------------------
// Block (row i, head h, split sp) covers positions [sp*CH, min(sp*CH+CH, pos+1)) of
// the row's own prefix (committed slots, then the ancestors' and its own slot),
// all read from the row's depth plane.  16 lanes share one cache row (HD/16
// elements each, vector loads); each half-warp keeps 8 positions' K and V loads
// in flight and folds them into an online softmax (one pass over the cache).  The 8 half-warps merge in fixed order; the split's (max, sum,
// unnormalised acc) goes to `opart`, and the last block of the (row, head) to
// finish merges all splits in split order and writes the O-GEMM input row
// (deterministic whichever block comes last).
//
// FUSED (decode passes): the block also performs the QKV epilogue for its head
// -- q from the QKV GEMM partials with RoPE, and, in the block that holds the
// row's own position, k (RoPE) and v written to the row's cache slot.  This is
// valid because within one decode pass no row reads a cache row that another
// row of the same pass writes: a row's ancestors sit at strictly greater depth
// (planes differ) and siblings never hold each other's positions.  Prefill
// rows of one chunk do read each other's rows, so prefill runs the separate
// QKV epilogue first (FUSED = false) and reads q from `q`.
template <typename T>
__host__ __device__ constexpr int att_u() {  // positions per half-warp in flight
  return 8;
}

// Everything one attention work item reads or writes (device pointers).
struct AttnArgs {
  const float* q;            // [C][d] queries (prefill; FUSED reads the QKV partials)
  void* kv;                  // cache pool (T)
  int plane_base;            // first plane of this layer
  const int* tagsrc;         // per row: plane offset (depth or readout tag), or null
  int tag_off;
  int S, d, H;               // slots, model width, heads
  const int* r_pos;
  const int* r_blen;
  const int* r_boff;
  const int* lists;
  const int* chain;
  int W, max_splits;
  float* opart;              // [C][H][max_splits][HD + 2] split partials
  int* counters;             // [C][H] split tickets (the last block resets)
  void* X;                   // [C][d] O-GEMM operand rows (T)
  size_t lo;                 // fp32 models: offset of the low tf32 plane
  const float* part;         // QKV GEMM partials (FUSED)
  GemmShape qs_shape;
  int C;
  const int* r_slot;
  const float2* rope;
  const float* ssq;          // RMSNorm sum-of-squares tile parts of the rows (FUSED)
  int ssq_tiles;
  float eps;
  int* err;
  int kv_prefetch;           // 1: request the item's K/V rows into L2 before the dependency wait
};

template <int HD>
struct AttnSmem {
  float qsm[HD];
  int sl[ATT_CH];
  float hm[8], hl[8];
  float hacc[8][HD];
  int last;
};

// One work item: (row i, head h, 128-position split sp of ns).  Run by 128
// threads (tid 0..127); `bar` synchronises them, `dep` returns once the
// inputs written by the preceding phase may be read (the QKV partials, the
// rows' sums of squares).  Work that does not need them -- the slot list, L2
// requests for the K/V rows and (RR_EARLY) the row's RMSNorm factor -- comes
// first.  Returns true in the block that merged the row's splits (written X).
template <typename T, int HD, bool FUSED, bool RR_EARLY, class Bar, class Dep>
__device__ bool attn_item(const AttnArgs& a, AttnSmem<HD>& sm, int h, int i, int sp, int ns,
                          int tid, Bar bar, Dep dep) {
  constexpr int EPL = HD / 16;
  constexpr int NT = 128;
  T* const kv = reinterpret_cast<T*>(a.kv);
  const int S = a.S, d = a.d, H = a.H, C = a.C;
  const int n = a.r_pos[i] + 1;
  const int start = sp * ATT_CH;
  const int cnt = min(ATT_CH, n - start);
  const int plane = a.plane_base + (a.tagsrc ? a.tagsrc[i] : 0) + a.tag_off;
  {
    const int blen = a.r_blen[i], boff = a.r_boff[i];
    for (int t = tid; t < cnt; t += NT) {
      const int j = start + t;
      int s = j < blen ? a.lists[boff + j] : a.chain[i * a.W + (j % a.W)];
      if (s < 0 || s >= S) {
        set_err(a.err, DEV_BAD_INDEX);
        s = 0;
      }
      sm.sl[t] = s;
      if (a.kv_prefetch) {
        const T* kr = kv + kv_off<T>(plane, s, 0, S, d) + (size_t)h * HD;
        const T* vr = kv + kv_off<T>(plane, s, 1, S, d) + (size_t)h * HD;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(kr),
                     "r"((int)(HD * sizeof(T)))
                     : "memory");
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(vr),
                     "r"((int)(HD * sizeof(T)))
                     : "memory");
      }
    }
  }
  // fused prologue inputs that do not depend on the QKV GEMM
  const int half = HD / 2;
  const bool own = sp == ns - 1;  // this block holds the row's own position
  float rr = 1.f;
  float2 cs = make_float2(1.f, 0.f);
  int4 tiA = make_int4(0, -1, 0, 0), tiB = tiA, tiV = tiA;
  int nA = 0, nB = 0, nV = 0;
  bool is_k = false;
  if constexpr (FUSED) {
    if constexpr (RR_EARLY) rr = inv_rms_parts(a.ssq, a.ssq_tiles, C, i, d, a.eps);
    const int t = tid;
    if (t < 2 * half) {
      const int e = t < half ? t : t - half;
      is_k = t >= half;
      nA = (is_k ? d : 0) + h * HD + e;
      nB = nA + half;
      tiA = __ldg(a.qs_shape.tinfo + (nA >> 7));
      tiB = __ldg(a.qs_shape.tinfo + (nB >> 7));
      cs = a.rope[(size_t)(n - 1) * half + e];
    }
    if (t < HD) {
      nV = 2 * d + h * HD + t;
      tiV = __ldg(a.qs_shape.tinfo + (nV >> 7));
    }
  }
  dep();
  if constexpr (FUSED && !RR_EARLY) rr = inv_rms_parts(a.ssq, a.ssq_tiles, C, i, d, a.eps);
  const int hw = tid >> 4, l16 = tid & 15;
  const float scale = rsqrtf((float)HD);
  float qv[EPL];
  if constexpr (FUSED) {
    const int slot = a.r_slot[i];
    T* krow = kv + kv_off<T>(plane, slot, 0, S, d) + (size_t)h * HD;
    T* vrow = kv + kv_off<T>(plane, slot, 1, S, d) + (size_t)h * HD;
    const int t = tid;
    float a1 = 0.f, a2 = 0.f, av = 0.f;
    const bool do_pair = t < 2 * half && (!is_k || own);
    if (do_pair) {
      a1 = rr * sk_reduce_ti(a.part, a.qs_shape, tiA, C, i, nA);
      a2 = rr * sk_reduce_ti(a.part, a.qs_shape, tiB, C, i, nB);
    }
    if (own && t < HD) av = rr * sk_reduce_ti(a.part, a.qs_shape, tiV, C, i, nV);
    if (do_pair) {
      const int e = t < half ? t : t - half;
      const float r1 = a1 * cs.x - a2 * cs.y, r2 = a2 * cs.x + a1 * cs.y;
      if (is_k) {
        krow[e] = from_f<T>(r1);
        krow[e + half] = from_f<T>(r2);
      } else {
        sm.qsm[e] = r1;
        sm.qsm[e + half] = r2;
      }
    }
    if (own && t < HD) vrow[t] = from_f<T>(av);
    bar();  // the own cache row is complete and visible to these threads
#pragma unroll
    for (int e = 0; e < EPL; ++e) qv[e] = sm.qsm[l16 * EPL + e] * scale;
  } else {
    load_vec<float, EPL>(a.q + (size_t)i * d + h * HD + l16 * EPL, qv);
#pragma unroll
    for (int e = 0; e < EPL; ++e) qv[e] *= scale;
    bar();
  }
  const size_t head_off = (size_t)h * HD + l16 * EPL;
  const T* kbase = kv + kv_off<T>(plane, 0, 0, S, d) + head_off;
  const T* vbase = kv + kv_off<T>(plane, 0, 1, S, d) + head_off;
  const size_t slot_stride = (size_t)2 * d;
  float m = -INFINITY, l = 0.f, acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
  // both half-warps of a warp run the same trip count (the shuffles need the warp)
  constexpr int ATT_U = att_u<T>();
  for (int tb = (hw & ~1) * ATT_U; tb < cnt; tb += 8 * ATT_U) {
    const int t0 = tb + (hw & 1) * ATT_U;
    RawVec<T, EPL> kx[ATT_U], vx[ATT_U];
#pragma unroll
    for (int u = 0; u < ATT_U; ++u) {
      const int t = t0 + u;
      if (t < cnt) {
        const size_t off = (size_t)sm.sl[t] * slot_stride;
        kx[u].load(kbase + off);
        vx[u].load(vbase + off);
      } else {
        kx[u].zero();
        vx[u].zero();
      }
    }
    float sc[ATT_U];
#pragma unroll
    for (int u = 0; u < ATT_U; ++u) {
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) dot += qv[e] * kx[u].get(e);
      sc[u] = dot;
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1)
#pragma unroll
      for (int u = 0; u < ATT_U; ++u) sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], o);
    float mloc = -INFINITY;
#pragma unroll
    for (int u = 0; u < ATT_U; ++u)
      if (t0 + u < cnt) mloc = fmaxf(mloc, sc[u]);
    if (mloc == -INFINITY) continue;  // nothing valid for this half-warp (uniform per half)
    const float mnew = fmaxf(m, mloc);
    const float c = __expf(m - mnew);
    l *= c;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] *= c;
#pragma unroll
    for (int u = 0; u < ATT_U; ++u) {
      if (t0 + u < cnt) {
        const float w = __expf(sc[u] - mnew);
        l += w;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] += w * vx[u].get(e);
      }
    }
    m = mnew;
  }
  if (l16 == 0) {
    sm.hm[hw] = m;
    sm.hl[hw] = l;
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) sm.hacc[hw][l16 * EPL + e] = acc[e];
  bar();
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < 8; ++w) M = fmaxf(M, sm.hm[w]);
  float* out = a.opart + ((size_t)(i * H + h) * a.max_splits + sp) * (HD + 2);
  for (int e = tid; e < HD; e += NT) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w)
      if (sm.hm[w] != -INFINITY) v += sm.hacc[w][e] * __expf(sm.hm[w] - M);
    out[2 + e] = v;
  }
  if (tid == 0) {
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w)
      if (sm.hm[w] != -INFINITY) L += sm.hl[w] * __expf(sm.hm[w] - M);
    out[0] = M;
    out[1] = L;
  }
  // the last split block of this (row, head) combines all splits in order;
  // release: the split's stores before the ticket (acq_rel, not a full
  // sequentially consistent fence)
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
  bar();
  if (tid == 0) {
    const int ticket = atomicAdd(&a.counters[i * H + h], 1);
    sm.last = ticket == ns - 1;
    if (sm.last) a.counters[i * H + h] = 0;
  }
  bar();
  const bool last = sm.last;
  if (last) {
    asm volatile("fence.acq_rel.gpu;" ::: "memory");  // acquire: the other splits' stores
    // Merge all splits in split order.  One round of independent loads: thread s
    // fetches split s's (max, sum) into shared memory while every thread fetches
    // its accumulator element of the first ATT_MB splits; then the weights
    // exp(max_s - M) come from shared memory.
    const float* base = a.opart + (size_t)(i * H + h) * a.max_splits * (HD + 2);
    constexpr int ATT_MB = 16;
    constexpr int CAP = 4 * HD;  // splits whose (max, sum) fit in hacc
    float* sM = &sm.hacc[0][0];
    float* sL = sM + CAP;
    const int e = tid;  // element of the head (128 threads >= HD)
    float av[ATT_MB];
#pragma unroll
    for (int k = 0; k < ATT_MB; ++k)
      av[k] = (e < HD && k < ns) ? __ldcg(base + (size_t)k * (HD + 2) + 2 + e) : 0.f;
    if (ns <= CAP) {
      for (int s2 = tid; s2 < ns; s2 += NT) {
        sM[s2] = __ldcg(base + (size_t)s2 * (HD + 2));
        sL[s2] = __ldcg(base + (size_t)s2 * (HD + 2) + 1);
      }
    }
    bar();
    auto mx_of = [&](int s2) { return ns <= CAP ? sM[s2] : __ldcg(base + (size_t)s2 * (HD + 2)); };
    auto l_of = [&](int s2) { return ns <= CAP ? sL[s2] : __ldcg(base + (size_t)s2 * (HD + 2) + 1); };
    float Mx = -INFINITY;
    for (int s2 = 0; s2 < ns; ++s2) Mx = fmaxf(Mx, mx_of(s2));
    float Lx = 0.f;
    for (int s2 = 0; s2 < ns; ++s2) Lx += l_of(s2) * __expf(mx_of(s2) - Mx);
    if (e < HD) {
      float o = 0.f;
#pragma unroll
      for (int k = 0; k < ATT_MB; ++k)
        if (k < ns) o += av[k] * __expf(mx_of(k) - Mx);
      for (int s2 = ATT_MB; s2 < ns; ++s2)
        o += __ldcg(base + (size_t)s2 * (HD + 2) + 2 + e) * __expf(mx_of(s2) - Mx);
      store_act<T>(reinterpret_cast<T*>(a.X) + (size_t)i * d + h * HD, e, o / Lx, a.lo);
    }
  }
  bar();  // shared memory is reused by the next item
  return last;
}

// Items of the active rows in row order: item -> (row, split, the row's
// split count); row = -1 past the last item.  One thread.
__device__ __forceinline__ int3 attn_resolve(const int* __restrict__ mask,
                                             const int* __restrict__ r_pos, int C, int item) {
  int acc = 0, row = -1, spl = 0, nsr = 0;
#pragma unroll 8
  for (int k = 0; k < C; ++k) {
    const int nk = mask[k] ? (r_pos[k] + ATT_CH) / ATT_CH : 0;
    if (row < 0 && item < acc + nk) {
      row = k;
      spl = item - acc;
      nsr = nk;
    }
    acc += nk;
  }
  return make_int3(row, spl, nsr);
}

// Block (head h, y): block y takes items y, y + gridDim.y, ...  The grid holds
// about one resident wave (a grid of every possible item would be mostly empty
// blocks, each still scheduled and retired before the O GEMM may start).  Row
// bookkeeping, slot lists, the cache rows of earlier positions and (fused) the
// RMSNorm sums of squares were written by kernels that finished before this
// grid was launched: for the first item they are read -- and the block's K/V
// rows are requested into L2 -- before the dependency wait, while the QKV GEMM
// in front of this kernel still runs.
template <typename T, int HD, bool FUSED>
__global__ void __launch_bounds__(128) k_attn(const AttnArgs a, const int* __restrict__ mask) {
  __shared__ AttnSmem<HD> sm;
  __shared__ int s_item[3];
  const int h = blockIdx.x;
  for (int item = blockIdx.y, it = 0;; item += gridDim.y, ++it) {
    if (threadIdx.x == 0) {
      const int3 r = attn_resolve(mask, a.r_pos, a.C, item);
      s_item[0] = r.x;
      s_item[1] = r.y;
      s_item[2] = r.z;
    }
    __syncthreads();
    const int i = s_item[0], sp = s_item[1], ns = s_item[2];
    if (i < 0) {
      if (it == 0) {
        pdl_wait();
        pdl_trigger();
      }
      break;
    }
    attn_item<T, HD, FUSED, true>(
        a, sm, h, i, sp, ns, threadIdx.x, [] { __syncthreads(); },
        [it] {
          if (it == 0) {
            pdl_wait();
            pdl_trigger();
          }
        });
  }
}

// ---- attention with a shared-memory ring (the launch path) -----------------------
// Same work items and the same arithmetic as attn_item (per half-warp the same
// positions in the same order, the same merges), so the results are the same
// bits.  What changes is how the K/V rows arrive: a block walks its items as a
// stream of 64-position chunks and keeps the next chunk in flight with cp.async
// into a shared-memory ring, across item boundaries, so the next item's slot
// list and rows load while the current chunk is computed.  Row metadata and
// (fused) the rows' RMSNorm factors are read once per block.  Used for
// contexts up to ATT_RING_MAX_CTX: with many items per block (long contexts)
// the item round trips the ring does not hide, at fewer blocks per SM, make
// k_attn faster.
constexpr int A2_CH = 64;  // positions per chunk: 8 half-warps x 8 positions
// ring stages: two (one chunk ahead, ~74 KB, three blocks per SM) measured
// faster than three (~108 KB, two blocks per SM) on the decode step
constexpr int A2_NS = 2;
constexpr int A2_MAXC = 64;
constexpr int ATT_RING_MAX_CTX = 3072;  // longest context served by k_attn2

template <typename T, int HD>
struct A2Smem {
  T kv[A2_NS][2][A2_CH][HD];  // K then V rows of one chunk
  int sl[A2_NS][ATT_CH];      // slot lists of the items in flight
  int rec[A2_NS][8];          // item records: row, split, splits, head, count, plane, chunks
  float qsm[HD];
  float own_k[HD], own_v[HD];  // (fused) the item's own position
  float hm[8], hl[8];
  float hacc[8][HD];
  int rmask[A2_MAXC], rpos[A2_MAXC], rblen[A2_MAXC], rboff[A2_MAXC], rslot[A2_MAXC],
      rtag[A2_MAXC];
  int rsplit0[A2_MAXC + 1];  // prefix sums of the active rows' splits
  float rr[A2_MAXC];         // (fused) RMSNorm factors
  int last;
};

template <typename T, int HD>
constexpr size_t a2_smem_bytes() {
  return sizeof(A2Smem<T, HD>);
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  const int n = valid ? 16 : 0;  // 0: zero fill
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait(int pending) {
  switch (pending) {
    case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
    case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
    default: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
  }
}

// Grid: about one resident wave of 128-thread blocks; block b takes the items
// w = b, b + gridDim.x, ... with w -> (head w % H, the (w / H)-th (row, split)
// item in row order).
template <typename T, int HD, bool FUSED>
__global__ void __launch_bounds__(128) k_attn2(const AttnArgs a, const int* __restrict__ mask) {
  static_assert(A2_NS <= 3, "cp_async_wait covers up to two pending chunks");
  extern __shared__ __align__(16) unsigned char a2raw[];
  A2Smem<T, HD>& sm = *reinterpret_cast<A2Smem<T, HD>*>(a2raw);
  constexpr int EPL = HD / 16;
  constexpr int PPR = HD * (int)sizeof(T) / 16;  // 16-byte pieces per K or V row
  constexpr int EPP = 16 / (int)sizeof(T);       // elements per piece
  const int tid = threadIdx.x;
  const int H = a.H, C = a.C, S = a.S, d = a.d;
  T* const kv = reinterpret_cast<T*>(a.kv);

  // row metadata: written by kernels that finished before this grid
  if (tid < C) {
    const int m = mask[tid];
    sm.rmask[tid] = m;
    sm.rpos[tid] = a.r_pos[tid];
    sm.rblen[tid] = a.r_blen[tid];
    sm.rboff[tid] = a.r_boff[tid];
    sm.rslot[tid] = a.r_slot[tid];
    sm.rtag[tid] = a.tagsrc ? a.tagsrc[tid] : 0;
    if constexpr (FUSED) sm.rr[tid] = m ? inv_rms_parts(a.ssq, a.ssq_tiles, C, tid, d, a.eps) : 1.f;
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int r = 0; r < C; ++r) {
      sm.rsplit0[r] = acc;
      acc += sm.rmask[r] ? (sm.rpos[r] + ATT_CH) / ATT_CH : 0;
    }
    sm.rsplit0[C] = acc;
  }
  __syncthreads();
  const int items = H * sm.rsplit0[C];
  const int nit = (int)blockIdx.x < items ? (items - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
  if (nit == 0) {
    pdl_wait();
    pdl_trigger();
    return;
  }

  // item k of this block -> record q = k % A2_NS and its slot list (all threads)
  auto prep_item = [&](int k) {
    const int q = k % A2_NS;
    const int w = (int)blockIdx.x + k * (int)gridDim.x;
    const int h = w % H, j = w / H;
    int row = 0;
    while (row + 1 < C && sm.rsplit0[row + 1] <= j) ++row;
    const int sp = j - sm.rsplit0[row];
    const int ns = (sm.rpos[row] + ATT_CH) / ATT_CH;
    const int n = sm.rpos[row] + 1, start = sp * ATT_CH;
    const int cnt = min(ATT_CH, n - start);
    const int blen = sm.rblen[row], boff = sm.rboff[row];
    for (int t = tid; t < cnt; t += 128) {
      const int jj = start + t;
      int s = jj < blen ? a.lists[boff + jj] : a.chain[row * a.W + (jj % a.W)];
      if (s < 0 || s >= S) {
        set_err(a.err, DEV_BAD_INDEX);
        s = 0;
      }
      sm.sl[q][t] = s;
    }
    if (tid == 0) {
      int* r = sm.rec[q];
      r[0] = row;
      r[1] = sp;
      r[2] = ns;
      r[3] = h;
      r[4] = cnt;
      r[5] = a.plane_base + sm.rtag[row] + a.tag_off;
      r[6] = (cnt + A2_CH - 1) / A2_CH;
    }
  };
  // issue the cp.async copies of chunk jc of item k into ring stage st
  auto issue_chunk = [&](int k, int jc, int st) {
    const int q = k % A2_NS;
    const int h = sm.rec[q][3], cnt = sm.rec[q][4], plane = sm.rec[q][5];
    const int p0 = jc * A2_CH, np = min(A2_CH, cnt - p0);
    for (int idx = tid; idx < A2_CH * 2 * PPR; idx += 128) {
      const int p = idx / (2 * PPR), which = (idx / PPR) & 1, pc = idx - (idx / PPR) * PPR;
      T* dst = &sm.kv[st][which][p][pc * EPP];
      const bool ok = p < np;
      const T* src = ok ? kv + kv_off<T>(plane, sm.sl[q][p0 + p], which, S, d) + (size_t)h * HD + pc * EPP
                        : kv;
      cp_async16(dst, src, ok);
    }
    cp_async_commit();
  };

  // the chunk stream: issue cursor (item ki, chunk ji, count ci), compute cursor cc
  int ki = 0, ji = 0, ci = 0, cc = 0;
  auto issue_upto = [&](int upto) {
    while (ci < upto && ki < nit) {
      if (ji == 0) {
        prep_item(ki);
        __syncthreads();  // slot list and record visible
      }
      issue_chunk(ki, ji, ci % A2_NS);
      ++ci;
      if (++ji == sm.rec[ki % A2_NS][6]) {
        ji = 0;
        ++ki;
      }
    }
  };
  if constexpr (!FUSED) {  // the rows of a prefill chunk read each other's fresh cache rows
    pdl_wait();
    pdl_trigger();
  }
  // fused: every ring stage is requested before the dependency wait (the
  // cache rows of earlier positions were written by earlier kernels), so an
  // item's whole 128-position split is in flight while the QKV GEMM finishes
  issue_upto(FUSED ? A2_NS : A2_NS - 1);
  if constexpr (FUSED) {
    pdl_wait();
    pdl_trigger();
  }

  const int hw = tid >> 4, l16 = tid & 15;
  const float scale = rsqrtf((float)HD);
  const int half = HD / 2;
  for (int k = 0; k < nit; ++k) {
    const int q = k % A2_NS;
    const int i = sm.rec[q][0], sp = sm.rec[q][1], ns = sm.rec[q][2], h = sm.rec[q][3];
    const int cnt = sm.rec[q][4], plane = sm.rec[q][5], nch = sm.rec[q][6];
    const bool own = sp == ns - 1;  // this item holds the row's own position
    const int n = sm.rpos[i] + 1;
    float qv[EPL];
    if constexpr (FUSED) {
      // q (RoPE) from the QKV partials; in the own item also k (RoPE) and v, which
      // go to the row's cache slot and into the ring at the own position
      const float rr = sm.rr[i];
      const int t = tid;
      const bool is_k = t >= half && t < 2 * half;
      const int e = t < half ? t : t - half;
      const bool do_pair = t < 2 * half && (!is_k || own);
      float a1 = 0.f, a2 = 0.f, av = 0.f;
      float2 cs = make_float2(1.f, 0.f);
      int nA = 0, nB = 0;
      if (do_pair) {
        nA = (is_k ? d : 0) + h * HD + e;
        nB = nA + half;
        const int4 tiA = __ldg(a.qs_shape.tinfo + (nA >> 7));
        const int4 tiB = __ldg(a.qs_shape.tinfo + (nB >> 7));
        cs = a.rope[(size_t)(n - 1) * half + e];
        a1 = rr * sk_reduce_ti(a.part, a.qs_shape, tiA, C, i, nA);
        a2 = rr * sk_reduce_ti(a.part, a.qs_shape, tiB, C, i, nB);
      }
      if (own && t < HD) {
        const int nV = 2 * d + h * HD + t;
        av = rr * sk_reduce_ti(a.part, a.qs_shape, __ldg(a.qs_shape.tinfo + (nV >> 7)), C, i, nV);
      }
      if (do_pair) {
        const float r1 = a1 * cs.x - a2 * cs.y, r2 = a2 * cs.x + a1 * cs.y;
        if (is_k) {
          T* krow = kv + kv_off<T>(plane, sm.rslot[i], 0, S, d) + (size_t)h * HD;
          krow[e] = from_f<T>(r1);
          krow[e + half] = from_f<T>(r2);
          sm.own_k[e] = to_f<T>(from_f<T>(r1));
          sm.own_k[e + half] = to_f<T>(from_f<T>(r2));
        } else {
          sm.qsm[e] = r1;
          sm.qsm[e + half] = r2;
        }
      }
      if (own && t < HD) {
        T* vrow = kv + kv_off<T>(plane, sm.rslot[i], 1, S, d) + (size_t)h * HD;
        vrow[t] = from_f<T>(av);
        sm.own_v[t] = to_f<T>(from_f<T>(av));
      }
      __syncthreads();
#pragma unroll
      for (int e2 = 0; e2 < EPL; ++e2) qv[e2] = sm.qsm[l16 * EPL + e2] * scale;
    } else {
      load_vec<float, EPL>(a.q + (size_t)i * d + h * HD + l16 * EPL, qv);
#pragma unroll
      for (int e2 = 0; e2 < EPL; ++e2) qv[e2] *= scale;
    }
    float m = -INFINITY, l = 0.f, acc[EPL];
#pragma unroll
    for (int e2 = 0; e2 < EPL; ++e2) acc[e2] = 0.f;
    for (int jc = 0; jc < nch; ++jc, ++cc) {
      issue_upto(cc + A2_NS);       // keep A2_NS - 1 chunks ahead of this one
      cp_async_wait(ci - 1 - cc);   // this thread's copies of chunk cc have landed
      __syncthreads();              // ... and every thread's
      const int st = cc % A2_NS;
      const int p0 = jc * A2_CH;
      if constexpr (FUSED) {
        const int pown = (cnt - 1) - p0;  // the own position, if it is in this chunk
        if (own && pown >= 0 && pown < A2_CH) {
          if (tid < HD) {
            sm.kv[st][0][pown][tid] = from_f<T>(sm.own_k[tid]);
            sm.kv[st][1][pown][tid] = from_f<T>(sm.own_v[tid]);
          }
          __syncthreads();
        }
      }
      // positions hw * 8 .. hw * 8 + 7 of the chunk (the old loop's assignment)
      constexpr int U = 8;
      const int t0 = p0 + hw * U;
      float sc[U];
      RawVec<T, EPL> vx[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int pl = hw * U + u;
        RawVec<T, EPL> kx;
        const uint32_t* kp = reinterpret_cast<const uint32_t*>(&sm.kv[st][0][pl][l16 * EPL]);
        const uint32_t* vp = reinterpret_cast<const uint32_t*>(&sm.kv[st][1][pl][l16 * EPL]);
#pragma unroll
        for (int c2 = 0; c2 < RawVec<T, EPL>::WORDS; ++c2) {
          kx.w[c2] = kp[c2];
          vx[u].w[c2] = vp[c2];
        }
        float dot = 0.f;
#pragma unroll
        for (int e2 = 0; e2 < EPL; ++e2) dot += qv[e2] * kx.get(e2);
        sc[u] = dot;
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1)
#pragma unroll
        for (int u = 0; u < U; ++u) sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], o);
      float mloc = -INFINITY;
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (t0 + u < cnt) mloc = fmaxf(mloc, sc[u]);
      if (mloc != -INFINITY) {
        const float mnew = fmaxf(m, mloc);
        const float c = __expf(m - mnew);
        l *= c;
#pragma unroll
        for (int e2 = 0; e2 < EPL; ++e2) acc[e2] *= c;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          if (t0 + u < cnt) {
            const float wgt = __expf(sc[u] - mnew);
            l += wgt;
#pragma unroll
            for (int e2 = 0; e2 < EPL; ++e2) acc[e2] += wgt * vx[u].get(e2);
          }
        }
        m = mnew;
      }
      __syncthreads();  // ring stage st may be refilled
    }
    // merge the half-warps in fixed order, write the split's partial
    if (l16 == 0) {
      sm.hm[hw] = m;
      sm.hl[hw] = l;
    }
#pragma unroll
    for (int e2 = 0; e2 < EPL; ++e2) sm.hacc[hw][l16 * EPL + e2] = acc[e2];
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int w2 = 0; w2 < 8; ++w2) M = fmaxf(M, sm.hm[w2]);
    float* out = a.opart + ((size_t)(i * H + h) * a.max_splits + sp) * (HD + 2);
    for (int e2 = tid; e2 < HD; e2 += 128) {
      float v = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < 8; ++w2)
        if (sm.hm[w2] != -INFINITY) v += sm.hacc[w2][e2] * __expf(sm.hm[w2] - M);
      out[2 + e2] = v;
    }
    if (tid == 0) {
      float L = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < 8; ++w2)
        if (sm.hm[w2] != -INFINITY) L += sm.hl[w2] * __expf(sm.hm[w2] - M);
      out[0] = M;
      out[1] = L;
    }
    // the last split of this (row, head) to finish merges all splits in order
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    __syncthreads();
    if (tid == 0) {
      const int ticket = atomicAdd(&a.counters[i * H + h], 1);
      sm.last = ticket == ns - 1;
      if (sm.last) a.counters[i * H + h] = 0;
    }
    __syncthreads();
    if (sm.last) {
      asm volatile("fence.acq_rel.gpu;" ::: "memory");
      const float* base = a.opart + (size_t)(i * H + h) * a.max_splits * (HD + 2);
      constexpr int ATT_MB = 16;
      constexpr int CAP = 4 * HD;  // splits whose (max, sum) fit in hacc
      float* sM = &sm.hacc[0][0];
      float* sL = sM + CAP;
      const int e2 = tid;
      float av[ATT_MB];
#pragma unroll
      for (int kk = 0; kk < ATT_MB; ++kk)
        av[kk] = (e2 < HD && kk < ns) ? __ldcg(base + (size_t)kk * (HD + 2) + 2 + e2) : 0.f;
      if (ns <= CAP) {
        for (int s2 = tid; s2 < ns; s2 += 128) {
          sM[s2] = __ldcg(base + (size_t)s2 * (HD + 2));
          sL[s2] = __ldcg(base + (size_t)s2 * (HD + 2) + 1);
        }
      }
      __syncthreads();
      auto mx_of = [&](int s2) { return ns <= CAP ? sM[s2] : __ldcg(base + (size_t)s2 * (HD + 2)); };
      auto l_of = [&](int s2) { return ns <= CAP ? sL[s2] : __ldcg(base + (size_t)s2 * (HD + 2) + 1); };
      float Mx = -INFINITY;
      for (int s2 = 0; s2 < ns; ++s2) Mx = fmaxf(Mx, mx_of(s2));
      float Lx = 0.f;
      for (int s2 = 0; s2 < ns; ++s2) Lx += l_of(s2) * __expf(mx_of(s2) - Mx);
      if (e2 < HD) {
        float o = 0.f;
#pragma unroll
        for (int kk = 0; kk < ATT_MB; ++kk)
          if (kk < ns) o += av[kk] * __expf(mx_of(kk) - Mx);
        for (int s2 = ATT_MB; s2 < ns; ++s2)
          o += __ldcg(base + (size_t)s2 * (HD + 2) + 2 + e2) * __expf(mx_of(s2) - Mx);
        store_act<T>(reinterpret_cast<T*>(a.X) + (size_t)i * d + h * HD, e2, o / Lx, a.lo);
      }
    }
    __syncthreads();  // hacc, qsm and the item record are reused
  }
}

// ---- long contexts: each block streams a contiguous range of splits -----------
// The per-split arithmetic is attn_item's and k_attn2's (per half-warp the same
// positions in the same order, the same merges), so the results are the same
// bits.  The work assignment differs.  Units are (head, row, split) triples in
// head, row, split order; block b of G streams units [b*U/G, (b+1)*U/G) of the
// U units, so the blocks hold the same number of 128-position splits to within
// one, however the rows' lengths fall.  Consecutive units of a block mostly
// belong to one (row, head): the query is formed once per such run, and one
// ticket per run replaces one per split.  K/V rows come through a shared-memory
// ring NS chunks deep (cp.async), and each unit's slot list is loaded into
// registers one unit before its first chunk is requested, so no slot-list round
// trip sits between two chunks.
template <typename T, int HD, int NS>
struct A3Smem {
  T kv[NS][2][A2_CH][HD];  // K then V rows of one chunk
  int sl[NS][ATT_CH];      // slot lists of the units in flight
  int rec[NS][8];          // unit records: row, split, splits, head, count, plane, chunks
  float qsm[HD];
  float own_k[HD], own_v[HD];  // (fused) the row's own position
  float hm[8], hl[8];
  float hacc[8][HD];
  int rmask[A2_MAXC], rpos[A2_MAXC], rblen[A2_MAXC], rboff[A2_MAXC], rslot[A2_MAXC],
      rtag[A2_MAXC];
  int rsplit0[A2_MAXC + 1];  // prefix sums of the active rows' splits
  float rr[A2_MAXC];         // (fused) RMSNorm factors
  int last;
};

// ring depth: about 96 KB of K/V stages (two blocks per SM for bf16, head 128)
template <typename T, int HD>
constexpr int a3_stages() {
  constexpr int stage = 2 * A2_CH * HD * (int)sizeof(T);
  constexpr int n = (96 * 1024) / stage;
  return n < 2 ? 2 : (n > 4 ? 4 : n);
}

template <typename T, int HD>
constexpr size_t a3_smem_bytes() {
  return sizeof(A3Smem<T, HD, a3_stages<T, HD>()>);
}

__device__ __forceinline__ void cp_async_wait_upto3(int pending) {
  switch (pending) {
    case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
    case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
    case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
    default: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
  }
}

template <typename T, int HD, bool FUSED>
__global__ void __launch_bounds__(128) k_attn3(const AttnArgs a, const int* __restrict__ mask) {
  constexpr int NS = a3_stages<T, HD>();
  static_assert(NS >= 2 && NS <= 4, "cp_async_wait_upto3 covers up to three pending chunks");
  extern __shared__ __align__(16) unsigned char a3raw[];
  A3Smem<T, HD, NS>& sm = *reinterpret_cast<A3Smem<T, HD, NS>*>(a3raw);
  constexpr int EPL = HD / 16;
  constexpr int PPR = HD * (int)sizeof(T) / 16;  // 16-byte pieces per K or V row
  constexpr int EPP = 16 / (int)sizeof(T);       // elements per piece
  const int tid = threadIdx.x;
  const int H = a.H, C = a.C, S = a.S, d = a.d;
  T* const kv = reinterpret_cast<T*>(a.kv);

  // row metadata: written by kernels that finished before this grid
  if (tid < C) {
    const int m = mask[tid];
    sm.rmask[tid] = m;
    sm.rpos[tid] = a.r_pos[tid];
    sm.rblen[tid] = a.r_blen[tid];
    sm.rboff[tid] = a.r_boff[tid];
    sm.rslot[tid] = a.r_slot[tid];
    sm.rtag[tid] = a.tagsrc ? a.tagsrc[tid] : 0;
    if constexpr (FUSED) sm.rr[tid] = m ? inv_rms_parts(a.ssq, a.ssq_tiles, C, tid, d, a.eps) : 1.f;
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int r = 0; r < C; ++r) {
      sm.rsplit0[r] = acc;
      acc += sm.rmask[r] ? (sm.rpos[r] + ATT_CH) / ATT_CH : 0;
    }
    sm.rsplit0[C] = acc;
  }
  __syncthreads();
  const int TS = sm.rsplit0[C];  // splits of one head
  const long long U = (long long)H * TS;
  const int u0 = (int)(U * blockIdx.x / gridDim.x);
  const int nit = (int)(U * (blockIdx.x + 1) / gridDim.x) - u0;
  if (nit <= 0) {
    pdl_wait();
    pdl_trigger();
    return;
  }

  // unit k of this block: head, row, split, first position, position count
  struct Unit {
    int h, row, sp, start, cnt;
  };
  auto unit = [&](int k) {
    Unit x;
    const int u = u0 + k;
    x.h = u / TS;
    const int j = u - x.h * TS;
    int lo = 0, hi = C - 1;  // the last row whose first split is <= j (it has splits)
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sm.rsplit0[mid] <= j)
        lo = mid;
      else
        hi = mid - 1;
    }
    x.row = lo;
    x.sp = j - sm.rsplit0[lo];
    x.start = x.sp * ATT_CH;
    x.cnt = min(ATT_CH, sm.rpos[lo] + 1 - x.start);
    return x;
  };
  // this thread's slot of unit x (position start + tid); the load is not waited on here
  auto slot_load = [&](Unit x) {
    if (tid >= x.cnt) return 0;
    const int jj = x.start + tid;
    return jj < sm.rblen[x.row] ? a.lists[sm.rboff[x.row] + jj]
                                : a.chain[x.row * a.W + (jj % a.W)];
  };

  // issue side: unit ki (record written when ji == 0), its chunk ji, chunk count ci
  int ki = 0, ji = 0, ci = 0, cc = 0;
  Unit xi = unit(0);
  int nslot = slot_load(xi);  // slot of unit ki for this thread
  auto issue_upto = [&](int upto) {
    while (ci < upto && ki < nit) {
      const int q = ki % NS;
      if (ji == 0) {
        if (tid < xi.cnt) {
          int s = nslot;
          if (s < 0 || s >= S) {
            set_err(a.err, DEV_BAD_INDEX);
            s = 0;
          }
          sm.sl[q][tid] = s;
        }
        if (tid == 0) {
          int* r = sm.rec[q];
          r[0] = xi.row;
          r[1] = xi.sp;
          r[2] = (sm.rpos[xi.row] + ATT_CH) / ATT_CH;
          r[3] = xi.h;
          r[4] = xi.cnt;
          r[5] = a.plane_base + sm.rtag[xi.row] + a.tag_off;
          r[6] = (xi.cnt + A2_CH - 1) / A2_CH;
        }
        if (ki + 1 < nit) {  // the next unit's slot list starts on its way now
          xi = unit(ki + 1);
          nslot = slot_load(xi);
        }
        __syncthreads();  // slot list and record visible
      }
      // the cp.async copies of chunk ji of unit ki into ring stage ci % NS
      const int st = ci % NS;
      const int h = sm.rec[q][3], cnt = sm.rec[q][4], plane = sm.rec[q][5];
      const int p0 = ji * A2_CH, np = min(A2_CH, cnt - p0);
      for (int idx = tid; idx < A2_CH * 2 * PPR; idx += 128) {
        const int p = idx / (2 * PPR), which = (idx / PPR) & 1, pc = idx - (idx / PPR) * PPR;
        T* dst = &sm.kv[st][which][p][pc * EPP];
        const bool ok = p < np;
        const T* src = ok ? kv + kv_off<T>(plane, sm.sl[q][p0 + p], which, S, d) + (size_t)h * HD + pc * EPP
                          : kv;
        cp_async16(dst, src, ok);
      }
      cp_async_commit();
      ++ci;
      if (++ji == sm.rec[q][6]) {
        ji = 0;
        ++ki;
      }
    }
  };
  if constexpr (!FUSED) {  // the rows of a prefill chunk read each other's fresh cache rows
    pdl_wait();
    pdl_trigger();
  }
  // fused: every ring stage is requested before the dependency wait (the cache
  // rows of earlier positions were written by earlier kernels)
  issue_upto(FUSED ? NS : NS - 1);
  if constexpr (FUSED) {
    pdl_wait();
    pdl_trigger();
  }

  const int hw = tid >> 4, l16 = tid & 15;
  const float scale = rsqrtf((float)HD);
  const int half = HD / 2;
  // the (row, head) run in progress: its splits done here since the last ticket
  int cur_i = -1, cur_h = -1, cur_ns = 0, npend = 0;
  // Ticket for the run's npend splits; the block that completes the (row, head)
  // merges all its splits in split order (deterministic whichever block is last).
  auto finish_run = [&]() {
    asm volatile("fence.acq_rel.gpu;" ::: "memory");  // release: the run's partials
    __syncthreads();
    if (tid == 0) {
      const int ticket = atomicAdd(&a.counters[cur_i * H + cur_h], npend);
      sm.last = ticket + npend == cur_ns;
      if (sm.last) a.counters[cur_i * H + cur_h] = 0;
    }
    __syncthreads();
    if (sm.last) {
      asm volatile("fence.acq_rel.gpu;" ::: "memory");  // acquire: the other blocks' partials
      const int ns = cur_ns;
      const float* base = a.opart + (size_t)(cur_i * H + cur_h) * a.max_splits * (HD + 2);
      constexpr int ATT_MB = 16;
      constexpr int CAP = 4 * HD;  // splits whose (max, sum) fit in hacc
      float* sM = &sm.hacc[0][0];
      float* sL = sM + CAP;
      const int e2 = tid;
      float av[ATT_MB];
#pragma unroll
      for (int kk = 0; kk < ATT_MB; ++kk)
        av[kk] = (e2 < HD && kk < ns) ? __ldcg(base + (size_t)kk * (HD + 2) + 2 + e2) : 0.f;
      if (ns <= CAP) {
        for (int s2 = tid; s2 < ns; s2 += 128) {
          sM[s2] = __ldcg(base + (size_t)s2 * (HD + 2));
          sL[s2] = __ldcg(base + (size_t)s2 * (HD + 2) + 1);
        }
      }
      __syncthreads();
      auto mx_of = [&](int s2) { return ns <= CAP ? sM[s2] : __ldcg(base + (size_t)s2 * (HD + 2)); };
      auto l_of = [&](int s2) { return ns <= CAP ? sL[s2] : __ldcg(base + (size_t)s2 * (HD + 2) + 1); };
      float Mx = -INFINITY;
      for (int s2 = 0; s2 < ns; ++s2) Mx = fmaxf(Mx, mx_of(s2));
      float Lx = 0.f;
      for (int s2 = 0; s2 < ns; ++s2) Lx += l_of(s2) * __expf(mx_of(s2) - Mx);
      if (e2 < HD) {
        float o = 0.f;
#pragma unroll
        for (int kk = 0; kk < ATT_MB; ++kk)
          if (kk < ns) o += av[kk] * __expf(mx_of(kk) - Mx);
        for (int s2 = ATT_MB; s2 < ns; ++s2)
          o += __ldcg(base + (size_t)s2 * (HD + 2) + 2 + e2) * __expf(mx_of(s2) - Mx);
        store_act<T>(reinterpret_cast<T*>(a.X) + (size_t)cur_i * d + cur_h * HD, e2, o / Lx, a.lo);
      }
      __syncthreads();  // hacc is reused
    }
    npend = 0;
  };

  float qv[EPL];
  for (int k = 0; k < nit; ++k) {
    const int q = k % NS;
    const int i = sm.rec[q][0], sp = sm.rec[q][1], ns = sm.rec[q][2], h = sm.rec[q][3];
    const int cnt = sm.rec[q][4], plane = sm.rec[q][5], nch = sm.rec[q][6];
    const bool own = sp == ns - 1;  // this unit holds the row's own position
    const bool newrun = i != cur_i || h != cur_h;
    if (newrun && npend > 0) finish_run();
    cur_i = i;
    cur_h = h;
    cur_ns = ns;
    const int n = sm.rpos[i] + 1;
    if constexpr (FUSED) {
      if (newrun || own) {
        // q (RoPE) from the QKV partials at a run's start; in the own unit also
        // k (RoPE) and v, which go to the row's cache slot and into the ring at
        // the own position
        const float rr = sm.rr[i];
        const int t = tid;
        const bool is_k = t >= half && t < 2 * half;
        const int e = t < half ? t : t - half;
        const bool do_pair = t < 2 * half && (is_k ? own : newrun);
        float a1 = 0.f, a2 = 0.f, av = 0.f;
        float2 cs = make_float2(1.f, 0.f);
        if (do_pair) {
          const int nA = (is_k ? d : 0) + h * HD + e;
          const int nB = nA + half;
          const int4 tiA = __ldg(a.qs_shape.tinfo + (nA >> 7));
          const int4 tiB = __ldg(a.qs_shape.tinfo + (nB >> 7));
          cs = a.rope[(size_t)(n - 1) * half + e];
          a1 = rr * sk_reduce_ti(a.part, a.qs_shape, tiA, C, i, nA);
          a2 = rr * sk_reduce_ti(a.part, a.qs_shape, tiB, C, i, nB);
        }
        if (own && t < HD) {
          const int nV = 2 * d + h * HD + t;
          av = rr * sk_reduce_ti(a.part, a.qs_shape, __ldg(a.qs_shape.tinfo + (nV >> 7)), C, i, nV);
        }
        if (do_pair) {
          const float r1 = a1 * cs.x - a2 * cs.y, r2 = a2 * cs.x + a1 * cs.y;
          if (is_k) {
            T* krow = kv + kv_off<T>(plane, sm.rslot[i], 0, S, d) + (size_t)h * HD;
            krow[e] = from_f<T>(r1);
            krow[e + half] = from_f<T>(r2);
            sm.own_k[e] = to_f<T>(from_f<T>(r1));
            sm.own_k[e + half] = to_f<T>(from_f<T>(r2));
          } else {
            sm.qsm[e] = r1;
            sm.qsm[e + half] = r2;
          }
        }
        if (own && t < HD) {
          T* vrow = kv + kv_off<T>(plane, sm.rslot[i], 1, S, d) + (size_t)h * HD;
          vrow[t] = from_f<T>(av);
          sm.own_v[t] = to_f<T>(from_f<T>(av));
        }
        __syncthreads();
        if (newrun) {
#pragma unroll
          for (int e2 = 0; e2 < EPL; ++e2) qv[e2] = sm.qsm[l16 * EPL + e2] * scale;
        }
      }
    } else {
      if (newrun) {
        load_vec<float, EPL>(a.q + (size_t)i * d + h * HD + l16 * EPL, qv);
#pragma unroll
        for (int e2 = 0; e2 < EPL; ++e2) qv[e2] *= scale;
      }
    }
    float m = -INFINITY, l = 0.f, acc[EPL];
#pragma unroll
    for (int e2 = 0; e2 < EPL; ++e2) acc[e2] = 0.f;
    for (int jc = 0; jc < nch; ++jc, ++cc) {
      issue_upto(cc + NS);               // keep NS - 1 chunks ahead of this one
      cp_async_wait_upto3(ci - 1 - cc);  // this thread's copies of chunk cc have landed
      __syncthreads();                   // ... and every thread's
      const int st = cc % NS;
      const int p0 = jc * A2_CH;
      if constexpr (FUSED) {
        const int pown = (cnt - 1) - p0;  // the own position, if it is in this chunk
        if (own && pown >= 0 && pown < A2_CH) {
          if (tid < HD) {
            sm.kv[st][0][pown][tid] = from_f<T>(sm.own_k[tid]);
            sm.kv[st][1][pown][tid] = from_f<T>(sm.own_v[tid]);
          }
          __syncthreads();
        }
      }
      // positions hw * 8 .. hw * 8 + 7 of the chunk (attn_item's assignment)
      constexpr int U = 8;
      const int t0 = p0 + hw * U;
      float sc[U];
      RawVec<T, EPL> vx[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int pl = hw * U + u;
        RawVec<T, EPL> kx;
        const uint32_t* kp = reinterpret_cast<const uint32_t*>(&sm.kv[st][0][pl][l16 * EPL]);
        const uint32_t* vp = reinterpret_cast<const uint32_t*>(&sm.kv[st][1][pl][l16 * EPL]);
#pragma unroll
        for (int c2 = 0; c2 < RawVec<T, EPL>::WORDS; ++c2) {
          kx.w[c2] = kp[c2];
          vx[u].w[c2] = vp[c2];
        }
        float dot = 0.f;
#pragma unroll
        for (int e2 = 0; e2 < EPL; ++e2) dot += qv[e2] * kx.get(e2);
        sc[u] = dot;
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1)
#pragma unroll
        for (int u = 0; u < U; ++u) sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], o);
      float mloc = -INFINITY;
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (t0 + u < cnt) mloc = fmaxf(mloc, sc[u]);
      if (mloc != -INFINITY) {
        const float mnew = fmaxf(m, mloc);
        const float c = __expf(m - mnew);
        l *= c;
#pragma unroll
        for (int e2 = 0; e2 < EPL; ++e2) acc[e2] *= c;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          if (t0 + u < cnt) {
            const float wgt = __expf(sc[u] - mnew);
            l += wgt;
#pragma unroll
            for (int e2 = 0; e2 < EPL; ++e2) acc[e2] += wgt * vx[u].get(e2);
          }
        }
        m = mnew;
      }
      __syncthreads();  // ring stage st may be refilled
    }
    // merge the half-warps in fixed order, write the split's partial
    if (l16 == 0) {
      sm.hm[hw] = m;
      sm.hl[hw] = l;
    }
#pragma unroll
    for (int e2 = 0; e2 < EPL; ++e2) sm.hacc[hw][l16 * EPL + e2] = acc[e2];
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int w2 = 0; w2 < 8; ++w2) M = fmaxf(M, sm.hm[w2]);
    float* out = a.opart + ((size_t)(i * H + h) * a.max_splits + sp) * (HD + 2);
    for (int e2 = tid; e2 < HD; e2 += 128) {
      float v = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < 8; ++w2)
        if (sm.hm[w2] != -INFINITY) v += sm.hacc[w2][e2] * __expf(sm.hm[w2] - M);
      out[2 + e2] = v;
    }
    if (tid == 0) {
      float L = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < 8; ++w2)
        if (sm.hm[w2] != -INFINITY) L += sm.hl[w2] * __expf(sm.hm[w2] - M);
      out[0] = M;
      out[1] = L;
    }
    ++npend;
    __syncthreads();  // hacc, qsm and the unit record are reused
  }
  finish_run();
}

// ---- RoPE table: (cos, sin) of pos * theta^(-2e/hd), computed in double ------------
static __global__ void k_rope_table(float2* __restrict__ rope, int max_pos, int hd, double theta) {
  const int half = hd / 2;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= max_pos * half) return;
  const int pos = idx / half, e = idx - pos * half;
  const double inv = pow(theta, -2.0 * e / hd);
  double sn, cs;
  sincos((double)pos * inv, &sn, &cs);
  rope[idx] = make_float2((float)cs, (float)sn);
}

}  // namespace lt
