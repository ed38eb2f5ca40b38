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
#include "tc.cuh"

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

// ---- paged, per-depth, branch-aware decode attention ------------------------------
// A row attends to positions [0, pos] of its own prefix (committed slots, then
// the ancestors' and its own slot), all read from the row's depth plane, in
// splits of ATT_CH positions; each split's (max, sum, unnormalised acc) goes to
// `opart`, and the block that completes a (row, head) merges the splits in split
// order and writes the O-GEMM input row.  Split boundaries depend on the
// position only, so a row's result does not depend on the other rows of a pass.
//
// FUSED (decode passes): attention also performs the QKV epilogue for its head
// -- q from the QKV GEMM partials with RoPE, and, for the split that holds the
// row's own position, k (RoPE) and v written to the row's cache slot.  This is
// valid because within one decode pass no row reads a cache row that another
// row of the same pass writes: a row's ancestors sit at strictly greater depth
// (planes differ) and siblings never hold each other's positions.  Prefill
// rows of one chunk do read each other's rows, so prefill runs the separate
// QKV epilogue first (FUSED = false) and reads q from `q`.
constexpr int ATT_CHUNK = 64;  // positions per ring stage (16 groups x 4 positions)
constexpr int ATT_MAXC = 64;   // rows a pass may hold

// Everything the attention kernel reads or writes (device pointers).
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
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  const int n = valid ? 16 : 0;  // 0: zero fill
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async16_full(void* dst, const void* src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// ---- the attention kernel: each block streams a contiguous range of splits ------
// Units are (head, row, 128-position split) triples in head, row, split order.
// Block b of a resident wave of G blocks streams units [b*U/G, (b+1)*U/G) of
// the U units, so every block holds the same number of splits to within one,
// however the rows' lengths fall.  A block's consecutive units mostly belong to
// one (row, head): the query is formed once per such run, and one split ticket
// per run replaces one per split.  K/V rows come through a shared-memory ring
// of NS stages (cp.async; a stage holds one chunk of 64 positions, and the next
// chunks are in flight while one is computed).  Each unit's slot list is loaded
// into registers one unit before its first chunk is requested.
//
// Compute layout: 16 groups of 8 lanes.  Group g takes positions g, g + 16,
// g + 32 and g + 48 of a chunk.  Lane j of a group takes pieces j, j + 8, ... of
// a head's K and V rows (PB bytes each), so one shared-memory load per piece
// reads contiguous bytes across the group; a lane loads all of its pieces of a
// chunk before the math.  bf16 caches: the query and the softmax weights enter
// the products as bf16 (fma.rn.f32.bf16, exact products, fp32 accumulation);
// fp32 caches: fp32 throughout.  A group keeps an online softmax state
// (max, sum, accumulator) over its positions of the split.  Positions past the
// split's end score -inf, and their zero-filled V rows add nothing.  At the
// split's end the 16 states merge in group order into the split's partial.  The
// block that completes a (row, head) merges its splits in split order, so the
// result is deterministic whichever block comes last.
template <typename T, int HD, int NS>
struct AttnSmem {
  T kv[NS][2][ATT_CHUNK][HD];  // K then V rows of one chunk (a consumed stage doubles as scratch)
  int sl[NS][ATT_CH];      // slot lists of the units in flight
  int rec[NS][8];          // unit records: row, split, splits, head, count, plane, chunks
  float qsm[HD];
  float own_k[HD], own_v[HD];  // (fused) the row's own position
  int rmask[ATT_MAXC], rpos[ATT_MAXC], rblen[ATT_MAXC], rboff[ATT_MAXC], rslot[ATT_MAXC],
      rtag[ATT_MAXC];
  int rsplit0[ATT_MAXC + 1];  // prefix sums of the active rows' splits
  float rr[ATT_MAXC];         // (fused) RMSNorm factors
  int last;
};

// A lane's share of one head's row: NP pieces of PB bytes (EPP elements each).
template <typename T, int HD>
struct AttnLane {
  static constexpr int ROWB = HD * (int)sizeof(T);
  static constexpr int PB = (ROWB / 16) % 8 == 0 ? 16 : 8;
  static constexpr int NP = ROWB / PB / 8;
  static constexpr int EPP = PB / (int)sizeof(T);
  static constexpr int EL = NP * EPP;  // elements per lane
  static_assert(ROWB % (8 * PB) == 0 && EPP % 2 == 0, "lane layout");
};

template <int PB>
__device__ __forceinline__ void lds_piece(const void* p, uint32_t* w) {
  if constexpr (PB == 16) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    w[0] = u.x;
    w[1] = u.y;
    w[2] = u.z;
    w[3] = u.w;
  } else {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    w[0] = u.x;
    w[1] = u.y;
  }
}

// element t of a piece held as 32-bit words
template <typename T>
__device__ __forceinline__ float piece_elem(const uint32_t* w, int t) {
  if constexpr (sizeof(T) == 2)
    return __uint_as_float((t & 1) ? (w[t >> 1] & 0xFFFF0000u) : (w[t >> 1] << 16));
  else
    return __uint_as_float(w[t]);
}

// bf16 caches: products of two bf16 halves accumulated in fp32 with one rounding
// per step (a bf16 product is exact in fp32, so each step equals fmaf of the
// widened operands); saves the widening instruction per element.
// c + a.lo * b.lo + a.hi * b.hi, in that order
__device__ __forceinline__ float fma_bf16_pair(uint32_t a, uint32_t b, float c) {
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %1;\n\t"
      "mov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, al, bl, %0;\n\t"
      "fma.rn.f32.bf16 %0, ah, bh, %0;\n\t}"
      : "+f"(c)
      : "r"(a), "r"(b));
  return c;
}
// a0 += v.lo * w.lo, a1 += v.hi * w.hi
__device__ __forceinline__ void fma_bf16_split(uint32_t v, uint32_t w, float& a0, float& a1) {
  asm("{\n\t.reg .b16 vl, vh, wl, wh;\n\t"
      "mov.b32 {vl, vh}, %2;\n\t"
      "mov.b32 {wl, wh}, %3;\n\t"
      "fma.rn.f32.bf16 %0, vl, wl, %0;\n\t"
      "fma.rn.f32.bf16 %1, vh, wh, %1;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "r"(v), "r"(w));
}
__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

// ring depth: two stages (one chunk ahead) keep three blocks per SM for bf16,
// head 128, which measured faster than three stages at two blocks per SM on
// contexts of 256-8192 positions (more resident blocks overlap the per-chunk
// compute better than a deeper ring hides it)
template <typename T, int HD>
constexpr int attn_stages() {
  return 2;
}

template <typename T, int HD, int NS>
constexpr size_t attn_smem_bytes() {
  return sizeof(AttnSmem<T, HD, NS>);
}

__device__ __forceinline__ void cp_async_wait(int pending) {
  switch (pending) {
    case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
    case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
    case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
    default: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
  }
}

template <typename T, int HD, int NS, bool FUSED>
__global__ void __launch_bounds__(128, 3) k_attn(const AttnArgs a, const int* __restrict__ mask) {
  static_assert(NS >= 2 && NS <= 4, "cp_async_wait covers up to three pending chunks");
  using L = AttnLane<T, HD>;
  extern __shared__ __align__(16) unsigned char attn_raw[];
  AttnSmem<T, HD, NS>& sm = *reinterpret_cast<AttnSmem<T, HD, NS>*>(attn_raw);
  constexpr int PPR = HD * (int)sizeof(T) / 16;  // 16-byte copy pieces per K or V row
  constexpr int EPP16 = 16 / (int)sizeof(T);     // elements per copy piece
  // Copy roles: a chunk is 2 * ATT_CHUNK rows (K and V of ATT_CHUNK positions) of PPR
  // pieces; PP2 is PPR rounded up to a power of two.  Thread tid always moves
  // piece tid % PP2 (if < PPR) of the rows r = tid / PP2 + k * RSTEP, so its K/V
  // choice is fixed and each copy costs a slot load and one multiply-add.
  constexpr int PP2 = PPR <= 4 ? 4 : PPR <= 8 ? 8 : PPR <= 16 ? 16 : PPR <= 32 ? 32 : 64;
  static_assert(PPR <= 64, "copy roles");
  constexpr int RSTEP = 128 / PP2;          // rows a round of 128 threads covers (even)
  constexpr int NCOPY = 2 * ATT_CHUNK / RSTEP;  // copies per thread per chunk
  constexpr int SCR = 2 * ATT_CHUNK * HD * (int)sizeof(T) / 4;  // floats of scratch in a stage
  static_assert(SCR >= 48 + 16 * HD, "a stage holds the 16 group states");
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
          r[6] = (xi.cnt + ATT_CHUNK - 1) / ATT_CHUNK;
        }
        if (ki + 1 < nit) {  // the next unit's slot list starts on its way now
          xi = unit(ki + 1);
          nslot = slot_load(xi);
        }
        __syncthreads();  // slot list and record visible
      }
      // the cp.async copies of chunk ji of unit ki into ring stage ci % NS
      // (rows past the unit's end are zero-filled)
      const int st = ci % NS;
      {
        const int h = sm.rec[q][3], cnt = sm.rec[q][4], plane = sm.rec[q][5];
        const int p0 = ji * ATT_CHUNK, np = min(ATT_CHUNK, cnt - p0);
        const int pc = tid % PP2, r0 = tid / PP2, which = r0 & 1;
        if (pc < PPR) {
          const T* src0 = kv + kv_off<T>(plane, 0, which, S, d) + (size_t)h * HD + pc * EPP16;
          const int* sl = &sm.sl[q][p0];
          T* dst0 = &sm.kv[st][which][r0 >> 1][pc * EPP16];
          constexpr int DSTEP = (RSTEP / 2) * HD;  // elements between a thread's rows
          const size_t sstride = 2 * (size_t)d;
          if (np == ATT_CHUNK) {  // a full chunk: no predicates
#pragma unroll 4
            for (int k = 0; k < NCOPY; ++k)
              cp_async16_full(dst0 + k * DSTEP, src0 + (size_t)sl[(r0 >> 1) + k * (RSTEP / 2)] * sstride);
          } else {
#pragma unroll 4
            for (int k = 0; k < NCOPY; ++k) {
              const int p = (r0 >> 1) + k * (RSTEP / 2);
              const bool ok = p < np;
              cp_async16(dst0 + k * DSTEP, ok ? src0 + (size_t)sl[p] * sstride : kv, ok);
            }
          }
        }
        cp_async_commit();
      }
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

  const int g = tid >> 3, j = tid & 7;  // group, lane in the group
  const float scale = rsqrtf((float)HD);
  const int half = HD / 2;
  // the (row, head) run in progress: its splits done here since the last ticket
  int cur_i = -1, cur_h = -1, cur_ns = 0, npend = 0;
  // Ticket for the run's npend splits; the block that completes the (row, head)
  // merges all its splits in split order.  Scratch: the ring stage that holds
  // no chunk in flight (the one consumed last).
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
      constexpr int CAP = SCR / 2;  // splits whose (max, sum) fit in the scratch
      float* sM = reinterpret_cast<float*>(&sm.kv[(cc + NS - 1) % NS][0][0][0]);
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
      __syncthreads();  // the scratch stage is refilled next
    }
    npend = 0;
  };

  // the query, scaled: fp32 (fp32 caches) or bf16 pairs in the cache's word layout
  float qv[L::EL];
  uint32_t qb[L::EL / 2];
  auto pack_q = [&]() {
    if constexpr (sizeof(T) == 2) {
#pragma unroll
      for (int t2 = 0; t2 < L::EL / 2; ++t2) qb[t2] = bf16x2_bits(qv[2 * t2], qv[2 * t2 + 1]);
    }
  };
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
          for (int kp = 0; kp < L::NP; ++kp)
#pragma unroll
            for (int t2 = 0; t2 < L::EPP; ++t2)
              qv[kp * L::EPP + t2] = sm.qsm[(kp * 8 + j) * L::EPP + t2] * scale;
          pack_q();
        }
      }
    } else {
      if (newrun) {
        const float* qrow = a.q + (size_t)i * d + h * HD;
#pragma unroll
        for (int kp = 0; kp < L::NP; ++kp)
#pragma unroll
          for (int t2 = 0; t2 < L::EPP; ++t2) qv[kp * L::EPP + t2] = qrow[(kp * 8 + j) * L::EPP + t2] * scale;
        pack_q();
      }
    }
    float m = -INFINITY, l = 0.f, acc[L::EL];
#pragma unroll
    for (int e2 = 0; e2 < L::EL; ++e2) acc[e2] = 0.f;
    for (int jc = 0; jc < nch; ++jc, ++cc) {
      issue_upto(cc + NS);               // keep NS - 1 chunks ahead of this one
      cp_async_wait(ci - 1 - cc);  // this thread's copies of chunk cc have landed
      __syncthreads();                   // ... and every thread's
      const int st = cc % NS;
      const int p0 = jc * ATT_CHUNK;
      if constexpr (FUSED) {
        const int pown = (cnt - 1) - p0;  // the own position, if it is in this chunk
        if (own && pown >= 0 && pown < ATT_CHUNK) {
          if (tid < HD) {
            sm.kv[st][0][pown][tid] = from_f<T>(sm.own_k[tid]);
            sm.kv[st][1][pown][tid] = from_f<T>(sm.own_v[tid]);
          }
          __syncthreads();
        }
      }
      // the group's four positions: every K and V piece of the lane is loaded
      // first (independent shared-memory loads in flight together), then the
      // lane's partial dot products and a butterfly over the group's 8 lanes
      uint32_t kw[4][L::NP][L::PB / 4], vw[4][L::NP][L::PB / 4];
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4)
#pragma unroll
        for (int kp = 0; kp < L::NP; ++kp) {
          lds_piece<L::PB>(&sm.kv[st][0][g + 16 * k4][(kp * 8 + j) * L::EPP], kw[k4][kp]);
          lds_piece<L::PB>(&sm.kv[st][1][g + 16 * k4][(kp * 8 + j) * L::EPP], vw[k4][kp]);
        }
      float sc[4];
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        float dot = 0.f;
#pragma unroll
        for (int kp = 0; kp < L::NP; ++kp) {
          float pd = 0.f;
          if constexpr (sizeof(T) == 2) {
#pragma unroll
            for (int w2 = 0; w2 < L::EPP / 2; ++w2) pd = fma_bf16_pair(kw[k4][kp][w2], qb[kp * L::EPP / 2 + w2], pd);
          } else {
#pragma unroll
            for (int t2 = 0; t2 < L::EPP; ++t2) pd = fmaf(qv[kp * L::EPP + t2], piece_elem<T>(kw[k4][kp], t2), pd);
          }
          dot += pd;
        }
        sc[k4] = dot;
      }
#pragma unroll
      for (int o = 4; o > 0; o >>= 1)
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) sc[k4] += __shfl_xor_sync(0xffffffffu, sc[k4], o);
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) sc[k4] = p0 + g + 16 * k4 < cnt ? sc[k4] : -INFINITY;
      const float mnew = fmaxf(m, fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3])));
      const float ms = mnew == -INFINITY ? 0.f : mnew;  // no valid position yet: weights 0
      const float c = __expf(m - ms);
      float wk[4];
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) wk[k4] = __expf(sc[k4] - ms);
      l = l * c + ((wk[0] + wk[1]) + (wk[2] + wk[3]));
#pragma unroll
      for (int e2 = 0; e2 < L::EL; ++e2) acc[e2] *= c;
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        // bf16 caches: the weight in bf16, as the V operand (bf16 attention's usual P)
        const uint32_t wb = sizeof(T) == 2 ? bf16x2_bits(wk[k4], wk[k4]) : 0u;
#pragma unroll
        for (int kp = 0; kp < L::NP; ++kp) {
          if constexpr (sizeof(T) == 2) {
#pragma unroll
            for (int w2 = 0; w2 < L::EPP / 2; ++w2)
              fma_bf16_split(vw[k4][kp][w2], wb, acc[kp * L::EPP + 2 * w2], acc[kp * L::EPP + 2 * w2 + 1]);
          } else {
#pragma unroll
            for (int t2 = 0; t2 < L::EPP; ++t2)
              acc[kp * L::EPP + t2] = fmaf(wk[k4], piece_elem<T>(vw[k4][kp], t2), acc[kp * L::EPP + t2]);
          }
        }
      }
      m = mnew;
      __syncthreads();  // ring stage st may be refilled
    }
    // merge the 16 group states in group order into the split's partial; the
    // stage consumed last is scratch: [0, 16) maxima, [16, 32) sums, [32, 48)
    // the groups' weights, then 16 accumulators of HD
    {
      float* scr = reinterpret_cast<float*>(&sm.kv[(cc + NS - 1) % NS][0][0][0]);
      if (j == 0) {
        scr[g] = m;
        scr[16 + g] = l;
      }
#pragma unroll
      for (int kp = 0; kp < L::NP; ++kp)
#pragma unroll
        for (int t2 = 0; t2 < L::EPP; ++t2)
          scr[48 + g * HD + (kp * 8 + j) * L::EPP + t2] = acc[kp * L::EPP + t2];
      __syncthreads();
      float* out = a.opart + ((size_t)(i * H + h) * a.max_splits + sp) * (HD + 2);
      if (tid < 32) {  // warp 0: the split's max, the groups' weights and the sum
        const float mg = tid < 16 ? scr[tid] : -INFINITY;
        float M = mg;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        const float f = mg == -INFINITY ? 0.f : __expf(mg - M);
        float Ls = tid < 16 ? scr[16 + tid] * f : 0.f;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
        if (tid < 16) scr[32 + tid] = f;
        if (tid == 0) {
          out[0] = M;
          out[1] = Ls;
        }
      }
      __syncthreads();
      for (int e2 = tid; e2 < HD; e2 += 128) {
        float v = 0.f;
#pragma unroll
        for (int g2 = 0; g2 < 16; ++g2) v = fmaf(scr[48 + g2 * HD + e2], scr[32 + g2], v);
        out[2 + e2] = v;
      }
    }
    ++npend;
    __syncthreads();  // the scratch stage, qsm and the unit record are reused
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
