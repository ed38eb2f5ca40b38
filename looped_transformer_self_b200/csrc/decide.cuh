// Readout processing, proposal / accept / resample decisions and on-device
// branch + KV-slot bookkeeping of the pipelined speculative decoder.
//
// Follows "LoopSpec: Pipelined Self-Speculative Decoding for Looped
// Transformers" (liuzhao09.github.io/papers/loopspec.html):
//  * section 2.1: the readout C = final norm, LM head, temperature, optional
//    top-p truncation, normalisation -- applied at every readout depth;
//  * section 2.2, Eqs. 2-4: residual operator, accept min(1, p/q), resample
//    from p (-) q; a branch opens a child at its depth-d1 proposal and is
//    verified at depth R; a rejection prunes every descendant of the wrong
//    prefix; the tree is re-rooted on every verification;
//  * section 2.3, Eqs. 5-6: gated residual second proposal and the cascade;
//  * section 2.4: a child copies its parent's cache indices; pruning frees
//    only slots no surviving path needs.
// Readings where the pages are silent (shared with the test oracle, which is
// written separately): greedy readouts are one-hot argmax (lowest index on
// ties); top-p keeps every token with p >= theta*, theta* the largest
// probability value whose upper set holds >= top_p of the mass; draws use the
// exponential race over Philox-4x32-10 words keyed (seed, uid|position,
// purpose); the accept test is u * q(x) < p(x) with 24-bit u; the per-step
// order is: prelude, iterate, readouts, proposals (ascending uid), verify,
// prune / re-root (frees after this step's allocations).
#pragma once

#include "common.cuh"
#include <climits>

#include "readout.cuh"
#include <cooperative_groups.h>

namespace lt {

constexpr int CMAX = 64;        // branch-table capacity limit (= max GEMM columns)
constexpr int WIN = 32;         // chain window: uncommitted positions a branch may span
constexpr int MAX_SLOT_WORDS = 2048;  // slot bitmap words held in shared memory (65536 slots)
constexpr int CPMAX = 32;       // longest copy proposal

struct Ctl {
  int L;              // committed length (prompt + generated)
  int target_len;     // generation stops when L reaches it
  int pos_limit;      // a child is created only for pos + 1 < pos_limit
  int next_uid;
  int finished;
  int ar_mode;        // 1: full-depth autoregressive (no proposals)
  int prepared;       // table depths hold the next iteration's depths
  int flag_run, flag_new, flag_ro;  // work present in the prepared step
  int rows_cur;
  int commit_pending, commit_tok, commit_src;
  int n_commit;       // commits logged since the log was reset
  int err;
  // statistics (Eq. 9's counts, Fig. 5 rows, Table 6 gate rate)
  int steps, rows_sum, rows_max, n_first, n_second, n_fallback;
  int gate_checks, gate_opens, branches_created, resid_fallback;
  int copy_chains, copy_rows, copy_cut, n_copy;
};

struct Dev {
  int d, V, R, C, S, d1, d2, greedy, second_mode, trace_cap, max_ctx;
  float T, top_p;
  unsigned long long seed;
  int tag_of_depth[33];
  // context-copy proposals (copy_k = 0: off)
  int copy_k, copy_max, copy_cap, copy_reserve, copy_slack;
  float copy_tau;
  Ctl* ctl;
  // branch table
  int *b_alive, *b_uid, *b_parent, *b_slot, *b_pos, *b_tok, *b_depth, *b_x1, *b_x2, *b_gate,
      *b_c1, *b_c2, *b_chain;
  int *b_copy;   // x1 is a copied token and child1 the next copied row
  int *b_crow;   // the entry's token was copied
  // written by k_decide for k_book: screen failures, copy proposals, verify outcomes
  int *cp_fail, *cp_len, *cp_tok;  // cp_tok [C][CPMAX]
  int *v_tok, *v_src, *v_fb;
  // rows of the prepared pass
  int *r_tok, *r_pos, *r_slot, *r_depth, *r_ro, *r_blen, *r_boff, *m_alive, *m_new, *m_ro;
  int* lists;      // committed slots
  int* committed;  // committed tokens
  unsigned int* slot_bits;
  int *log_tok, *log_src, *log_step;
  int* trace;      // [trace_cap][C][4]
  int* ro_arg;
  float *logits, *P, *q1, *q2, *rho, *rho2;
  float* cb_val;  // per readout row and logit chunk: the chunk's max logit
  int* cb_idx;    // and its index
};

// ---------------------------------------------------------------------------
// block helpers (arg-min / arg-max, suffix scan and readout processing: readout.cuh)
// ---------------------------------------------------------------------------
// Exponential race over weights w[0..V) (w_j <= 0 never chosen).
__device__ __forceinline__ int block_race(const float* __restrict__ w, int V,
                                          unsigned long long seed, uint32_t stream,
                                          uint32_t purpose, float* sk, int* si) {
  float best = INFINITY;
  int bi = 0x7fffffff;
  for (int j = threadIdx.x; j < V; j += blockDim.x) {
    const float wj = w[j];
    if (wj > 0.f) {
      const float k = race_key(seed, stream, purpose, (uint32_t)j, wj);
      if (better_min(k, j, best, bi)) {
        best = k;
        bi = j;
      }
    }
  }
  return block_arg<true>(best, bi, sk, si);
}

// ---------------------------------------------------------------------------
// K4: readout processing of LM-head partials.
// k_logits: logits of every readout row (final RMSNorm factor times the
// reduced head GEMM partials) and each chunk's argmax, spread over
// ceil(V / RO_CHUNK) blocks per row so the row's partials stream in parallel;
// k_readout (one block of 1024 per readout row): the row's argmax from its
// chunks (lowest index on ties, as one pass over the row would give), then
// the readout processing (temperature, top-p, normalisation).
// ---------------------------------------------------------------------------
constexpr int RO_CHUNK = 2048;
constexpr int RO_THREADS = 256;

__host__ __device__ constexpr int ro_chunks(int V) { return (V + RO_CHUNK - 1) / RO_CHUNK; }

__global__ void __launch_bounds__(RO_THREADS)
    k_logits(const float* __restrict__ part, const GemmShape s, int C,
             const int* __restrict__ mask, int V, float* __restrict__ logits,
             float* __restrict__ cb_val, int* __restrict__ cb_idx, const float* __restrict__ ssq,
             int ssq_tiles, int d, float eps) {
  __shared__ float sk[33];
  __shared__ int si[33];
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.y;
  if (!mask[i]) return;
  const int nch = ro_chunks(V);
  float* z = logits + (size_t)i * V;
  const float rr = inv_rms_parts(ssq, ssq_tiles, C, i, d, eps);  // final RMSNorm factor
  const int j0 = blockIdx.x * RO_CHUNK, j1 = min(V, j0 + RO_CHUNK);
  float best = -INFINITY;
  int bi = 0x7fffffff;
  // four elements per round so their partial loads overlap
  for (int jb = j0 + threadIdx.x; jb < j1; jb += 4 * RO_THREADS) {
    float v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = jb + u * RO_THREADS;
      v[u] = j < j1 ? rr * sk_reduce(part, s, C, i, j) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = jb + u * RO_THREADS;
      if (j < j1) {
        z[j] = v[u];
        if (better_max(v[u], j, best, bi)) {
          best = v[u];
          bi = j;
        }
      }
    }
  }
  const int a = block_arg<false>(best, bi, sk, si);
  if (threadIdx.x == 0) {
    const bool ok = a >= j0 && a < j1;  // false only when no value compared (NaN)
    cb_val[(size_t)i * nch + blockIdx.x] = ok ? z[a] : -INFINITY;
    cb_idx[(size_t)i * nch + blockIdx.x] = ok ? a : 0x7fffffff;
  }
}

__global__ void __launch_bounds__(1024)
    k_readout(const int* __restrict__ mask, int V, int greedy, float T, float top_p,
              float* __restrict__ logits, float* __restrict__ P, int* __restrict__ arg,
              const float* __restrict__ cb_val, const int* __restrict__ cb_idx, int* err) {
  __shared__ float sk[33];
  __shared__ int si[33];
  __shared__ DistSmem ds;
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x;
  if (!mask[i]) return;
  const int nch = ro_chunks(V);
  float best = -INFINITY;
  int bi = 0x7fffffff;
  for (int c = threadIdx.x; c < nch; c += blockDim.x) {
    const float v = cb_val[(size_t)i * nch + c];
    const int j = cb_idx[(size_t)i * nch + c];
    if (better_max(v, j, best, bi)) {
      best = v;
      bi = j;
    }
  }
  int a = block_arg<false>(best, bi, sk, si);
  if (a < 0 || a >= V) {  // every logit was NaN
    if (threadIdx.x == 0) set_err(err, DEV_BAD_INDEX);
    a = 0;
  }
  if (threadIdx.x == 0) arg[i] = a;
  if (greedy) return;
  readout_dist(logits + (size_t)i * V, P + (size_t)i * V, V, a, T, top_p, ds);
}

// Sampled readouts on a thread-block cluster: the same processing as
// k_readout (argmax from the chunk maxima, then softmax at T, the exact top-p
// cut and normalisation; LoopSpec page section 2.1), with each readout row
// spread over the RO_CL CTAs of one cluster instead of one block.  CTA rank r
// holds the row's slice [r * S, (r + 1) * S), S = ceil(V / RO_CL), in
// registers (thread t: elements t + k * 1024), so the row is read once.  The
// softmax sum, the three 1024-bin levels of the radix select over the float
// bits of p (integer 2^-40 masses) and the kept-mass sum are merged through
// distributed shared memory after cluster barriers, every CTA adding the
// partials in rank order: all CTAs take the same decisions, and the result
// does not depend on scheduling.  Rows without a readout exit as a whole
// cluster (the mask is read by every CTA), so all CTAs of a cluster meet at
// the same barriers.
constexpr int RO_CL = 8;          // CTAs per readout row (the portable cluster size)
constexpr int RO_CL_MAXK = 12;    // elements per thread held in registers (V <= 98304)
constexpr int RO_CL_MAXV = RO_CL * 1024 * RO_CL_MAXK;  // larger vocabularies use k_readout

__global__ void __launch_bounds__(1024)
    k_readout_cl(const int* __restrict__ mask, int V, float T, float top_p,
                 const float* __restrict__ logits, float* __restrict__ P,
                 int* __restrict__ arg, const float* __restrict__ cb_val,
                 const int* __restrict__ cb_idx, int* err) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ float sk[33];
  __shared__ int si[33];
  __shared__ float red[33];
  __shared__ unsigned long long hist[2][1024];  // radix levels alternate between the two
  __shared__ unsigned long long wsum[32];
  __shared__ float part[2];            // this CTA's softmax sum / kept-mass sum
  __shared__ int sel[2];
  __shared__ unsigned long long sel_above;
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.y;
  if (!mask[i]) return;  // the whole cluster (same row) returns
  const unsigned rank = cluster.block_rank();
  const int tid = threadIdx.x;
  const int nch = ro_chunks(V);
  // the row's argmax from its chunk maxima (every CTA; lowest index on ties)
  float best = -INFINITY;
  int bi = 0x7fffffff;
  for (int c = tid; c < nch; c += blockDim.x) {
    const float v = cb_val[(size_t)i * nch + c];
    const int j = cb_idx[(size_t)i * nch + c];
    if (better_max(v, j, best, bi)) {
      best = v;
      bi = j;
    }
  }
  int a = block_arg<false>(best, bi, sk, si);
  if (a < 0 || a >= V) {  // every logit was NaN
    if (tid == 0 && rank == 0) set_err(err, DEV_BAD_INDEX);
    a = 0;
  }
  if (tid == 0 && rank == 0) arg[i] = a;
  const float* z = logits + (size_t)i * V;
  const float zmax = z[a];
  const float invT = 1.f / T;
  const int S = (V + RO_CL - 1) / RO_CL;
  const int lo = (int)rank * S, hi = min(V, lo + S);
  float p[RO_CL_MAXK];
  float ssum = 0.f;
#pragma unroll
  for (int k = 0; k < RO_CL_MAXK; ++k) {
    const int j = lo + tid + k * 1024;
    p[k] = 0.f;
    if (j < hi) {
      p[k] = expf((z[j] - zmax) * invT);
      ssum += p[k];
    }
  }
  // softmax sum: block sums, merged in rank order
  {
    const float b = block_sum(ssum, red);
    if (tid == 0) part[0] = b;
  }
  cluster.sync();
  float Z = 0.f;
  for (int r = 0; r < RO_CL; ++r) Z += *cluster.map_shared_rank(&part[0], r);
  const float invZ = 1.f / Z;
#pragma unroll
  for (int k = 0; k < RO_CL_MAXK; ++k) p[k] *= invZ;
  float* out = P + (size_t)i * V;
  if (!(top_p < 1.f)) {
#pragma unroll
    for (int k = 0; k < RO_CL_MAXK; ++k) {
      const int j = lo + tid + k * 1024;
      if (j < hi) out[j] = p[k];
    }
    cluster.sync();  // no CTA leaves while a peer may still read its part[]
    return;
  }
  const double SCALE = 1099511627776.0;  // 2^40
  const unsigned long long target = (unsigned long long)((double)top_p * SCALE + 0.5);
  unsigned long long above = 0ull;
  uint32_t prefix = 0u;
  const int shifts[3] = {20, 10, 0};
  bool all = false;
  for (int lvl = 0; lvl < 3; ++lvl) {
    hist[lvl & 1][tid] = 0ull;
    __syncthreads();
    const int sh = shifts[lvl];
#pragma unroll
    for (int k = 0; k < RO_CL_MAXK; ++k) {
      const int j = lo + tid + k * 1024;
      if (j < hi) {
        const uint32_t b = __float_as_uint(p[k]);
        if (lvl == 0 || (b >> (sh + 10)) == prefix) {
          const unsigned long long m = (unsigned long long)((double)p[k] * SCALE + 0.5);
          atomicAdd(&hist[lvl & 1][(b >> sh) & 1023u], m);
        }
      }
    }
    cluster.sync();  // every CTA's histogram of this level is complete
    const int bin = 1023 - tid;
    unsigned long long hv = 0ull;
    for (int r = 0; r < RO_CL; ++r) hv += *cluster.map_shared_rank(&hist[lvl & 1][bin], r);
    // (a histogram buffer is reset two levels later, after the next level's
    // barrier, which every CTA passes only after these reads)
    const unsigned long long cum = suffix_scan_1024(hv, wsum);  // mass of bins >= bin
    if (tid == 0) sel[0] = -1;
    __syncthreads();
    if (above + cum >= target && above + cum - hv < target) {
      sel[0] = bin;
      sel_above = above + cum - hv;
    }
    __syncthreads();
    if (sel[0] < 0) {
      all = true;
      break;
    }
    above = sel_above;
    prefix = (prefix << 10) | (uint32_t)sel[0];
    __syncthreads();
  }
  const uint32_t theta = all ? 0u : prefix;
  float ks = 0.f;
#pragma unroll
  for (int k = 0; k < RO_CL_MAXK; ++k) {
    const int j = lo + tid + k * 1024;
    if (j < hi && __float_as_uint(p[k]) >= theta) ks += p[k];
  }
  {
    const float b = block_sum(ks, red);
    if (tid == 0) part[1] = b;
  }
  cluster.sync();
  float Z2 = 0.f;
  for (int r = 0; r < RO_CL; ++r) Z2 += *cluster.map_shared_rank(&part[1], r);
  const float inv2 = 1.f / Z2;
#pragma unroll
  for (int k = 0; k < RO_CL_MAXK; ++k) {
    const int j = lo + tid + k * 1024;
    if (j < hi) out[j] = __float_as_uint(p[k]) >= theta ? p[k] * inv2 : 0.f;
  }
  cluster.sync();  // no CTA leaves while a peer may still read its part[]
}

// ---------------------------------------------------------------------------
// K5: proposals at d1 / d2 and the verification cascade at R (one block per
// readout row).  The table entry's x1 / gate / x2 and the q1 / q2 vectors are
// stored for the verification at R (D5 of the branch state).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float residual_into(const float* __restrict__ mu,
                                               const float* __restrict__ nu, int V,
                                               float* __restrict__ out, float* red) {
  float zs = 0.f;
  for (int j = threadIdx.x; j < V; j += blockDim.x) {
    const float w = fmaxf(mu[j] - nu[j], 0.f);
    out[j] = w;
    zs += w;
  }
  const float Z = block_sum(zs, red);
  if (Z > 0.f) {
    const float inv = 1.f / Z;
    for (int j = threadIdx.x; j < V; j += blockDim.x) out[j] *= inv;
  }
  __syncthreads();
  return Z;
}

// Parent value of a retiring entry: a former root left behind by an external
// commit.  It keeps running one iteration per step and its readouts, so its
// committed position gets its block and coda cache rows at every depth before
// any later row reads them, but it decides nothing (k_decide skips it), is
// never pruned, and leaves the table (keeping its slot, which holds a
// committed position) after its R-th iteration.
constexpr int BK_RETIRING = -2;

// Block-wide maximum of an int (every thread gets it).
__device__ __forceinline__ int block_max_int(int v, int* si) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = __reduce_max_sync(0xffffffffu, v);
  __syncthreads();
  if (lane == 0) si[w] = v;
  __syncthreads();
  if (w == 0) {
    int t = lane < nw ? si[lane] : INT_MIN;
    t = __reduce_max_sync(0xffffffffu, t);
    if (lane == 0) si[32] = t;
  }
  __syncthreads();
  return si[32];
}

// Screen score of token s (CopyLoop card: copied tokens are scored at a
// shallow depth): softmax of the row's logits z at T = 1, taken at s.
// a: the row's argmax.

// Copy proposal of entry i (position pos, L committed tokens): the end e of
// the earlier committed occurrence whose backward match with the prefix's end
// is longest (>= copy_k, capped at copy_cap; the most recent on ties), and
// the committed tokens after it (<= copy_max).  Returns the proposal's length
// (0: none) with its tokens in out[].  tail[]: shared memory, WIN entries.
__device__ int copy_lookup(const Dev& D, int i, int L, int* tail, int* si, int* out) {
  const int pos = D.b_pos[i];
  if (threadIdx.x == 0) {  // the prefix's uncommitted tokens, from the entry up its ancestors
    int cur = i;
    for (int guard = 0; cur >= 0 && D.b_pos[cur] >= L && guard <= WIN; ++guard) {
      tail[D.b_pos[cur] - L] = D.b_tok[cur];
      const int pu = D.b_parent[cur];
      int nx = -1;
      if (pu >= 0)
        for (int k = 0; k < D.C; ++k)
          if (D.b_alive[k] && D.b_uid[k] == pu) nx = k;
      cur = nx;
    }
  }
  __syncthreads();
  const int* cm = D.committed;
  auto seq = [&](int t) { return t < L ? cm[t] : tail[t - L]; };
  int best = -1;  // m * 65536 + e (e < 65536: at most 65536 slots)
  for (int e = D.copy_k - 1 + (int)threadIdx.x; e <= L - 2; e += blockDim.x) {
    int m = 0;
    while (m < D.copy_cap && m <= e && seq(e - m) == seq(pos - m)) ++m;
    if (m >= D.copy_k) best = max(best, m * 65536 + e);
  }
  best = block_max_int(best, si);
  if (best < 0) return 0;
  const int e = best & 0xffff;
  const int n = min(D.copy_max, L - 1 - e);
  for (int t = threadIdx.x; t < n; t += blockDim.x) out[t] = cm[e + 1 + t];
  __syncthreads();
  return n;
}

__global__ void __launch_bounds__(1024) k_decide(Dev D) {
  __shared__ float sk[33];
  __shared__ int si[33];
  __shared__ float red[33];
  __shared__ int tail[WIN];
  __shared__ int prop[CPMAX];
  pdl_wait();
  pdl_trigger();
  Ctl* c = D.ctl;
  const int i = blockIdx.x;
  // rows without a readout, and retiring entries, decide nothing
  if (c->finished || !D.m_ro[i] || D.b_parent[i] == BK_RETIRING) return;
  const int r = D.r_depth[i];
  const int uid = D.b_uid[i];
  const bool ar = c->ar_mode != 0;
  const int V = D.V;
  const bool t0 = threadIdx.x == 0;
  const bool copied_x1 = !ar && D.b_copy[i];  // x1 is a copied token (child1 exists)
  const bool prop1 = !ar && r == D.d1;
  const bool prop2 = !ar && D.d2 > 0 && r == D.d2 && D.b_x1[i] >= 0 && !copied_x1;
  const float* z = D.logits + (size_t)i * V;
  const int a = D.ro_arg[i];
  // at depth d1: screen a copied x1, or propose (and look up a copy proposal)
  bool draw1 = prop1;
  if (prop1 && copied_x1) {
    const bool pass = copy_score(z, V, a, D.b_x1[i], red) >= D.copy_tau;
    if (t0) D.cp_fail[i] = !pass;
    draw1 = !pass;
  }
  if (prop1 && !copied_x1 && D.copy_k > 0) {
    int n = copy_lookup(D, i, c->L, tail, si, prop);
    if (n > 0 && copy_score(z, V, a, prop[0], red) < D.copy_tau) n = 0;
    if (t0) D.cp_len[i] = n;
    for (int t = threadIdx.x; t < n; t += blockDim.x) D.cp_tok[(size_t)i * CPMAX + t] = prop[t];
  }
  if (D.greedy) {
    if (!t0) return;
    if (draw1) D.b_x1[i] = a;
    if (prop2) {
      const int g = a != D.b_x1[i];
      D.b_gate[i] = g;
      D.b_x2[i] = g ? a : -1;
      atomicAdd(&c->gate_checks, 1);
      atomicAdd(&c->gate_opens, g);
    }
    if (r == D.R) {
      int src = 0;
      if (!ar) {
        if (D.b_x1[i] >= 0 && a == D.b_x1[i]) src = 1;
        else if (D.b_gate[i] && a == D.b_x2[i]) src = 2;
      }
      D.v_tok[i] = a;
      D.v_src[i] = src;
      D.v_fb[i] = 0;
    }
    return;
  }
  const float* p = D.P + (size_t)i * V;
  float* q1 = D.q1 + (size_t)i * V;
  float* q2 = D.q2 + (size_t)i * V;
  if (draw1) {
    for (int j = threadIdx.x; j < V; j += blockDim.x) q1[j] = p[j];
    const int x1 = block_race(p, V, D.seed, (uint32_t)uid, P_PROP1, sk, si);
    if (t0) D.b_x1[i] = x1;
  }
  if (prop2) {
    const int x1 = D.b_x1[i];
    int open = 0;
    if (D.second_mode == 0) {  // gated residual (Eqs. 5-6)
      if (p[x1] < q1[x1]) open = residual_into(p, q1, V, q2, red) > 0.f;
    } else if (D.second_mode == 1) {  // residual, no gate (ablation)
      open = residual_into(p, q1, V, q2, red) > 0.f;
    } else {  // non-residual ablation (section 3.4): p_d2 with x1 removed, renormalised
      float zs = 0.f;
      for (int j = threadIdx.x; j < V; j += blockDim.x) {
        const float w = j == x1 ? 0.f : p[j];
        q2[j] = w;
        zs += w;
      }
      const float Z = block_sum(zs, red);
      if (Z > 0.f) {
        for (int j = threadIdx.x; j < V; j += blockDim.x) q2[j] /= Z;
        open = 1;
      }
      __syncthreads();
    }
    int x2 = -1;
    if (open) x2 = block_race(q2, V, D.seed, (uint32_t)uid, P_PROP2, sk, si);
    if (t0) {
      D.b_gate[i] = open;
      D.b_x2[i] = x2;
      atomicAdd(&c->gate_checks, 1);
      atomicAdd(&c->gate_opens, open);
    }
  }
  if (r != D.R) return;
  // verification at full depth (every row at R: a copied chain reaches R
  // together; the bookkeeping applies the outcomes in chain order)
  int x, src = 0, fb = 0;
  float* rho_i = D.rho + (size_t)i * V;
  float* rho2_i = D.rho2 + (size_t)i * V;
  if (ar) {
    x = block_race(p, V, D.seed, (uint32_t)(D.r_pos[i] + 1), P_AR, sk, si);
  } else if (D.b_x1[i] < 0) {
    x = block_race(p, V, D.seed, (uint32_t)uid, P_RES, sk, si);
  } else if (copied_x1) {
    // one-hot proposal: accept with probability p(x1), else draw from p without x1
    const int x1 = D.b_x1[i];
    const float u1 = uniform01(D.seed, (uint32_t)uid, P_ACC1);
    if (u1 < p[x1]) {
      x = x1;
      src = 1;
    } else {
      float zs = 0.f;
      for (int j = threadIdx.x; j < V; j += blockDim.x) {
        const float w = j == x1 ? 0.f : p[j];
        rho_i[j] = w;
        zs += w;
      }
      const float Z = block_sum(zs, red);
      const float* rho1 = rho_i;
      if (Z > 0.f) {
        const float inv = 1.f / Z;
        for (int j = threadIdx.x; j < V; j += blockDim.x) rho_i[j] *= inv;
      } else {
        rho1 = p;  // unreachable: p(x1) = 1 always accepts
        fb = 1;
      }
      __syncthreads();
      x = block_race(rho1, V, D.seed, (uint32_t)uid, P_RES, sk, si);
    }
  } else {
    const int x1 = D.b_x1[i];
    const float u1 = uniform01(D.seed, (uint32_t)uid, P_ACC1);
    if (u1 * q1[x1] < p[x1]) {
      x = x1;
      src = 1;
    } else {
      const float* rho1 = rho_i;
      if (!(residual_into(p, q1, V, rho_i, red) > 0.f)) {
        rho1 = p;  // unreachable in exact arithmetic
        fb = 1;
      }
      const int x2 = D.b_x2[i];
      if (D.b_gate[i] && x2 >= 0) {
        const float u2 = uniform01(D.seed, (uint32_t)uid, P_ACC2);
        if (u2 * q2[x2] < rho1[x2]) {
          x = x2;
          src = 2;
        } else {
          const float* r2 = rho2_i;
          if (!(residual_into(rho1, q2, V, rho2_i, red) > 0.f)) {
            r2 = rho1;
            fb += 1;
          }
          x = block_race(r2, V, D.seed, (uint32_t)uid, P_RES, sk, si);
        }
      } else {
        x = block_race(rho1, V, D.seed, (uint32_t)uid, P_RES, sk, si);
      }
    }
  }
  if (t0) {
    D.v_tok[i] = x;
    D.v_src[i] = src;
    D.v_fb[i] = fb;
  }
}

// The sampled path of k_decide on a thread-block cluster of RO_CL CTAs per
// readout row (greedy decoding keeps k_decide: it needs only the argmax).  CTA
// rank r owns the slice [r * S, (r + 1) * S) of every V-long vector of the row
// (q1, q2, the residuals) and only ever touches that slice, so no CTA reads
// another's global writes; sums merge in rank order through distributed shared
// memory, and an exponential race takes each CTA's (key, index) winner and the
// smallest key over the cluster (lowest index on ties) -- the same token a
// race over the whole row picks.  A residual's value at one index is recomputed
// from its definition where a decision needs it.  Every decision comes from
// cluster-wide values, so all CTAs of a row take the same branches and meet at
// the same cluster barriers; scalar state is written by rank 0 only.
__global__ void __launch_bounds__(1024) k_decide_cl(Dev D) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ float sk[33];
  __shared__ int si[33];
  __shared__ float red[33];
  __shared__ int tail[WIN];
  __shared__ int prop[CPMAX];
  __shared__ float slot_f[2];  // block partials of cluster reductions (alternating)
  __shared__ int slot_i[2];
  pdl_wait();
  pdl_trigger();
  Ctl* c = D.ctl;
  const int i = blockIdx.y;
  // rows without a readout, and retiring entries, decide nothing (the whole cluster)
  if (c->finished || !D.m_ro[i] || D.b_parent[i] == BK_RETIRING) return;
  const int tid = threadIdx.x;
  const unsigned rank = cluster.block_rank();
  const bool lead = rank == 0 && tid == 0;
  const int r = D.r_depth[i];
  const int uid = D.b_uid[i];
  const bool ar = c->ar_mode != 0;
  const int V = D.V;
  const int S = (V + RO_CL - 1) / RO_CL;
  const int lo = (int)rank * S, hi = min(V, lo + S);
  const bool copied_x1 = !ar && D.b_copy[i];
  const bool prop1 = !ar && r == D.d1;
  const bool prop2 = !ar && D.d2 > 0 && r == D.d2 && D.b_x1[i] >= 0 && !copied_x1;
  const float* z = D.logits + (size_t)i * V;
  const int a = D.ro_arg[i];
  int nred = 0;  // cluster reductions so far: the slot of the next one
  // a slot is written again two reductions later, after the barrier of the one
  // in between, which every CTA passes only after reading it
  auto csum = [&](float v) -> float {
    const float b = block_sum(v, red);
    const int sl = nred++ & 1;
    if (tid == 0) slot_f[sl] = b;
    cluster.sync();
    float t = 0.f;
    for (int q = 0; q < RO_CL; ++q) t += *cluster.map_shared_rank(&slot_f[sl], q);
    return t;
  };
  auto crace = [&](const float* w, uint32_t stream, uint32_t purpose) -> int {
    float best = INFINITY;
    int bi = 0x7fffffff;
    for (int j = lo + tid; j < hi; j += blockDim.x) {
      const float wj = w[j];
      if (wj > 0.f) {
        const float k = race_key(D.seed, stream, purpose, (uint32_t)j, wj);
        if (better_min(k, j, best, bi)) {
          best = k;
          bi = j;
        }
      }
    }
    const int loc = block_arg<true>(best, bi, sk, si);
    const int sl = nred++ & 1;
    if (tid == 0) {
      slot_i[sl] = loc;
      slot_f[sl] = loc < V ? race_key(D.seed, stream, purpose, (uint32_t)loc, w[loc]) : INFINITY;
    }
    cluster.sync();
    float bk = INFINITY;
    int bj = 0x7fffffff;
    for (int q = 0; q < RO_CL; ++q) {
      const float k2 = *cluster.map_shared_rank(&slot_f[sl], q);
      const int j2 = *cluster.map_shared_rank(&slot_i[sl], q);
      if (better_min(k2, j2, bk, bj)) {
        bk = k2;
        bj = j2;
      }
    }
    return bj;
  };
  // softmax of the row's logits at T = 1, at token s (the copy screen's score)
  auto cscore = [&](int s) -> float {
    const float zmax = z[a];
    float acc = 0.f;
    for (int j = lo + tid; j < hi; j += blockDim.x) acc += expf(z[j] - zmax);
    const float Z = csum(acc);
    return expf(z[s] - zmax) / Z;
  };
  // out = normalised (mu - nu)_+ over this CTA's slice; returns the cluster-wide mass
  auto cresidual = [&](const float* mu, const float* nu, float* out) -> float {
    float zs = 0.f;
    for (int j = lo + tid; j < hi; j += blockDim.x) {
      const float w = fmaxf(mu[j] - nu[j], 0.f);
      out[j] = w;
      zs += w;
    }
    const float Z = csum(zs);
    if (Z > 0.f) {
      const float inv = 1.f / Z;
      for (int j = lo + tid; j < hi; j += blockDim.x) out[j] *= inv;
    }
    return Z;
  };
  do {
    // at depth d1: screen a copied x1, or propose (and look up a copy proposal)
    bool draw1 = prop1;
    if (prop1 && copied_x1) {
      const bool pass = cscore(D.b_x1[i]) >= D.copy_tau;
      if (lead) D.cp_fail[i] = !pass;
      draw1 = !pass;
    }
    if (prop1 && !copied_x1 && D.copy_k > 0) {
      int n = copy_lookup(D, i, c->L, tail, si, prop);  // the same in every CTA
      if (n > 0 && cscore(prop[0]) < D.copy_tau) n = 0;
      if (lead) D.cp_len[i] = n;
      if (rank == 0)
        for (int t = tid; t < n; t += blockDim.x) D.cp_tok[(size_t)i * CPMAX + t] = prop[t];
    }
    const float* p = D.P + (size_t)i * V;
    float* q1 = D.q1 + (size_t)i * V;
    float* q2 = D.q2 + (size_t)i * V;
    if (draw1) {
      for (int j = lo + tid; j < hi; j += blockDim.x) q1[j] = p[j];
      const int x1 = crace(p, (uint32_t)uid, P_PROP1);
      if (lead) D.b_x1[i] = x1;
    }
    if (prop2) {
      const int x1 = D.b_x1[i];
      int open = 0;
      if (D.second_mode == 0) {  // gated residual (Eqs. 5-6)
        if (p[x1] < q1[x1]) open = cresidual(p, q1, q2) > 0.f;
      } else if (D.second_mode == 1) {  // residual, no gate (ablation)
        open = cresidual(p, q1, q2) > 0.f;
      } else {  // non-residual ablation (section 3.4): p_d2 with x1 removed, renormalised
        float zs = 0.f;
        for (int j = lo + tid; j < hi; j += blockDim.x) {
          const float w = j == x1 ? 0.f : p[j];
          q2[j] = w;
          zs += w;
        }
        const float Z = csum(zs);
        if (Z > 0.f) {
          for (int j = lo + tid; j < hi; j += blockDim.x) q2[j] /= Z;
          open = 1;
        }
      }
      int x2 = -1;
      if (open) x2 = crace(q2, (uint32_t)uid, P_PROP2);
      if (lead) {
        D.b_gate[i] = open;
        D.b_x2[i] = x2;
        atomicAdd(&c->gate_checks, 1);
        atomicAdd(&c->gate_opens, open);
      }
    }
    if (r != D.R) break;
    // verification at full depth
    int x, src = 0, fb = 0;
    float* rho_i = D.rho + (size_t)i * V;
    float* rho2_i = D.rho2 + (size_t)i * V;
    if (ar) {
      x = crace(p, (uint32_t)(D.r_pos[i] + 1), P_AR);
    } else if (D.b_x1[i] < 0) {
      x = crace(p, (uint32_t)uid, P_RES);
    } else if (copied_x1) {
      // one-hot proposal: accept with probability p(x1), else draw from p without x1
      const int x1 = D.b_x1[i];
      const float u1 = uniform01(D.seed, (uint32_t)uid, P_ACC1);
      if (u1 < p[x1]) {
        x = x1;
        src = 1;
      } else {
        float zs = 0.f;
        for (int j = lo + tid; j < hi; j += blockDim.x) {
          const float w = j == x1 ? 0.f : p[j];
          rho_i[j] = w;
          zs += w;
        }
        const float Z = csum(zs);
        const float* rho1 = rho_i;
        if (Z > 0.f) {
          const float inv = 1.f / Z;
          for (int j = lo + tid; j < hi; j += blockDim.x) rho_i[j] *= inv;
        } else {
          rho1 = p;  // unreachable: p(x1) = 1 always accepts
          fb = 1;
        }
        x = crace(rho1, (uint32_t)uid, P_RES);
      }
    } else {
      const int x1 = D.b_x1[i];
      const float u1 = uniform01(D.seed, (uint32_t)uid, P_ACC1);
      if (u1 * q1[x1] < p[x1]) {
        x = x1;
        src = 1;
      } else {
        const float Z1 = cresidual(p, q1, rho_i);
        const float* rho1 = rho_i;
        if (!(Z1 > 0.f)) {
          rho1 = p;  // unreachable in exact arithmetic
          fb = 1;
        }
        const int x2 = D.b_x2[i];
        if (D.b_gate[i] && x2 >= 0) {
          // rho1 at x2, from its definition (the owning CTA stores the same value)
          const float rho1_x2 = Z1 > 0.f ? fmaxf(p[x2] - q1[x2], 0.f) * (1.f / Z1) : p[x2];
          const float u2 = uniform01(D.seed, (uint32_t)uid, P_ACC2);
          if (u2 * q2[x2] < rho1_x2) {
            x = x2;
            src = 2;
          } else {
            const float* r2 = rho2_i;
            if (!(cresidual(rho1, q2, rho2_i) > 0.f)) {
              r2 = rho1;
              fb += 1;
            }
            x = crace(r2, (uint32_t)uid, P_RES);
          }
        } else {
          x = crace(rho1, (uint32_t)uid, P_RES);
        }
      }
    }
    if (lead) {
      D.v_tok[i] = x;
      D.v_src[i] = src;
      D.v_fb[i] = fb;
    }
  } while (false);
  cluster.sync();  // no CTA leaves while a peer may still read its shared memory
}

// First token after prefill: full-depth readout of the last prompt position,
// drawn with the stream (position P, AR) like every autoregressive draw.
__global__ void __launch_bounds__(1024) k_first_token(Dev D, int row, int P_len) {
  __shared__ float sk[33];
  __shared__ int si[33];
  pdl_wait();
  pdl_trigger();
  int x;
  if (D.greedy) x = D.ro_arg[row];
  else x = block_race(D.P + (size_t)row * D.V, D.V, D.seed, (uint32_t)P_len, P_AR, sk, si);
  if (threadIdx.x == 0) {
    D.committed[P_len] = x;
    D.ctl->L = P_len + 1;
  }
}

// ---------------------------------------------------------------------------
// K6: branch / KV-slot bookkeeping (one block; the tree logic runs on one
// thread over shared-memory copies of the table, which is <= 64 entries).
// mode 0: apply this step's proposals and commit, prune / re-root, prepare the
// next step.  mode 1: make sure a root exists and the next step is prepared.
// ---------------------------------------------------------------------------
struct BookSmem {
  int alive[CMAX], uid[CMAX], parent[CMAX], slot[CMAX], pos[CMAX], tok[CMAX], depth[CMAX],
      x1[CMAX], x2[CMAX], gate[CMAX], c1[CMAX], c2[CMAX], copy[CMAX], crow[CMAX];
  int chain[CMAX * WIN];
  unsigned int bits[MAX_SLOT_WORDS];
  int order[CMAX];
};

__device__ int bk_alloc_slot(BookSmem& b, int S, int* err) {
  const int words = (S + 31) >> 5;
  for (int w = 0; w < words; ++w) {
    const unsigned int v = b.bits[w];
    if (v != 0xffffffffu) {
      const int bit = __ffs(~v) - 1;
      const int s = w * 32 + bit;
      if (s >= S) break;
      b.bits[w] = v | (1u << bit);
      return s;
    }
  }
  set_err(err, DEV_SLOTS_FULL);
  return -1;
}
__device__ void bk_free_slot(BookSmem& b, int s) { b.bits[s >> 5] &= ~(1u << (s & 31)); }

__device__ int bk_new_entry(BookSmem& b, const Dev& D, Ctl& c, int parent_e, int pos, int tok,
                            int depth, bool prepared) {
  int e = -1;
  for (int k = 0; k < D.C; ++k)
    if (!b.alive[k]) {
      e = k;
      break;
    }
  if (e < 0) {
    set_err(&c.err, DEV_TABLE_FULL);
    return -1;
  }
  const int s = bk_alloc_slot(b, D.S, &c.err);
  if (s < 0) return -1;
  if (pos - (c.L - 1) >= WIN) {
    set_err(&c.err, DEV_CHAIN);
    return -1;
  }
  b.alive[e] = 1;
  b.uid[e] = c.next_uid++;
  b.parent[e] = parent_e >= 0 ? b.uid[parent_e] : -1;
  b.slot[e] = s;
  b.pos[e] = pos;
  b.tok[e] = tok;
  b.depth[e] = depth;
  b.x1[e] = b.x2[e] = -1;
  b.gate[e] = 0;
  b.c1[e] = b.c2[e] = -1;
  b.copy[e] = b.crow[e] = 0;
  if (parent_e >= 0)
    for (int k = 0; k < WIN; ++k) b.chain[e * WIN + k] = b.chain[parent_e * WIN + k];
  b.chain[e * WIN + (pos % WIN)] = s;
  c.branches_created++;
  (void)prepared;
  return e;
}

__device__ int bk_find_uid(const BookSmem& b, int C, int uid) {
  if (uid < 0) return -1;
  for (int k = 0; k < C; ++k)
    if (b.alive[k] && b.uid[k] == uid) return k;
  return -1;
}

// Is entry k in the subtree of entry r (r itself included)?  A descendant holds
// r's slot at r's position in its chain.
__device__ __forceinline__ bool bk_in_subtree(const BookSmem& b, int k, int r) {
  return k == r || (b.pos[k] > b.pos[r] && b.chain[k * WIN + (b.pos[r] % WIN)] == b.slot[r]);
}

// Removes entry r's subtree (r included) and frees its slots; returns the count.
__device__ int bk_prune_subtree(BookSmem& b, int C, int r) {
  int n = 0;
  for (int k = 0; k < C; ++k)
    if (b.alive[k] && k != r && bk_in_subtree(b, k, r)) {
      b.alive[k] = 0;
      bk_free_slot(b, b.slot[k]);
      ++n;
    }
  b.alive[r] = 0;
  bk_free_slot(b, b.slot[r]);
  return n + 1;
}

// Copy proposal of entry e at depth d1 (its x1 already drawn): allowed when no
// copied entry outside e's own ancestors is alive; cut to the free table rows
// beyond the reserve, to the uncommitted window (room left for the tail's
// children) and to the token budget.  Opens the chain: child1 of e and each
// row the child of the previous one, all at depth 0.  Returns whether it did.
__device__ bool bk_open_copy(BookSmem& b, const Dev& D, Ctl& c, int e) {
  const int C = D.C;
  int n = D.cp_len[e];
  if (n <= 0) return false;
  int alive = 0;
  for (int k = 0; k < C; ++k) {
    if (!b.alive[k]) continue;
    ++alive;
    if (b.crow[k] && b.parent[k] != BK_RETIRING && k != e && !bk_in_subtree(b, e, k)) return false;
  }
  n = min(n, C - alive - D.copy_reserve);
  n = min(n, WIN - 2 - (b.pos[e] - (c.L - 1)) - D.copy_slack);
  n = min(n, c.pos_limit - 1 - b.pos[e]);
  if (n < 1) return false;
  const int* tok = D.cp_tok + (size_t)e * CPMAX;
  c.copy_chains++;
  c.copy_rows += n;
  b.x1[e] = tok[0];
  b.copy[e] = 1;
  int par = e;
  for (int j = 0; j < n; ++j) {
    const int ch = bk_new_entry(b, D, c, par, b.pos[par] + 1, tok[j], 0, false);
    if (ch < 0) return true;  // error recorded
    b.crow[ch] = 1;
    b.c1[par] = b.uid[ch];
    if (par != e) {
      b.x1[par] = tok[j];
      b.copy[par] = 1;
    }
    par = ch;
  }
  return true;
}

__device__ void bk_logic(BookSmem& b, const Dev& D, Ctl& c, int mode, int arg) {
  const int C = D.C;
  if (mode == 2 || mode == 3) {
    // explicit edits between steps: 2 = roll back branch `arg` (uid) with its
    // subtree; 3 = commit child `arg` of the root without verification
    const int e = bk_find_uid(b, C, arg);
    int root = -1;
    for (int k = 0; k < C; ++k)
      if (b.alive[k] && b.pos[k] == c.L - 1) root = k;
    if (e < 0 || root < 0 || e == root || b.parent[e] == BK_RETIRING ||
        (mode == 3 && b.parent[e] != b.uid[root])) {
      set_err(&c.err, DEV_STATE);
      return;
    }
    if (mode == 2) {
      const int par = bk_find_uid(b, C, b.parent[e]);
      for (int k = 0; k < C; ++k)
        if (b.alive[k] && k != e && bk_in_subtree(b, k, e)) {
          b.alive[k] = 0;
          bk_free_slot(b, b.slot[k]);
        }
      b.alive[e] = 0;
      bk_free_slot(b, b.slot[e]);
      if (par >= 0) {
        if (b.c1[par] == arg) b.c1[par] = -1;
        if (b.c2[par] == arg) b.c2[par] = -1;
      }
      return;
    }
    if (c.L >= D.max_ctx) {
      set_err(&c.err, DEV_NO_ROOT);
      return;
    }
    D.committed[c.L] = b.tok[e];
    D.log_tok[c.n_commit] = b.tok[e];
    D.log_src[c.n_commit] = 3;
    D.log_step[c.n_commit] = c.steps;
    c.n_commit++;
    c.L++;
    for (int k = 0; k < C; ++k) {
      if (!b.alive[k] || bk_in_subtree(b, k, e) || b.parent[k] == BK_RETIRING) continue;
      if (k == root) {  // it has iterations left: it retires instead
        b.parent[k] = BK_RETIRING;
        b.c1[k] = b.c2[k] = b.x1[k] = b.x2[k] = -1;
        b.gate[k] = 0;
        continue;
      }
      b.alive[k] = 0;
      bk_free_slot(b, b.slot[k]);
    }
    b.parent[e] = -1;
    D.lists[c.L - 1] = b.slot[e];
    if (c.L >= c.target_len) c.finished = 1;
    return;
  }
  if (mode == 0 && c.prepared) {
    c.prepared = 0;
    c.steps++;
    c.rows_sum += c.rows_cur;
    c.rows_max = max(c.rows_max, c.rows_cur);
    for (int k = 0; k < C; ++k)  // retiring entries that ran their R-th iteration
      if (b.alive[k] && b.parent[k] == BK_RETIRING && b.depth[k] >= D.R) b.alive[k] = 0;
    int n = 0;
    for (int k = 0; k < C; ++k)
      if (b.alive[k]) b.order[n++] = k;
    for (int a = 1; a < n; ++a) {  // ascending uid
      const int v = b.order[a];
      int j = a - 1;
      while (j >= 0 && b.uid[b.order[j]] > b.uid[v]) {
        b.order[j + 1] = b.order[j];
        --j;
      }
      b.order[j + 1] = v;
    }
    if (!c.ar_mode) {
      for (int a = 0; a < n; ++a) {
        const int e = b.order[a];
        if (!b.alive[e] || b.parent[e] == BK_RETIRING) continue;  // pruned by a screen above
        // a child's position stays inside the token budget and the uncommitted window
        const bool spawn = b.pos[e] + 1 < c.pos_limit && b.pos[e] + 1 - (c.L - 1) < WIN;
        if (b.depth[e] == D.d1 && b.x1[e] >= 0) {
          if (b.copy[e]) {
            if (!D.cp_fail[e]) continue;  // the copied token goes on
            const int ch = bk_find_uid(b, C, b.c1[e]);
            if (ch >= 0) c.copy_cut += bk_prune_subtree(b, C, ch);
            b.copy[e] = 0;
            b.c1[e] = -1;
          } else if (spawn && D.copy_k > 0 && bk_open_copy(b, D, c, e)) {
            if (c.err) return;
            continue;
          }
          if (!spawn) continue;
          const int ch = bk_new_entry(b, D, c, e, b.pos[e] + 1, b.x1[e], 0, false);
          if (ch < 0) return;
          b.c1[e] = b.uid[ch];
        } else if (spawn && D.d2 > 0 && b.depth[e] == D.d2 && b.gate[e] && b.x2[e] >= 0) {
          const int ch = bk_new_entry(b, D, c, e, b.pos[e] + 1, b.x2[e], 0, false);
          if (ch < 0) return;
          b.c2[e] = b.uid[ch];
        }
      }
    }
    // verification outcomes (k_decide) of the root, repeated while the new
    // root also ran depth R in this step (a copied chain reaches R together)
    while (!c.finished) {
      int root = -1;
      for (int k = 0; k < C; ++k)
        if (b.alive[k] && b.pos[k] == c.L - 1 && b.parent[k] != BK_RETIRING) root = k;
      if (root < 0 || b.depth[root] != D.R) break;
      if (c.L >= D.max_ctx) {
        set_err(&c.err, DEV_NO_ROOT);
        return;
      }
      const int x = D.v_tok[root], src = D.v_src[root];
      if (D.v_fb[root]) c.resid_fallback += D.v_fb[root];
      D.committed[c.L] = x;
      D.log_tok[c.n_commit] = x;
      D.log_src[c.n_commit] = src;
      D.log_step[c.n_commit] = c.steps;
      c.n_commit++;
      c.L++;
      if (src == 1) {
        c.n_first++;
        c.n_copy += b.copy[root];
      } else if (src == 2) {
        c.n_second++;
      } else {
        c.n_fallback++;
      }
      const int surv = bk_find_uid(b, C, src == 1 ? b.c1[root] : src == 2 ? b.c2[root] : -1);
      for (int k = 0; k < C; ++k) {
        if (!b.alive[k] || b.parent[k] == BK_RETIRING) continue;
        const bool keep = surv >= 0 && bk_in_subtree(b, k, surv);
        if (!keep) {
          b.alive[k] = 0;
          if (k != root) bk_free_slot(b, b.slot[k]);
        }
      }
      if (surv >= 0) {
        b.parent[surv] = -1;
        D.lists[c.L - 1] = b.slot[surv];
      } else if (c.L < c.target_len) {
        const int e = bk_new_entry(b, D, c, -1, c.L - 1, x, 0, false);
        if (e < 0) return;
        D.lists[c.L - 1] = b.slot[e];
      }
      if (c.L >= c.target_len) c.finished = 1;
    }
    if (c.finished) return;
    for (int k = 0; k < C; ++k)  // every row that ran depth R has been verified
      if (b.alive[k] && b.parent[k] != BK_RETIRING && b.depth[k] >= D.R) {
        set_err(&c.err, DEV_STATE);
        return;
      }
    for (int k = 0; k < C; ++k)
      if (b.alive[k]) b.depth[k]++;
    c.prepared = 1;
  } else if (mode == 1) {
    if (c.finished) return;
    int root = -1;
    for (int k = 0; k < C; ++k)
      if (b.alive[k] && b.pos[k] == c.L - 1) root = k;
    if (root < 0) {
      const int e = bk_new_entry(b, D, c, -1, c.L - 1, D.committed[c.L - 1], c.prepared ? 1 : 0,
                                 c.prepared);
      if (e < 0) return;
      D.lists[c.L - 1] = b.slot[e];
    }
    if (!c.prepared) {
      for (int k = 0; k < C; ++k)
        if (b.alive[k]) b.depth[k]++;
      c.prepared = 1;
    }
  }
}

__global__ void __launch_bounds__(256) k_book(Dev D, int mode, int arg) {
  __shared__ BookSmem b;
  pdl_wait();
  pdl_trigger();
  Ctl* cg = D.ctl;
  const int C = D.C, words = (D.S + 31) >> 5;
  for (int k = threadIdx.x; k < C; k += blockDim.x) {
    b.alive[k] = D.b_alive[k];
    b.uid[k] = D.b_uid[k];
    b.parent[k] = D.b_parent[k];
    b.slot[k] = D.b_slot[k];
    b.pos[k] = D.b_pos[k];
    b.tok[k] = D.b_tok[k];
    b.depth[k] = D.b_depth[k];
    b.x1[k] = D.b_x1[k];
    b.x2[k] = D.b_x2[k];
    b.gate[k] = D.b_gate[k];
    b.c1[k] = D.b_c1[k];
    b.c2[k] = D.b_c2[k];
    b.copy[k] = D.b_copy[k];
    b.crow[k] = D.b_crow[k];
  }
  for (int k = threadIdx.x; k < C * WIN; k += blockDim.x) b.chain[k] = D.b_chain[k];
  for (int k = threadIdx.x; k < words; k += blockDim.x) b.bits[k] = D.slot_bits[k];
  __shared__ Ctl c;
  if (threadIdx.x == 0) c = *cg;
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!c.err) bk_logic(b, D, c, mode, arg);
    if (c.err) c.finished = 1;
    // rebuild the rows of the prepared step
    int rows = 0, any_new = 0, any_ro = 0;
    const bool on_all = c.prepared && !c.finished;
    for (int k = 0; k < C; ++k) {
      const int on = on_all && b.alive[k];
      const int dep = b.depth[k];
      int ro = -1;
      if (on && dep >= 1 && dep <= D.R) ro = c.ar_mode ? (dep == D.R ? D.tag_of_depth[D.R] : -1)
                                                      : D.tag_of_depth[dep];
      D.m_alive[k] = on;
      D.m_new[k] = on && dep == 1;
      D.m_ro[k] = ro >= 0;
      D.r_ro[k] = ro;
      D.r_tok[k] = b.tok[k];
      D.r_pos[k] = b.pos[k];
      D.r_slot[k] = b.slot[k];
      D.r_depth[k] = dep;
      D.r_blen[k] = c.L;
      D.r_boff[k] = 0;
      rows += on;
      any_new |= on && dep == 1;
      any_ro |= ro >= 0;
    }
    c.rows_cur = rows;
    c.flag_run = rows > 0;
    c.flag_new = any_new;
    c.flag_ro = any_ro;
    if (on_all && c.steps < D.trace_cap) {
      int n = 0;
      for (int k = 0; k < C; ++k)
        if (b.alive[k]) b.order[n++] = k;
      for (int a = 1; a < n; ++a) {
        const int v = b.order[a];
        int j = a - 1;
        while (j >= 0 && b.uid[b.order[j]] > b.uid[v]) {
          b.order[j + 1] = b.order[j];
          --j;
        }
        b.order[j + 1] = v;
      }
      int* tr = D.trace + (size_t)c.steps * C * 4;
      for (int a = 0; a < C; ++a) {
        const int e = a < n ? b.order[a] : -1;
        tr[4 * a + 0] = e >= 0 ? b.uid[e] : -1;
        tr[4 * a + 1] = e >= 0 ? b.slot[e] : -1;
        tr[4 * a + 2] = e >= 0 ? b.pos[e] : -1;
        tr[4 * a + 3] = e >= 0 ? b.depth[e] : -1;
      }
    }
    *cg = c;
  }
  __syncthreads();
  for (int k = threadIdx.x; k < C; k += blockDim.x) {
    D.b_alive[k] = b.alive[k];
    D.b_uid[k] = b.uid[k];
    D.b_parent[k] = b.parent[k];
    D.b_slot[k] = b.slot[k];
    D.b_pos[k] = b.pos[k];
    D.b_tok[k] = b.tok[k];
    D.b_depth[k] = b.depth[k];
    D.b_x1[k] = b.x1[k];
    D.b_x2[k] = b.x2[k];
    D.b_gate[k] = b.gate[k];
    D.b_c1[k] = b.c1[k];
    D.b_c2[k] = b.c2[k];
    D.b_copy[k] = b.copy[k];
    D.b_crow[k] = b.crow[k];
  }
  for (int k = threadIdx.x; k < C * WIN; k += blockDim.x) D.b_chain[k] = b.chain[k];
  for (int k = threadIdx.x; k < words; k += blockDim.x) D.slot_bits[k] = b.bits[k];
}

// Rows of one prefill chunk: prompt positions c0 .. c0+n-1 (slots = positions).
__global__ void k_prefill_rows(Dev D, int c0, int n, int P_len, int depth, int ro_tag) {
  pdl_wait();
  pdl_trigger();
  for (int k = threadIdx.x; k < D.C; k += blockDim.x) {
    const int on = k < n;
    D.m_alive[k] = on;
    D.m_new[k] = on && depth == 0;
    D.r_tok[k] = on ? D.committed[c0 + k] : 0;
    D.r_pos[k] = on ? c0 + k : 0;
    D.r_slot[k] = on ? c0 + k : 0;
    D.r_depth[k] = depth;
    D.r_ro[k] = on ? ro_tag : -1;
    D.m_ro[k] = on && ro_tag >= 0;
    D.r_blen[k] = P_len;
    D.r_boff[k] = 0;
  }
}

}  // namespace lt
