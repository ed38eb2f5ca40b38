// tcgen05 / TMEM / TMA weight-streaming GEMM (see gemm.cuh for the design).
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <type_traits>

#include "gemm.cuh"
#include "gemm_epi.cuh"
#include "tc.cuh"

namespace lt {

// ---------------------------------------------------------------------------
// kernel
// ---------------------------------------------------------------------------
// MODE 0: bf16 operands.  MODE 1: tf32 operands.  MODE 2: fp32 operands as
// hi + lo tf32 pairs (hi = value with the low 13 mantissa bits cleared, lo =
// the exact remainder); each k-step issues hi*hi + hi*lo + lo*hi, which keeps
// the products to ~2^-21 relative error (fp32-grade) on the tensor cores.
template <int MODE, int NC>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    k_gemm(const __grid_constant__ GemmOperand W, const __grid_constant__ GemmOperand Wlo,
           const __grid_constant__ GemmOperand X, const __grid_constant__ GemmOperand Xlo,
           float* __restrict__ part, const GemmShape s, const int stages,
           const int* __restrict__ run_flag, int* __restrict__ err, const GemmEpi ep,
           const __grid_constant__ GemmOperand Next, const GemmShape sNext) {
  using TX = typename std::conditional<MODE == 0, __nv_bfloat16, float>::type;
  __shared__ EpiSmem esm;
  constexpr bool TF32 = MODE != 0;
  constexpr int NSPLIT = MODE == 2 ? 2 : 1;
  constexpr uint32_t A_BYTES = GEMM_BM * GEMM_CHUNK_BYTES;  // one chunk of one tile
  constexpr uint32_t B_BYTES = NC * GEMM_CHUNK_BYTES;
  constexpr int BKE = TF32 ? 32 : 64;  // elements per k-chunk
  // stage layout: W [hi chunks 0..kc-1][lo chunks], X [hi chunks][lo chunks]
  const int KC = s.kc;
  const uint32_t SA = NSPLIT * KC * A_BYTES, SB = NSPLIT * KC * B_BYTES;  // per-stage bytes
  constexpr int TCOLS = tmem_cols<NC>();
  constexpr uint32_t IDESC = instr_desc<TF32, NC>();

  const int c = blockIdx.x;
  const int u0 = sk_u0(c, s.units, s.grid), u1 = sk_u0(c + 1, s.units, s.grid);
  if (u0 >= u1) {
    pdl_wait();
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t a_base = base;
  const uint32_t b_base = base + stages * SA;
  const uint32_t bar_base = b_base + stages * SB;  // 8-byte aligned
  // barriers: full[stages], empty[stages], accf[2], acce[2], drain
  auto full_bar = [&](int i) { return bar_base + 8u * i; };
  auto empty_bar = [&](int i) { return bar_base + 8u * (stages + i); };
  auto accf_bar = [&](int i) { return bar_base + 8u * (2 * stages + i); };
  auto acce_bar = [&](int i) { return bar_base + 8u * (2 * stages + 2 + i); };
  const uint32_t drain_bar = bar_base + 8u * (2 * stages + 4);
  uint8_t* misc = gbase + (bar_base - base) + 8u * (2 * stages + 5);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(full_bar(i), 1);
      mbar_init(empty_bar(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(accf_bar(i), 1);
      mbar_init(acce_bar(i), 128);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    const GemmOperand* ops[4] = {&W, &X, &Wlo, &Xlo};
    for (int o = 0; o < 2 * NSPLIT; ++o) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&ops[o]->chunk))
                   : "memory");
      if (KC > 1 && s.nfull >= KC)  // the 3-D view exists
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&ops[o]->group))
                     : "memory");
    }
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32((const void*)tmem_slot)),
                 "r"(TCOLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Unit uu = (tile t, k-group j): chunks c0 .. c0 + n - 1 of tile t.  A group
  // of kc whole chunks is one 3-D request per operand; a group that reaches
  // the end of K is one 2-D request per chunk (the ragged chunk zero-filled).
  auto unit_of = [&](int uu, int& t, int& c0) -> int {
    t = uu / s.kch;
    c0 = (uu - t * s.kch) * KC;
    return (KC > 1 && c0 + KC <= s.nfull) ? 0 : min(KC, s.nch - c0);  // 0: one 3-D box
  };
  auto load_w = [&](int uu, uint32_t dst, uint32_t bar, uint64_t pol) -> uint32_t {
    int t, c0;
    const int n = unit_of(uu, t, c0);
    if (n == 0) {
      tma_load_3d(dst, &W.group, t * GEMM_BM, c0, bar, pol);
      if constexpr (NSPLIT == 2) tma_load_3d(dst + KC * A_BYTES, &Wlo.group, t * GEMM_BM, c0, bar, pol);
      return NSPLIT * KC * A_BYTES;
    }
    for (int j = 0; j < n; ++j) {
      tma_load_2d(dst + j * A_BYTES, &W.chunk, (c0 + j) * BKE, t * GEMM_BM, bar, pol);
      if constexpr (NSPLIT == 2)
        tma_load_2d(dst + (KC + j) * A_BYTES, &Wlo.chunk, (c0 + j) * BKE, t * GEMM_BM, bar, pol);
    }
    return NSPLIT * n * A_BYTES;
  };
  auto w_bytes = [&](int uu) -> uint32_t {
    int t, c0;
    const int n = unit_of(uu, t, c0);
    return NSPLIT * (n == 0 ? KC : n) * A_BYTES;
  };
  auto load_x = [&](int uu, uint32_t dst, uint32_t bar, uint64_t pol) {
    int t, c0;
    const int n = unit_of(uu, t, c0);
    if (n == 0) {
      tma_load_3d(dst, &X.group, 0, c0, bar, pol);
      if constexpr (NSPLIT == 2) tma_load_3d(dst + KC * B_BYTES, &Xlo.group, 0, c0, bar, pol);
      return;
    }
    for (int j = 0; j < n; ++j) {
      tma_load_2d(dst + j * B_BYTES, &X.chunk, (c0 + j) * BKE, 0, bar, pol);
      if constexpr (NSPLIT == 2)
        tma_load_2d(dst + (KC + j) * B_BYTES, &Xlo.chunk, (c0 + j) * BKE, 0, bar, pol);
    }
  };
  auto x_bytes = [&](int uu) -> uint32_t {
    int t, c0;
    const int n = unit_of(uu, t, c0);
    return NSPLIT * (n == 0 ? KC : n) * B_BYTES;
  };

  // Weights do not depend on earlier kernels: the first `npre` stages of
  // weight tiles are requested before waiting on the preceding grid, so with
  // programmatic dependent launch this CTA's prologue and pipeline fill overlap
  // the kernels in front of it.  Their barriers get the weight bytes now
  // (expect_tx without arrival) and the activation bytes plus the arrival once
  // the activations may be read.
  const int npre = min(min(stages, s.prewait), u1 - u0);
  const uint64_t pol_w = policy_evict_first(), pol_x = policy_evict_last();
  if (warp == 0 && lane == 0) {
    for (int g = 0; g < npre; ++g) {
      mbar_expect_tx_only(full_bar(g), w_bytes(u0 + g));
      load_w(u0 + g, a_base + g * SA, full_bar(g), pol_w);
    }
    // The rest of this CTA's weight range goes to L2 now (often already there:
    // the GEMM in front of this one requested it), and so does this CTA's
    // slice of the NEXT GEMM's weights (sNext.units > 0), so HBM keeps
    // streaming weights through this kernel's tail and the kernels that follow
    // (attention, epilogues) until the next GEMM's ring is filled.
    const int nl2 = min(u1 - u0, npre + s.l2_own / (int)(KC * A_BYTES));
    for (int g = npre; g < nl2; ++g) {
      int t, c0;
      const int n = unit_of(u0 + g, t, c0);
      if (n == 0) {
        tma_prefetch_l2_3d(&W.group, t * GEMM_BM, c0);
        if constexpr (NSPLIT == 2) tma_prefetch_l2_3d(&Wlo.group, t * GEMM_BM, c0);
      } else {
        for (int j = 0; j < n; ++j) {
          tma_prefetch_l2(&W.chunk, (c0 + j) * BKE, t * GEMM_BM);
          if constexpr (NSPLIT == 2) tma_prefetch_l2(&Wlo.chunk, (c0 + j) * BKE, t * GEMM_BM);
        }
      }
    }
    if (sNext.units > 0 && c < sNext.grid) {
      const int v0 = sk_u0(c, sNext.units, sNext.grid), v1 = sk_u0(c + 1, sNext.units, sNext.grid);
      const int vend = min(v1, v0 + s.l2_next / (int)(sNext.kc * A_BYTES));
      for (int uu = v0; uu < vend; ++uu) {
        const int t = uu / sNext.kch, c0 = (uu - t * sNext.kch) * sNext.kc;
        if (sNext.kc > 1 && c0 + sNext.kc <= sNext.nfull) {
          tma_prefetch_l2_3d(&Next.group, t * GEMM_BM, c0);
        } else {
          for (int j = 0; j < min(sNext.kc, sNext.nch - c0); ++j)
            tma_prefetch_l2(&Next.chunk, (c0 + j) * BKE, t * GEMM_BM);
        }
      }
    }
  }
  pdl_wait();
  // the next kernels may become resident (and a following GEMM may prefetch
  // its weights) while this one streams
  pdl_trigger();
  const bool skip = run_flag != nullptr && *run_flag == 0;
  if (skip) {
    if (warp == 0 && lane == 0) {
      // let the prefetched weight tiles land before the CTA goes away
      volatile int dummy = 0;
      for (int g = 0; g < npre; ++g) {
        mbar_arrive(full_bar(g));
        mbar_wait(full_bar(g), 0, &dummy);
      }
    }
  } else if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int g = 0;
      for (int uu = u0; uu < u1; ++uu, ++g) {
        const int st = g % stages, n = g / stages;
        if (g < npre) {  // weights already requested
          mbar_expect_tx(full_bar(st), x_bytes(uu));
        } else {
          if (!mbar_wait(empty_bar(st), (n & 1) ^ 1, abort_flag)) break;
          mbar_expect_tx(full_bar(st), w_bytes(uu) + x_bytes(uu));
          load_w(uu, a_base + st * SA, full_bar(st), pol_w);
        }
        load_x(uu, b_base + st * SB, full_bar(st), pol_x);
      }
      // on abort: arrive on prefetched stages never reached so their loads can land
      for (int gg = g; gg < npre; ++gg) mbar_arrive(full_bar(gg));
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      int g = 0, seg = 0;
      bool ok = true;
      for (int u = u0; u < u1 && ok; ++seg) {
        const int t = u / s.kch;
        const int seg_end = min(u1, (t + 1) * s.kch);
        const int b = seg & 1, use = seg >> 1;
        if (!mbar_wait(acce_bar(b), (use & 1) ^ 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(b * NC);
        for (int uu = u; uu < seg_end; ++uu, ++g) {
          const int st = g % stages, n = g / stages;
          int tt, c0;
          const int nc = unit_of(uu, tt, c0);
          const int nchunk = nc == 0 ? KC : nc;
          if (!mbar_wait(full_bar(st), n & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = a_base + st * SA, b0 = b_base + st * SB;
          for (int j = 0; j < nchunk; ++j) {
            const uint32_t aj = a0 + j * A_BYTES, bj = b0 + j * B_BYTES;
#pragma unroll
            for (int kk = 0; kk < GEMM_CHUNK_BYTES / 32; ++kk) {
              const uint32_t acc = (uu > u || j > 0 || kk > 0) ? 1u : 0u;
              if constexpr (NSPLIT == 2) {
                // small cross terms first, then the leading product
                tc_mma<TF32>(d_tmem, smem_desc(aj + KC * A_BYTES + 32u * kk),
                             smem_desc(bj + 32u * kk), IDESC, acc);
                tc_mma<TF32>(d_tmem, smem_desc(aj + 32u * kk),
                             smem_desc(bj + KC * B_BYTES + 32u * kk), IDESC, 1u);
                tc_mma<TF32>(d_tmem, smem_desc(aj + 32u * kk), smem_desc(bj + 32u * kk), IDESC,
                             1u);
              } else {
                tc_mma<TF32>(d_tmem, smem_desc(aj + 32u * kk), smem_desc(bj + 32u * kk), IDESC,
                             acc);
              }
            }
          }
          tc_commit(empty_bar(st));
        }
        if (!ok) break;
        tc_commit(accf_bar(b));
        u = seg_end;
      }
      // let every issued MMA finish before TMEM can be released
      tc_commit(drain_bar);
      volatile int dummy = 0;
      mbar_wait(drain_bar, 0, &dummy);
    }
  } else if (warp >= 2) {
    // ---------------- drain: TMEM -> fp32 partials (+ group epilogue) ----------------
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int et = threadIdx.x - 64;  // 0..127 over the drain warps
    if (ep.kind != EPI_NONE) {
      if (et == 0) {
        int na = 0;
        for (int i = 0; i < NC; ++i)
          if (ep.mask[i]) esm.rows[na++] = i;
        esm.nact = na;
      }
      // table entries of every group this CTA may complete (static tables)
      const int t0 = u0 / s.kch, nseg = (u1 - 1) / s.kch - t0 + 1;
      if (et < nseg && et < 8) {
        const int t = t0 + et;
        if (ep.kind == EPI_SWIGLU) {
          const int groups = ep.ffn / GEMM_BM, g = t % groups;
          esm.ti[et][0] = __ldg(s.tinfo + g);
          esm.ti[et][1] = __ldg(s.tinfo + g + groups);
        } else {
          esm.ti[et][0] = __ldg(s.tinfo + t);
        }
      }
      drain_sync();
      // the SwiGLU's RMSNorm factors (sums of squares written by the GEMM in
      // front of this one) are ready now, long before the first accumulator
      if (ep.kind == EPI_SWIGLU && et < esm.nact)
        esm.inv[et] = inv_rms_parts(ep.ssq_in, ep.ssq_tiles, NC, esm.rows[et], ep.d, ep.eps);
    }
    // Thread 0 takes every continue / stop decision and shares it through
    // esm.okb / esm.ok after a drain barrier, so the 128 drain threads always reach the
    // same barriers (an abort seen by some threads only would strand the rest).
    bool dead = false;
    int seg = 0;
    for (int u = u0; u < u1; ++seg) {
      const int t = u / s.kch;
      const int seg_end = min(u1, (t + 1) * s.kch);
      const int b = seg & 1, use = seg >> 1;
      // (two slots: a slot is rewritten only after the next barrier, which every
      // thread passes after reading it)
      if (et == 0) esm.okb[seg & 1] = mbar_wait(accf_bar(b), use & 1, abort_flag) ? 1 : 0;
      drain_sync();
      if (!esm.okb[seg & 1]) {
        dead = true;
        break;
      }
      tc_fence_after();
      uint32_t r[NC];
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * NC);
#pragma unroll
      for (int j = 0; j < NC / 8; ++j) tmem_ld8(taddr + 8u * j, r + 8 * j);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(acce_bar(b));
      float* dst = part + ((size_t)(c * s.jmax + seg) * NC) * GEMM_BM + q * 32 + lane;
#pragma unroll
      for (int i = 0; i < NC; ++i) dst[(size_t)i * GEMM_BM] = __uint_as_float(r[i]);
      if (ep.kind != EPI_NONE) {
        // publish this segment: the barrier orders the drain threads' partial
        // stores before thread 0's release atomic (cumulativity)
        drain_sync();
        if (et == 0) {
          const int grp = ep.kind == EPI_SWIGLU ? t % (ep.ffn / GEMM_BM) : t;
          unsigned long long old;
          asm volatile("atom.release.gpu.global.add.u64 %0, [%1], 1;"
                       : "=l"(old)
                       : "l"(ep.counters + grp)
                       : "memory");
          // earlier launches left the counter at a multiple of need
          const unsigned long long need = (unsigned long long)__ldg(ep.need + grp);
          if (seg < GEMM_MAX_SEGS) esm.target[seg] = (old / need + 1) * need;
        }
      }
      u = seg_end;
    }
    // Group epilogues.  Every segment of a group takes a share of its active
    // rows (share k of n: rows [k*nact/n, (k+1)*nact/n)), so a group's
    // partials are read by all of its contributors at once rather than by the
    // last to arrive.  Shares start only after this CTA published all of its
    // segments; a CTA that waits has published everything, and the grid (<= one
    // CTA per SM) is wholly resident before any dependent grid launches, so the
    // waits form no cycle.
    if (ep.kind != EPI_NONE && !dead) {
      const int t0 = u0 / s.kch, nseg = min((u1 - 1) / s.kch - t0 + 1, GEMM_MAX_SEGS);
      const bool sw = ep.kind == EPI_SWIGLU;
      const int groups = sw ? ep.ffn / GEMM_BM : s.tiles;
      for (int sg = 0; sg < nseg; ++sg) {
        const int t = t0 + sg;
        const int grp = sw ? t % groups : t;
        const int4 ta = sg < 8 ? esm.ti[sg][0] : __ldg(s.tinfo + grp);
        const int4 tb = !sw ? ta : (sg < 8 ? esm.ti[sg][1] : __ldg(s.tinfo + grp + groups));
        const int need = __ldg(ep.need + grp);
        const int share = !sw ? c - ta.x : (t < groups ? c - ta.x : (ta.y - ta.x + 1) + c - tb.x);
        if (et == 0) {
          const unsigned long long target = esm.target[sg];
          const long long w0 = clock64();
          unsigned long long seen = 0;
          while (true) {
            asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(seen) : "l"(ep.counters + grp)
                         : "memory");
            if (seen >= target) break;
            // give up on a timeout here or in another CTA (whose group may never complete)
            if ((err && *reinterpret_cast<volatile int*>(err) == DEV_TIMEOUT) ||
                clock64() - w0 > WAIT_LIMIT_CYCLES) {
              *abort_flag = 1;
              break;
            }
          }
          esm.ok = *abort_flag ? 0 : 1;
        }
        drain_sync();
        if (!esm.ok) break;
        const int r0 = share * esm.nact / need, r1 = (share + 1) * esm.nact / need;
        if (r1 > r0) {
          if (!sw) epi_resid<TX>(ep, part, s, NC, t, ta, r0, r1, et, esm);
          else epi_swiglu<TX>(ep, part, s, NC, grp, ta, tb, r0, r1, et, esm);
        }
        drain_sync();
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    if (threadIdx.x == 0) {
      set_err(err, DEV_TIMEOUT);
      // give copies still in flight time to land before the CTA's smem is reused
      const long long t0 = clock64();
      while (clock64() - t0 < 4000000LL) {
      }
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TCOLS)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
GemmTuning gemm_tuning() {
  static GemmTuning t = [] {
    GemmTuning v;
    const char* e = getenv("LT_GEMM_KC");
    const int kc = e ? atoi(e) : 4;
    v.kc = (kc == 1 || kc == 2 || kc == 4) ? kc : 4;
    e = getenv("LT_GEMM_SMEM_KB");
    const int kb = e ? atoi(e) : (v.kc <= 2 ? 112 : 220);
    v.smem_budget = std::min(std::max(kb, 48), 224) * 1024;
    e = getenv("LT_GEMM_L2_OWN_KB");
    v.l2_own = std::max(0, e ? atoi(e) : 0) * 1024;
    e = getenv("LT_GEMM_L2_NEXT_KB");
    v.l2_next = std::max(0, e ? atoi(e) : 0) * 1024;
    e = getenv("LT_GEMM_PREWAIT");
    v.prewait = e ? std::max(0, atoi(e)) : 16;
    return v;
  }();
  return t;
}

static int stages_for(int ncols, int nsplit, int kc) {
  const int stage = nsplit * kc * (GEMM_BM + ncols) * GEMM_CHUNK_BYTES;
  const int st = (gemm_tuning().smem_budget - 1024 - 512) / stage;
  return std::min(st, 16);
}
static size_t smem_bytes(int ncols, int stages, int nsplit, int kc) {
  return 1024 + (size_t)stages * nsplit * kc * (GEMM_BM + ncols) * GEMM_CHUNK_BYTES +
         8 * (2 * stages + 5) + 16;
}

int gemm_kc(int ncols, bool f32) {
  const int nsplit = f32 ? 2 : 1;
  int kc = gemm_tuning().kc;
  while (kc > 1 && stages_for(ncols, nsplit, kc) < 2) kc /= 2;
  return kc;
}

int gemm_table_ints(int n_out, int k, bool f32, int ncols, int grid_cap) {
  GemmShape s;
  gemm_plan(n_out, k, f32, ncols, grid_cap, &s, nullptr, nullptr);
  return 2 * s.tiles + s.grid + 4 * s.tiles + 4;  // tile_c, cta_t0, (pad to 16 B), tinfo
}

int gemm_tinfo_offset(const GemmShape& s) {  // int offset of tinfo within the table block
  return ((2 * s.tiles + s.grid + 3) / 4) * 4;
}

void gemm_plan(int n_out, int k, bool f32, int ncols, int grid_cap, GemmShape* s, int* tile_c,
               int* cta_t0) {
  const int bke = f32 ? 32 : 64;
  s->n_out = n_out;
  s->k = k;
  s->kc = gemm_kc(ncols, f32);
  s->l2_own = gemm_tuning().l2_own;
  s->l2_next = gemm_tuning().l2_next;
  s->prewait = gemm_tuning().prewait;
  s->nch = (k + bke - 1) / bke;
  s->nfull = k / bke;
  s->kch = (s->nch + s->kc - 1) / s->kc;
  s->tiles = (n_out + GEMM_BM - 1) / GEMM_BM;
  s->units = s->tiles * s->kch;
  s->grid = std::min(grid_cap, s->units);
  int jmax = 1;
  for (int c = 0; c < s->grid; ++c) {
    const int u0 = sk_u0(c, s->units, s->grid), u1 = sk_u0(c + 1, s->units, s->grid);
    if (u1 > u0) jmax = std::max(jmax, (u1 - 1) / s->kch - u0 / s->kch + 1);
    if (cta_t0) cta_t0[c] = u0 / s->kch;
  }
  s->jmax = jmax;
  if (tile_c) {
    for (int t = 0; t < s->tiles; ++t) {
      tile_c[2 * t] = sk_cta_of(t * s->kch, s->units, s->grid);
      tile_c[2 * t + 1] = sk_cta_of(t * s->kch + s->kch - 1, s->units, s->grid);
    }
    // tinfo follows cta_t0 (rounded up to 16 bytes): (c_lo, c_hi, j of c_lo, 0)
    int* ti = tile_c + ((2 * s->tiles + s->grid + 3) / 4) * 4;
    for (int t = 0; t < s->tiles; ++t) {
      const int clo = tile_c[2 * t];
      ti[4 * t] = clo;
      ti[4 * t + 1] = tile_c[2 * t + 1];
      ti[4 * t + 2] = t - sk_u0(clo, s->units, s->grid) / s->kch;
      ti[4 * t + 3] = 0;
    }
  }
  s->tile_c = nullptr;
  s->cta_t0 = nullptr;
}

void gemm_group_need(const GemmShape& s, const int* tile_c_host, int group_tiles, int* need) {
  const int groups = group_tiles > 0 ? s.tiles / group_tiles : s.tiles;
  for (int g = 0; g < groups; ++g) need[g] = 0;
  for (int t = 0; t < s.tiles; ++t) {
    const int g = group_tiles > 0 ? t % groups : t;
    need[g] += tile_c_host[2 * t + 1] - tile_c_host[2 * t] + 1;
  }
}

size_t gemm_part_bytes(const GemmShape& s, int ncols) {
  return (size_t)s.grid * s.jmax * ncols * GEMM_BM * sizeof(float);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

int make_tmap(CUtensorMap* map, const void* base, bool f32, uint64_t rows, uint64_t k,
              uint32_t box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return -1;
  const uint32_t esz = f32 ? 4 : 2;
  if (((uintptr_t)base & 15) || ((k * esz) & 15) || box_rows == 0 || box_rows > 256) return -2;
  cuuint64_t dims[2] = {k, rows};
  cuuint64_t strides[1] = {k * esz};
  cuuint32_t box[2] = {GEMM_CHUNK_BYTES / esz, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -3;
}

// 3-D view of a K-major operand: (128-byte row piece, row, chunk), the chunk
// dimension stepping 128 bytes along K.  Only whole chunks are mapped, so a
// box never reads past a row's end.
static int make_group_map(CUtensorMap* map, const void* base, bool f32, uint64_t rows,
                          uint64_t k, uint32_t box_rows, int kc) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return -1;
  const uint32_t esz = f32 ? 4 : 2, bke = GEMM_CHUNK_BYTES / esz;
  if (((uintptr_t)base & 15) || ((k * esz) & 15) || box_rows == 0 || box_rows > 256) return -2;
  cuuint64_t dims[3] = {bke, rows, k / bke};
  cuuint64_t strides[2] = {k * esz, GEMM_CHUNK_BYTES};
  cuuint32_t box[3] = {bke, box_rows, (cuuint32_t)kc};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -3;
}

int make_operand(GemmOperand* op, const void* base, bool f32, uint64_t rows, uint64_t k,
                 uint32_t box_rows, int kc) {
  memset(op, 0, sizeof(*op));
  if (int e = make_tmap(&op->chunk, base, f32, rows, k, box_rows)) return e;
  const uint64_t bke = GEMM_CHUNK_BYTES / (f32 ? 4 : 2);
  if (kc > 1 && k / bke >= (uint64_t)kc)
    return make_group_map(&op->group, base, f32, rows, k, box_rows, kc);
  return 0;
}

template <int MODE, int NC>
static cudaError_t launch_t(const GemmOperand& W, const GemmOperand& Wlo, const GemmOperand& X,
                            const GemmOperand& Xlo, float* part, const GemmShape& s,
                            const int* run_flag, int* err, cudaStream_t stream, bool pdl,
                            const GemmEpi& ep, const GemmOperand& N, const GemmShape& sN) {
  const int nsplit = MODE == 2 ? 2 : 1;
  const int stages = stages_for(NC, nsplit, s.kc);
  if (stages < 1) return cudaErrorInvalidValue;
  const size_t smem = smem_bytes(NC, stages, nsplit, s.kc);
  // function attributes belong to a context: remembered per device ordinal
  static size_t attr_bytes[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  size_t& done = attr_bytes[dev >= 0 && dev < 64 ? dev : 0];
  if (smem > done) {
    cudaError_t e = cudaFuncSetAttribute(k_gemm<MODE, NC>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    done = smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(s.grid);
  cfg.blockDim = dim3(GEMM_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_gemm<MODE, NC>, W, Wlo, X, Xlo, part, s, stages, run_flag, err,
                            ep, N, sN);
}

cudaError_t gemm_launch(const GemmOperand& W, const GemmOperand& Wlo, const GemmOperand& X,
                        const GemmOperand& Xlo, float* part, const GemmShape& s, int ncols,
                        int mode, const int* run_flag, int* err, cudaStream_t stream, bool pdl,
                        const GemmEpi* epi, const GemmOperand* next_w,
                        const GemmShape* next_s) {
  GemmEpi none = {};
  none.kind = EPI_NONE;
  const GemmEpi& ep = epi ? *epi : none;
  GemmShape no_next = {};
  const bool has_next = next_w && next_s && mode != 2;
  const GemmShape& sN = has_next ? *next_s : no_next;
  const GemmOperand& N = has_next ? *next_w : W;
#define LT_GEMM_CASE(C)                                                                           \
  case C:                                                                                         \
    return mode == 2   ? launch_t<2, C>(W, Wlo, X, Xlo, part, s, run_flag, err, stream, pdl, ep, N, sN) \
           : mode == 1 ? launch_t<1, C>(W, Wlo, X, Xlo, part, s, run_flag, err, stream, pdl, ep, N, sN) \
                       : launch_t<0, C>(W, Wlo, X, Xlo, part, s, run_flag, err, stream, pdl, ep, N, sN);
  switch (ncols) {
    LT_GEMM_CASE(8)
    LT_GEMM_CASE(16)
    LT_GEMM_CASE(32)
    LT_GEMM_CASE(64)
    default:
      return cudaErrorInvalidValue;
  }
#undef LT_GEMM_CASE
}

__global__ void k_split_tf32(const float* __restrict__ src, float* __restrict__ hi,
                             float* __restrict__ lo, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const float v = src[i];
    const float h = __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
    hi[i] = h;
    lo[i] = v - h;
  }
}

cudaError_t split_tf32(const float* src, float* hi, float* lo, size_t n, cudaStream_t stream) {
  const int blocks = (int)std::min<size_t>((n + 255) / 256, 4096);
  k_split_tf32<<<blocks, 256, 0, stream>>>(src, hi, lo, n);
  return cudaGetLastError();
}

}  // namespace lt
