// Persistent decode pass over the shared block (see pass.cuh for the design).
#include <algorithm>

#include "gemm_epi.cuh"
#include "pass.cuh"
#include "tc.cuh"

namespace lt {

namespace {

// Relaxed poll of a counter written by other CTAs (release side: red.release).
__device__ __forceinline__ unsigned ld_relaxed(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Acquire side of the polls (after the counters were seen complete).
__device__ __forceinline__ void fence_acquire() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}
// Makes data observed through the generic proxy visible to this thread's later
// TMA (async proxy) reads.
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void group_sync(int g) {
  asm volatile("bar.sync %0, 128;" ::"r"(1 + g) : "memory");
}

// Units of one GEMM, as the kernel walks them: (layer, gemm, unit).
struct Cursor {
  int l, g, u;
};

}  // namespace

template <int NC, int HD>
__global__ void __launch_bounds__(PASS_THREADS, 1) k_pass(const __grid_constant__ PassParams P) {
  using T = __nv_bfloat16;
  __shared__ EpiSmem esm;
  __shared__ AttnSmem<HD> asmem[PASS_GROUPS];
  __shared__ int s_item[PASS_GROUPS][4];
  __shared__ int s_ok[PASS_GROUPS];
  __shared__ int s_nsplit;  // attention items per head (sum of the rows' splits)
  __shared__ int s_nrows;
  constexpr uint32_t A_BYTES = GEMM_BM * GEMM_CHUNK_BYTES;
  constexpr uint32_t B_BYTES = NC * GEMM_CHUNK_BYTES;
  constexpr int BKE = 64;
  constexpr int TCOLS = tmem_cols<NC>();
  constexpr uint32_t IDESC = instr_desc<false, NC>();
  const int KC = P.sh[0].kc;
  const int stages = P.stages;
  const uint32_t SA = KC * A_BYTES, SB = KC * B_BYTES;
  const int L = P.n_layers;
  const int c = blockIdx.x, G = gridDim.x;

  if (P.run_flag != nullptr && *P.run_flag == 0) return;  // same for every CTA

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t a_base = base;
  const uint32_t b_base = base + stages * SA;
  const uint32_t bar_base = b_base + stages * SB;
  auto full_bar = [&](int i) { return bar_base + 8u * i; };
  auto empty_bar = [&](int i) { return bar_base + 8u * (stages + i); };
  auto accf_bar = [&](int i) { return bar_base + 8u * (2 * stages + i); };
  auto acce_bar = [&](int i) { return bar_base + 8u * (2 * stages + 2 + i); };
  const uint32_t drain_bar = bar_base + 8u * (2 * stages + 4);
  uint8_t* misc = gbase + (bar_base - base) + 8u * (2 * stages + 5);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);

  // this CTA's unit range of each GEMM
  int u0[4], u1[4];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const GemmShape& s = P.sh[g];
    u0[g] = c < s.grid ? sk_u0(c, s.units, s.grid) : 0;
    u1[g] = c < s.grid ? sk_u0(c + 1, s.units, s.grid) : 0;
  }
  int per_layer = 0;
#pragma unroll
  for (int g = 0; g < 4; ++g) per_layer += u1[g] - u0[g];
  const int total = L * per_layer;  // stages this CTA runs

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
  }
  if (threadIdx.x == 64) {
    int na = 0, nsplit = 0;
    for (int i = 0; i < P.C; ++i)
      if (P.mask[i]) {
        esm.rows[na++] = i;
        nsplit += (P.att.r_pos[i] + ATT_CH) / ATT_CH;
      }
    esm.nact = na;
    s_nrows = na;
    s_nsplit = nsplit;
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
  const int nrows = s_nrows;

  // --- unit geometry (see k_gemm) -------------------------------------------
  // returns 0 for a whole k-group (one 3-D box), else the chunks of a ragged group
  auto unit_of = [&](int g, int uu, int& t, int& c0) -> int {
    const GemmShape& s = P.sh[g];
    t = uu / s.kch;
    c0 = (uu - t * s.kch) * KC;
    return (KC > 1 && c0 + KC <= s.nfull) ? 0 : min(KC, s.nch - c0);
  };
  auto chunks_of = [&](int g, int uu) {
    int t, c0;
    const int n = unit_of(g, uu, t, c0);
    return n == 0 ? KC : n;
  };
  auto first_cursor = [&]() {
    Cursor cu = {0, 0, u0[0]};
    while (cu.l < L && cu.u >= u1[cu.g]) {
      if (++cu.g == 4) {
        cu.g = 0;
        ++cu.l;
      }
      cu.u = u0[cu.g];
    }
    return cu;
  };
  auto advance = [&](Cursor& cu) {
    ++cu.u;
    while (cu.l < L && cu.u >= u1[cu.g]) {
      if (++cu.g == 4) {
        cu.g = 0;
        ++cu.l;
      }
      cu.u = u0[cu.g];
    }
  };
  auto give_up = [&](long long t0) {
    if (clock64() - t0 > WAIT_LIMIT_CYCLES ||
        *reinterpret_cast<volatile int*>(P.err) == DEV_TIMEOUT) {
      *abort_flag = 1;
      return true;
    }
    return *abort_flag != 0;
  };
  // Are counters[lo..hi] (stride 1) all >= need[k] (or >= `all` when need is null)?
  // Up to 16 counters per round are loaded back to back before any compare, so
  // a round costs one memory round trip, not one per counter.
  auto complete = [&](const unsigned* ctr, const int* need, int lo, int hi, unsigned all) {
    bool ok = true;
    for (int k0 = lo; k0 <= hi; k0 += 16) {
      unsigned v[16], want[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int k = k0 + j;
        v[j] = k <= hi ? ld_relaxed(ctr + k) : 0xffffffffu;
        want[j] = k <= hi ? (need ? (unsigned)__ldg(need + k) : all) : 0u;
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) ok = ok && v[j] >= want[j];
    }
    return ok;
  };
  // Whether the activation rows of unit (l, g, uu) -- features f0..f1, or
  // (whole) all of K -- are complete.
  auto x_ready_range = [&](const Cursor& cu, bool whole) -> bool {
    int t, c0;
    const int n = unit_of(cu.g, cu.u, t, c0);
    const int K = P.sh[cu.g].k;
    const int f0 = whole ? 0 : c0 * BKE;
    const int f1 = whole ? K - 1 : min((c0 + (n == 0 ? KC : n)) * BKE, K) - 1;
    switch (cu.g) {
      case PG_QKV:  // Xd: the previous layer's down epilogue (layer 0: staged before the pass)
        if (cu.l == 0) return true;
        return complete(P.ctr + P.off_done[PG_D] + (cu.l - 1) * P.groups[PG_D], P.need[PG_D],
                        f0 >> 7, f1 >> 7, 0);
      case PG_O:  // Xo: every active row's merged attention of the heads in range
        return complete(P.ctr + P.off_att + cu.l * P.H, nullptr, f0 / HD, f1 / HD,
                        (unsigned)nrows);
      case PG_GU:  // Xm: the O epilogue
        return complete(P.ctr + P.off_done[PG_O] + cu.l * P.groups[PG_O], P.need[PG_O], f0 >> 7,
                        f1 >> 7, 0);
      default:  // Xf: the SwiGLU epilogue
        return complete(P.ctr + P.off_done[PG_GU] + cu.l * P.groups[PG_GU], P.need[PG_GU],
                        f0 >> 7, f1 >> 7, 0);
    }
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer: weights ahead, activations when ready ----------
      const uint64_t pol_w = policy_evict_first(), pol_x = policy_evict_last();
      Cursor cw = first_cursor(), cx = cw, cp = cw;
      int gw = 0, gx = 0, gp = 0;
      // (layer, gemm) whose whole activation input is known complete: its
      // remaining units need no poll
      int ready_l = -1, ready_g = -1;
      auto x_ready = [&](const Cursor& cu) -> bool {
        if (cu.l == ready_l && cu.g == ready_g) return true;
        if (!x_ready_range(cu, false)) return false;
        if (x_ready_range(cu, true)) {
          ready_l = cu.l;
          ready_g = cu.g;
        }
        return true;
      };
      long long t_prog = clock64();
      while (gx < total) {
        bool prog = false;
        // weights further ahead go to L2 (no shared memory needed), so HBM keeps
        // streaming while the ring waits on activations
        while (gp < total && gp < gw + P.l2_ahead) {
          const GemmOperand& W = P.layers[cp.l].w[cp.g];
          int t, c0;
          const int nc = unit_of(cp.g, cp.u, t, c0);
          if (nc == 0) {
            tma_prefetch_l2_3d(&W.group, t * GEMM_BM, c0);
          } else {
            for (int j = 0; j < nc; ++j) tma_prefetch_l2(&W.chunk, (c0 + j) * BKE, t * GEMM_BM);
          }
          ++gp;
          advance(cp);
        }
        if (gw < total && gw < gx + stages) {
          const int st = gw % stages, n = gw / stages;
          if (gw < stages || mbar_test(empty_bar(st), (n & 1) ^ 1)) {
            const GemmOperand& W = P.layers[cw.l].w[cw.g];
            int t, c0;
            const int nc = unit_of(cw.g, cw.u, t, c0);
            const uint32_t dst = a_base + st * SA;
            if (nc == 0) {
              mbar_expect_tx_only(full_bar(st), KC * A_BYTES);
              tma_load_3d(dst, &W.group, t * GEMM_BM, c0, full_bar(st), pol_w);
            } else {
              mbar_expect_tx_only(full_bar(st), nc * A_BYTES);
              for (int j = 0; j < nc; ++j)
                tma_load_2d(dst + j * A_BYTES, &W.chunk, (c0 + j) * BKE, t * GEMM_BM,
                            full_bar(st), pol_w);
            }
            ++gw;
            advance(cw);
            prog = true;
          }
        }
        if (gx < gw && x_ready(cx)) {
          fence_acquire();
          fence_proxy_async();
          const int st = gx % stages;
          const GemmOperand& X = P.x[cx.g];
          int t, c0;
          const int nc = unit_of(cx.g, cx.u, t, c0);
          const uint32_t dst = b_base + st * SB;
          if (nc == 0) {
            mbar_expect_tx(full_bar(st), KC * B_BYTES);
            tma_load_3d(dst, &X.group, 0, c0, full_bar(st), pol_x);
          } else {
            mbar_expect_tx(full_bar(st), nc * B_BYTES);
            for (int j = 0; j < nc; ++j)
              tma_load_2d(dst + j * B_BYTES, &X.chunk, (c0 + j) * BKE, 0, full_bar(st), pol_x);
          }
          ++gx;
          advance(cx);
          prog = true;
        }
        if (prog) {
          t_prog = clock64();
        } else if (give_up(t_prog)) {
          break;
        } else {
          __nanosleep(100);  // polls of hot counter lines slow their writers down
        }
      }
      // on abort: stages whose weights were requested but whose activations never
      // were get an arrival with no bytes, so their copies can land
      for (int gg = gx; gg < gw; ++gg) mbar_arrive(full_bar(gg % stages));
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      int gs = 0, seg = 0;
      bool ok = true;
      for (int l = 0; l < L && ok; ++l)
        for (int g = 0; g < 4 && ok; ++g) {
          const GemmShape& s = P.sh[g];
          for (int u = u0[g]; u < u1[g] && ok; ++seg) {
            const int t = u / s.kch;
            const int seg_end = min(u1[g], (t + 1) * s.kch);
            const int b = seg & 1, use = seg >> 1;
            if (!mbar_wait(acce_bar(b), (use & 1) ^ 1, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem + (uint32_t)(b * NC);
            for (int uu = u; uu < seg_end; ++uu, ++gs) {
              const int st = gs % stages, n = gs / stages;
              const int nchunk = chunks_of(g, uu);
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
                  tc_mma<false>(d_tmem, smem_desc(aj + 32u * kk), smem_desc(bj + 32u * kk), IDESC,
                                acc);
                }
              }
              tc_commit(empty_bar(st));
            }
            if (!ok) break;
            tc_commit(accf_bar(b));
            u = seg_end;
          }
        }
      tc_commit(drain_bar);
      volatile int dummy = 0;
      mbar_wait(drain_bar, 0, &dummy);
    }
  } else {
    // ---------------- groups: drains, epilogues (group 0) and attention items -------
    // Every decision a group takes (continue, stop) comes from one thread's
    // result shared through s_ok / s_item after a group barrier, so the 128
    // threads always reach the same named barriers (an abort seen by some
    // threads only would leave the others waiting at bar.sync for good).
    const int gi = (threadIdx.x - 64) >> 7;  // group
    const int et = (threadIdx.x - 64) & 127;  // thread within the group
    const int q = warp & 3;                   // TMEM lane quarter (group 0's warps 2..5)
    auto gsync = [gi] { group_sync(gi); };
    bool dead = false;  // uniform within the group
    // thread 0 waits for an mbarrier phase; the group shares the outcome
    auto gwait_mbar = [&](uint32_t bar, uint32_t parity) -> bool {
      if (et == 0) s_ok[gi] = mbar_wait(bar, parity, abort_flag) ? 1 : 0;
      gsync();
      return s_ok[gi] != 0;
    };
    // thread 0 waits until every counter lo..hi reaches its target, then orders
    // the group's later reads after the producers' writes
    auto wait_all = [&](const unsigned* ctr, const int* need, int lo, int hi, unsigned all) -> bool {
      if (et == 0) {
        const long long t0 = clock64();
        while (!complete(ctr, need, lo, hi, all)) {
          if (give_up(t0)) break;
          __nanosleep(100);
        }
        fence_acquire();
        s_ok[gi] = *abort_flag ? 0 : 1;
      }
      gsync();
      return s_ok[gi] != 0;
    };

    auto attention = [&](int l) {
      AttnArgs a = P.att;
      a.plane_base = P.layers[l].plane_base;
      const int items = P.H * s_nsplit;
      const int workers = PASS_GROUPS * G;
      for (int w = gi * G + c; w < items; w += workers) {
        const int h = w % P.H, k = w / P.H;
        if (et == 0) {
          const int3 r = attn_resolve(P.mask, a.r_pos, P.C, k);
          s_item[gi][0] = r.x;
          s_item[gi][1] = r.y;
          s_item[gi][2] = r.z;
          s_item[gi][3] = *abort_flag;
        }
        gsync();
        const int i = s_item[gi][0], sp = s_item[gi][1], ns = s_item[gi][2];
        if (i < 0 || s_item[gi][3]) {
          dead = s_item[gi][3] != 0;
          break;
        }
        auto dep = [&] {
          // q, k, v of head h: QKV tiles complete; the rows' sums of squares: the
          // previous layer's down epilogue (layer 0: staged before the pass)
          if (et == 0) {
            const long long t0 = clock64();
            const unsigned* arr = P.ctr + P.off_arr[PG_QKV] + l * P.groups[PG_QKV];
            bool qkv = false;
            while (true) {
              bool ok = true;
              if (!qkv) {
                for (int part = 0; part < 3; ++part) {
                  const int f0 = part * P.d + h * HD, f1 = f0 + HD - 1;
                  ok = ok && complete(arr, P.need[PG_QKV], f0 >> 7, f1 >> 7, 0);
                }
                qkv = ok;
              }
              if (ok && l > 0)
                ok = complete(P.ctr + P.off_done[PG_D] + (l - 1) * P.groups[PG_D], P.need[PG_D],
                              0, P.groups[PG_D] - 1, 0);
              if (ok || give_up(t0)) break;
              __nanosleep(100);
            }
            fence_acquire();
          }
          gsync();
        };
        const bool last =
            attn_item<T, HD, true, false>(a, asmem[gi], h, i, sp, ns, et, gsync, dep);
        if (last && et == 0) red_release_add(P.ctr + P.off_att + l * P.H + h, 1u);
      }
    };

    int seg = 0;
    for (int l = 0; l < L && !dead; ++l) {
      if (gi != 0) {
        attention(l);
        continue;
      }
      for (int g = 0; g < 4 && !dead; ++g) {
        if (g == PG_O) {
          attention(l);
          if (dead) break;
        }
        const GemmShape& s = P.sh[g];
        const int groups = P.groups[g];
        // drain this CTA's segments of GEMM g and publish them
        const int t0 = u0[g] / s.kch;
        for (int u = u0[g]; u < u1[g]; ++seg) {
          const int t = u / s.kch;
          const int seg_end = min(u1[g], (t + 1) * s.kch);
          const int b = seg & 1, use = seg >> 1;
          if (!gwait_mbar(accf_bar(b), use & 1)) {
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
          float* dst = P.part[g] + ((size_t)(c * s.jmax + (t - t0)) * NC) * GEMM_BM + q * 32 + lane;
#pragma unroll
          for (int i = 0; i < NC; ++i) dst[(size_t)i * GEMM_BM] = __uint_as_float(r[i]);
          gsync();
          if (et == 0) {
            const int grp = g == PG_GU ? t % groups : t;
            red_release_add(P.ctr + P.off_arr[g] + l * groups + grp, 1u);
          }
          u = seg_end;
        }
        if (g == PG_QKV || dead) continue;
        // group epilogues: every contributor takes a share of the active rows
        GemmEpi ep = P.epi[g];
        if (g == PG_O) ep.g = P.layers[l].g2;
        if (g == PG_D) ep.g = P.layers[l].g_next;
        if (g == PG_GU) {
          // the rows' RMSNorm factors need every tile of the O epilogue
          if (!wait_all(P.ctr + P.off_done[PG_O] + l * P.groups[PG_O], P.need[PG_O], 0,
                        P.groups[PG_O] - 1, 0)) {
            dead = true;
            break;
          }
          if (et < esm.nact)
            esm.inv[et] = inv_rms_parts(ep.ssq_in, ep.ssq_tiles, NC, esm.rows[et], ep.d, ep.eps);
          gsync();
        }
        if (u1[g] <= u0[g]) continue;
        const int nseg = (u1[g] - 1) / s.kch - t0 + 1;
        for (int sg = 0; sg < nseg; ++sg) {
          const int t = t0 + sg;
          const int grp = g == PG_GU ? t % groups : t;
          const int4 ta = __ldg(s.tinfo + grp);
          const int4 tb = g == PG_GU ? __ldg(s.tinfo + grp + groups) : ta;
          const int need = __ldg(P.need[g] + grp);
          const int share =
              g != PG_GU ? c - ta.x : (t < groups ? c - ta.x : (ta.y - ta.x + 1) + c - tb.x);
          if (!wait_all(P.ctr + P.off_arr[g] + l * groups, P.need[g], grp, grp, 0)) {
            dead = true;
            break;
          }
          const int r0 = share * esm.nact / need, r1 = (share + 1) * esm.nact / need;
          if (r1 > r0) {
            if (g != PG_GU)
              epi_resid<T>(ep, P.part[g], s, NC, t, ta, r0, r1, et, esm);
            else
              epi_swiglu<T>(ep, P.part[g], s, NC, grp, ta, tb, r0, r1, et, esm);
          }
          gsync();
          if (et == 0) red_release_add(P.ctr + P.off_done[g] + l * groups + grp, 1u);
        }
      }
    }
    if (dead && et == 0) *abort_flag = 1;
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    if (threadIdx.x == 0) {
      set_err(P.err, DEV_TIMEOUT);
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
size_t pass_ctr_layout(PassParams* p, int n_layers, int heads) {
  size_t off = 0;
  for (int g = 0; g < 4; ++g) {
    p->off_arr[g] = (int)off;
    off += (size_t)n_layers * p->groups[g];
  }
  for (int g = 0; g < 4; ++g) {
    p->off_done[g] = (int)off;
    if (g != PG_QKV) off += (size_t)n_layers * p->groups[g];
  }
  p->off_att = (int)off;
  off += (size_t)n_layers * heads;
  return off;
}

bool pass_supported(int ncols, int head_dim) {
  return (ncols == 8 || ncols == 16 || ncols == 32 || ncols == 64) &&
         (head_dim == 64 || head_dim == 96 || head_dim == 128);
}

int pass_stages(int ncols, int kc) {
  const int stage = kc * (GEMM_BM + ncols) * GEMM_CHUNK_BYTES;
  return std::min(4, (PASS_RING_BUDGET - 1024 - 256) / stage);
}

static size_t pass_smem_bytes(int ncols, int kc, int stages) {
  return 1024 + (size_t)stages * kc * (GEMM_BM + ncols) * GEMM_CHUNK_BYTES + 8 * (2 * stages + 5) +
         16;
}

template <int NC, int HD>
static cudaError_t launch_pass(const PassParams& p, cudaStream_t stream) {
  const size_t smem = pass_smem_bytes(NC, p.sh[0].kc, p.stages);
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  // function attributes belong to a context: remembered per device ordinal
  static size_t attr_bytes[64] = {};
  size_t& done = attr_bytes[dev >= 0 && dev < 64 ? dev : 0];
  if (smem > done) {
    cudaError_t e = cudaFuncSetAttribute(k_pass<NC, HD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    done = smem;
  }
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sms);
  cfg.blockDim = dim3(PASS_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the waits rely on it
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_pass<NC, HD>, p);
}

cudaError_t pass_launch(const PassParams& p, int ncols, int head_dim, cudaStream_t stream) {
#define LT_PASS_HD(N)                                              \
  switch (head_dim) {                                              \
    case 64: return launch_pass<N, 64>(p, stream);                 \
    case 96: return launch_pass<N, 96>(p, stream);                 \
    case 128: return launch_pass<N, 128>(p, stream);               \
    default: return cudaErrorInvalidValue;                         \
  }
  switch (ncols) {
    case 8: LT_PASS_HD(8)
    case 16: LT_PASS_HD(16)
    case 32: LT_PASS_HD(32)
    case 64: LT_PASS_HD(64)
    default: return cudaErrorInvalidValue;
  }
#undef LT_PASS_HD
}

}  // namespace lt
