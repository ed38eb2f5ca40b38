// Weight-streaming GEMM for few rows on sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Computes partial sums of Y[i][n] = sum_k X[i][k] * W[n][k] for the <= 64
// active rows i of a decode step and every output feature n of one weight
// matrix W [n_out x K] (nn.Linear layout, K contiguous).  The shared block's
// weights are read from HBM once per step however many rows ride along, which
// is the point of batching every (branch, position, depth) row into one pass
// ("LoopSpec", liuzhao09.github.io/papers/loopspec.html, sections 1 and 2.2:
// the current position and the branches opened from shallow proposals call the
// same shared block and are merged into one batched execution).
//
// Design (B200):
//  * swap-AB: W is the MMA's A operand (M = 128 output features per tile), the
//    rows are the B operand (N = ncols = table capacity, 8..64).  The MMA always
//    runs all ncols columns, so a row's result never depends on how many other
//    rows are active (batch invariance: the speculative and full-depth paths
//    give bit-identical rows).
//  * stream-K: the (tile, k-group) units are split evenly over one CTA per SM;
//    each CTA streams its contiguous unit range through a TMA ring in shared
//    memory, issues tcgen05.mma from one thread into double-buffered TMEM
//    accumulators, and drains each finished tile segment (tcgen05.ld) as an
//    fp32 partial.  The consumer adds a tile's partials in CTA order (fixed
//    order: deterministic).  The partition depends only on (n_out, K, kc,
//    #SMs), never on the active row count.
//  * one TMA request per operand per stage.  A k-group is kc consecutive
//    128-byte k-chunks of a 128-row tile; a 3-D view of W (128-byte rows x
//    rows x chunks) loads the whole group as kc standard 128B-swizzled tiles
//    in one request.  On B200 an SM's TMA completes roughly one request per
//    ~0.6 us whatever its size up to 32 KB, so 16 KB requests cap an SM near
//    27 GB/s (~4 TB/s for the GPU) while 64 KB requests reach the HBM rate.
//    Groups that reach a ragged K tail fall back to one 2-D request per chunk.
//  * bf16 operands: kind::f16 with fp32 accumulate; fp32 operands: kind::tf32,
//    either one pass or split hi + lo (three MMAs per k-step, fp32-grade).
//  * K tails and n_out tails are zero-filled by TMA.
//  * every mbarrier wait is bounded (~1 s); on timeout the kernel records
//    DEV_TIMEOUT, lets in-flight copies and MMAs land, frees TMEM and returns.
#pragma once

#include "common.cuh"

namespace lt {

constexpr int GEMM_BM = 128;            // output features per tile (MMA M)
constexpr int GEMM_CHUNK_BYTES = 128;   // K bytes per k-chunk (one 128B-swizzle row)
constexpr int GEMM_THREADS = 192;       // warp 0: TMA, warp 1: MMA, warps 2-5: drain
constexpr int GEMM_MAX_SEGS = 16;       // tiles one CTA may touch in a GEMM with an epilogue

// Ring geometry: k-chunks per stage (kc in {1, 2, 4}) and the shared-memory
// budget of the ring.  Default: kc 4 in ~218 KB (three 72 KB stages at 16
// rows, one CTA per SM).  kc 2 in ~109 KB lets the next GEMM's CTA be resident
// beside this one, but measured slower on the Ouro-1.4B decode step (1.70 vs
// 1.56 ms).  LT_GEMM_KC and LT_GEMM_SMEM_KB override them (read once per
// process).
// Weight bytes per CTA requested into L2 ahead of use: l2_own for this GEMM's
// range beyond the ring, l2_next for the next GEMM's slice (default 0: with
// 64 KB stages the ring requested before the dependency wait already keeps
// HBM busy; LT_GEMM_L2_OWN_KB / LT_GEMM_L2_NEXT_KB override).
struct GemmTuning {
  int kc;
  int smem_budget;
  int l2_own;
  int l2_next;
  int prewait;  // ring stages of weights requested before the dependency wait (LT_GEMM_PREWAIT)
};
GemmTuning gemm_tuning();
// Chunks per unit for this operand width (kc reduced until two stages fit).
int gemm_kc(int ncols, bool f32);

// Plans the stream-K split of one weight matrix.  `grid_cap`: CTAs (#SMs);
// `ncols`: the activation width the GEMM will run with (sets kc).
// Fills the host copies of the reducer tables: tile_c [2*tiles], cta_t0 [grid]
// and, when tile_c_host is given, the tinfo block after them (see gemm_table_ints;
// the caller sizes tile_c_host with gemm_table_ints).
void gemm_plan(int n_out, int k, bool f32, int ncols, int grid_cap, GemmShape* s,
               int* tile_c_host, int* cta_t0_host);
// Table block of one shape: tile_c [2*tiles], cta_t0 [grid], pad, tinfo [4*tiles]
// (int4, 16-byte aligned when the block is).  gemm_plan fills it from tile_c_host.
int gemm_table_ints(int n_out, int k, bool f32, int ncols, int grid_cap);
int gemm_tinfo_offset(const GemmShape& s);

// The two TMA views of one K-major operand (rows x k, 128B swizzle): `chunk`
// is 2-D with a box of box_rows x 128 bytes; `group` is 3-D (128-byte rows,
// rows, whole chunks) with a box of box_rows x kc chunks, present when
// kc > 1 and K holds at least kc whole chunks.
struct GemmOperand {
  CUtensorMap chunk;
  CUtensorMap group;
};
int make_operand(GemmOperand* op, const void* base, bool f32, uint64_t rows, uint64_t k,
                 uint32_t box_rows, int kc);

// Launches the GEMM.  ncols in {8, 16, 32, 64}.  mode: 0 bf16, 1 tf32, 2 fp32 as
// split tf32 (Wlo / Xlo view the low parts; ignored otherwise).  run_flag
// (device, may be null): skip when *run_flag == 0.  pdl: launch with
// programmatic stream serialization.
// epi (may be null): in-GEMM epilogue run by the CTA completing each tile group.
// next_w / next_s (may be null): the weights of the GEMM that follows, whose
// slice each CTA requests into L2.
cudaError_t gemm_launch(const GemmOperand& W, const GemmOperand& Wlo, const GemmOperand& X,
                        const GemmOperand& Xlo, float* part, const GemmShape& s, int ncols,
                        int mode, const int* run_flag, int* err, cudaStream_t stream, bool pdl,
                        const GemmEpi* epi = nullptr, const GemmOperand* next_w = nullptr,
                        const GemmShape* next_s = nullptr);

// Segments that complete each epilogue group (host).  group_tiles 0: one group
// per tile; else groups = tiles / group_tiles and tile t belongs to t % groups
// (SwiGLU: gate tile t pairs with up tile t + groups).
void gemm_group_need(const GemmShape& s, const int* tile_c_host, int group_tiles, int* need);

// hi = src with the low 13 mantissa bits cleared (exact in tf32), lo = src - hi.
cudaError_t split_tf32(const float* src, float* hi, float* lo, size_t n, cudaStream_t stream);

size_t gemm_part_bytes(const GemmShape& s, int ncols);

}  // namespace lt
