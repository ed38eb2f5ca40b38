// One decode pass over the shared block as a single persistent kernel.
//
// The multi-kernel pass launches five kernels per layer (QKV GEMM, attention,
// O, gate/up and down GEMMs); each boundary waits for a whole grid to drain,
// so every layer pays several memory round trips with HBM idle, and the next
// GEMM's weight stream starts only when its CTA becomes resident.  Here one
// CTA per SM runs every phase of every layer:
//
//  * warp 0 streams weight tiles through the TMA ring continuously, across
//    phase and layer boundaries (weights never depend on activations), and
//    requests each unit's activation rows once the tiles they come from are
//    complete (per-tile counters written by the producing phase);
//  * warp 1 issues the tcgen05 MMAs in the same unit order;
//  * group 0 (warps 2-5) drains the accumulators into fp32 partials, publishes
//    them, and runs its share of each group epilogue (residual, SwiGLU);
//  * groups 0-1 (warps 2-9) run the attention work items of each layer.
//
// Work partition, summation orders and epilogue arithmetic are those of the
// multi-kernel pass (same stream-K plans, same tile reductions, same attention
// items), so both produce the same bits.  Dependencies always point to an
// earlier phase and every CTA is resident (cooperative launch, one CTA per SM),
// so the waits form no cycle; each wait is bounded (~1 s, then DEV_TIMEOUT).
#pragma once

#include "gemm.cuh"
#include "layers.cuh"

namespace lt {

// Two groups keep the register budget (~200 per thread at 320 threads) the
// attention item needs to hold its loads in flight; three groups capped it at
// 128 and doubled the item latency.
constexpr int PASS_GROUPS = 2;                         // 128-thread groups
constexpr int PASS_THREADS = 64 + 128 * PASS_GROUPS;   // + TMA and MMA warps
constexpr int PASS_RING_BUDGET = 200 * 1024;           // shared memory for the ring

enum : int { PG_QKV = 0, PG_O = 1, PG_GU = 2, PG_D = 3 };

// One shared-block layer as the pass kernel sees it (device array).
struct PassLayer {
  GemmOperand w[4];     // QKV, O, gate/up, down weights
  const void* g2;       // O epilogue: Xm = g2 (.) h
  const void* g_next;   // down epilogue: Xd = g_next (.) h (next layer's g1; null for the last)
  int plane_base;       // first cache plane of the layer
};

struct PassParams {
  GemmOperand x[4];     // activation rows of each GEMM: Xd, Xo, Xm, Xf
  const PassLayer* layers;
  int n_layers;
  int stages;           // ring stages (pass_smem_bytes)
  int l2_ahead;         // units of weights requested into L2 ahead of the ring
  GemmShape sh[4];      // stream-K plans (tables on the device)
  float* part[4];       // fp32 partials of each GEMM
  const int* need[4];   // per group: segments that complete it
  unsigned* ctr;        // per-pass counters, zeroed before the launch
  int off_arr[4];       // arrivals  [layer][group] of each GEMM
  int off_done[4];      // finished epilogue shares [layer][group] (O, gate/up, down)
  int off_att;          // merged attention rows [layer][head]
  int groups[4];        // groups of each GEMM (QKV and O / down: tiles; gate/up: ffn / 128)
  GemmEpi epi[4];       // epilogues of O, gate/up, down (g and X per layer in the kernel)
  AttnArgs att;         // attention items (plane_base per layer in the kernel)
  const int* mask;      // active rows
  const int* run_flag;  // skip the pass when *run_flag == 0
  int* err;
  int C, H, d, ffn;
};

// Counters one pass uses (u32), and their offsets (filled into p).
size_t pass_ctr_layout(PassParams* p, int n_layers, int heads);
// Whether a pass kernel exists for this row capacity and head size (bf16 only).
bool pass_supported(int ncols, int head_dim);
// Ring stages and dynamic shared memory of the pass kernel.
int pass_stages(int ncols, int kc);
cudaError_t pass_launch(const PassParams& p, int ncols, int head_dim, cudaStream_t stream);

}  // namespace lt
