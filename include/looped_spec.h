/*
 * looped_spec.h -- C ABI of a B200 (sm_100a) library for pipelined
 * self-speculative decoding of looped Transformers.
 *
 * The method is the one of "LoopSpec: Pipelined Self-Speculative Decoding for
 * Looped Transformers" (liuzhao09.github.io/papers/loopspec.html).  A looped LM
 * is a prelude P, one shared block B applied R times and a coda/readout C
 * (section 2.1, Eq. 1).  Each decode step makes ONE batched pass of B's weights
 * over every active branch, each at its own loop depth; shallow readouts at
 * depths d1 and d2 propose the next token and open child branches, and full
 * depth R verifies them (sections 2.2-2.3).
 *
 * Conventions for every call:
 *  - Device pointers ("d_") are owned by the caller and must stay valid while
 *    the handle uses them; host pointers ("h_") are read or written before the
 *    call returns.  The library never allocates device memory.
 *  - Work is ordered on the CUDA stream given at creation (or per call);
 *    calls that return host data synchronise that stream only.
 *  - Return value: LT_OK (0) or a negative LT_ERR_* code; lt_last_error()
 *    gives a text.  No C++ exception crosses this boundary.  A device-side
 *    invariant violation is reported as LT_ERR_DEVICE_CHECK by the call that
 *    observes it.
 */
#ifndef LOOPED_SPEC_H
#define LOOPED_SPEC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { LT_F32 = 0, LT_BF16 = 1 };

enum {
  LT_OK = 0,
  LT_ERR_ARG = -1,          /* null pointer, bad enum or out-of-range argument */
  LT_ERR_SHAPE = -2,        /* unsupported or inconsistent sizes */
  LT_ERR_CAPACITY = -3,     /* a buffer, branch table or slot pool is too small */
  LT_ERR_CUDA = -4,         /* a CUDA runtime call failed */
  LT_ERR_DEVICE_CHECK = -5, /* a kernel reported an invariant violation or timeout */
  LT_ERR_STATE = -6         /* call out of order (e.g. decode before prefill) */
};

/* Model shape (section 2.1, Eq. 1; section 3.1 for the Ouro / Raven families).
 * The layer reading: pre-norm RMSNorm (rms_eps), QKV, RoPE (rope_theta,
 * rotate-half, absolute positions), causal softmax attention, O projection,
 * RMSNorm, SwiGLU MLP; resid_scale s multiplies both sublayer outputs of the
 * shared-block layers (prelude and coda layers use 1). */
typedef struct {
  int dtype;      /* LT_F32 (tf32 tensor-core operands) or LT_BF16 */
  int d_model, n_heads, head_dim, ffn, vocab;
  int n_prelude;  /* Transformer layers of P (0: P is the embedding) */
  int n_core;     /* layers of the shared block B */
  int n_coda;     /* Transformer layers of C before the final norm + LM head */
  int R;          /* full loop depth, 1..32 */
  float rms_eps, rope_theta, resid_scale;
} lt_model_config;

/* Decoding settings (sections 2.2-2.3). */
typedef struct {
  int d1;              /* first proposal depth, 1 <= d1 < R (0: full-depth AR only) */
  int d2;              /* second proposal depth, d1 < d2 < R, or 0 (single proposal) */
  float temperature;   /* 0 = greedy */
  float top_p;         /* (0, 1]; applied at every readout depth */
  uint64_t seed;       /* Philox-4x32-10 key */
  int max_branches;    /* branch-table capacity = GEMM columns: 8, 16, 32 or 64 */
  int max_ctx;         /* max committed length (prompt + 1 + generated) */
  int max_new;         /* default token budget of lt_decode_step */
  int second_mode;     /* 0: gated residual (the method); 1: residual, no gate;
                          2: p_d2 with x1 masked, no gate (ablations, section 3.4) */
  int trace_steps;     /* steps whose branch rows are logged (0: none) */
  /* Context-copy proposals (CopyLoop card, kongchang.com: copied continuations
   * screened at a shallow depth before the full-depth verify).  copy_k = 0
   * disables them.  A branch at depth d1 whose prefix ends with the longest
   * earlier match (>= copy_k tokens, backward match capped at copy_match_cap)
   * of the committed context proposes the committed tokens that followed it
   * (<= copy_max_len <= 32) as a chain of rows opened together; a copied token
   * goes on only while its depth-d1 softmax probability (T = 1) is >= copy_tau;
   * copy_reserve table rows stay free for the ordinary tree.  Copied tokens are
   * verified with a one-hot proposal (accepted with probability p_R(x), else a
   * draw from p_R without x), and a step commits every chain row that reached
   * R and was accepted in order. */
  int copy_k, copy_max_len, copy_match_cap, copy_reserve;
  float copy_tau;
} lt_decode_config;

/* Per-decode statistics (section 3.2 Eq. 9 counts, Fig. 5, Table 6, Fig. 6). */
typedef struct {
  int steps;            /* batched shared-block passes */
  int rows_sum, rows_max;  /* active branches per pass: sum and peak */
  int n_first, n_second, n_fallback;  /* commit sources */
  int gate_checks, gate_opens;
  int branches_created;
  int resid_fallback;   /* residuals with zero mass (expected 0) */
  int committed_len;    /* committed length after the call */
  int copy_chains, copy_rows;  /* copy proposals opened, rows they opened */
  int copy_cut;         /* copied rows removed by the depth-d1 screen */
  int n_copy;           /* committed tokens that were copied (included in n_first) */
} lt_stats;

typedef struct lt_handle lt_handle;

/*
 * Workspace: every device buffer of a handle (branch table, row arrays, KV
 * pool [planes][slots][K|V][d_model], activations, GEMM partials, readout
 * vectors, RoPE table).  Caller allocates >= lt_workspace_bytes() bytes of
 * device memory and keeps it alive until lt_destroy.  Errors: LT_ERR_SHAPE
 * for unsupported sizes (head_dim not in {32,64,96,128}, max_branches not in
 * {8,16,32,64}, R > 32, rows not 16-byte multiples, ...).
 */
int lt_workspace_bytes(const lt_model_config* m, const lt_decode_config* dc, size_t* bytes);
/* Creates a handle on `stream` (a cudaStream_t, not the legacy default stream:
 * decode steps are captured in a CUDA graph). */
int lt_create(const lt_model_config* m, const lt_decode_config* dc, void* d_workspace,
              size_t bytes, void* stream, lt_handle** out);
/*
 * Weights (device, caller-owned, dtype of the model, row-major nn.Linear
 * layout [out][in], 16-byte aligned): embedding [vocab][d], final norm [d],
 * LM head [vocab][d]; d_layers holds 6 pointers per layer in the order
 * prelude layers, shared-block layers, coda layers:
 *   g1 [d], wqkv [3d][d] (q rows, then k, then v), wo [d][d], g2 [d],
 *   wgu [2 ffn][d] (gate rows, then up rows), wd [d][ffn].
 */
int lt_load_weights(lt_handle* h, const void* d_embed, const void* d_final_norm,
                    const void* d_head, const void* const* d_layers);
/*
 * Prefill (section 2.2): the prompt runs through P and all R depths of B,
 * filling the per-depth caches, and through C at every readout depth
 * {d1, d2, R} (coda caches); the first token is committed from the full-depth
 * readout of the last position (drawn with the stream (n, AR)).  Resets the
 * decoding state.  h_first: the committed token.  Optional: h_argmax
 * [n][n_tags] argmax of every readout; d_logits [n][n_tags][vocab] (device)
 * logits of every readout; n_tags = |{d1, d2, R} minus 0|, ascending depth.
 */
int lt_prefill(lt_handle* h, const int32_t* h_tokens, int n, int32_t* h_first,
               int32_t* h_argmax, float* d_logits);
/*
 * Decode n tokens from the current state.  ar_mode 0: pipelined speculative
 * decoding (sections 2.2-2.3: proposals at d1 / d2, gate, cascade verify at R,
 * prune / re-root, all on the device); ar_mode 1: full-depth autoregressive
 * decoding with the same kernels (the comparison baseline; section 3.1).
 * h_out: the n committed tokens.  st: statistics of this call (may be NULL).
 * Greedy speculative output equals greedy AR output bit for bit.
 */
int lt_generate(lt_handle* h, int ar_mode, int n, int32_t* h_out, lt_stats* st);
/* What one batched pass did (section 3.2 Eq. 9 counts and section 3.4's
 * mechanism statistics, per step). */
typedef struct {
  int step;             /* 1-based index of the pass within the current decode */
  int rows;             /* active branches the pass advanced */
  int n_committed;      /* tokens it committed (0 or 1; with copy proposals several) */
  int n_first, n_second, n_fallback;  /* their sources: first / second proposal, full-depth draw */
  int n_copy;           /* of n_first: copied tokens */
  int gate_checks, gate_opens;  /* second-proposal gates evaluated / opened */
  int branches_created; /* children opened */
  int committed_len;    /* committed length after the pass */
  int finished;         /* 1 when the decode reached its token budget */
} lt_step_info;
/* One batched pass (the first call after lt_prefill starts a decode of
 * max_new tokens, or fewer if max_ctx leaves less room).  *n_committed = the
 * tokens this pass committed and *h_tok = the last of them; info (may be NULL)
 * receives the pass's statistics.  Synchronises the handle's stream. */
int lt_decode_step(lt_handle* h, int ar_mode, int32_t* h_tok, int* n_committed,
                   lt_step_info* info);
/* Running totals of the current decode (or the last one, once it finished):
 * the counters of lt_stats since lt_generate or the decode's first
 * lt_decode_step began.  Errors: LT_ERR_STATE before the first prefill. */
int lt_get_stats(lt_handle* h, lt_stats* st);
/*
 * Explicit edits of the branch tree between two decode steps (after
 * lt_decode_step; the next step sees the edited tree).  The pages' own
 * commits and rollbacks happen inside each step on the device (section 2.2:
 * accept keeps the child's subtree, reject prunes every descendant of the
 * wrong prefix); these calls expose the same two operations to callers that
 * decide acceptance themselves (e.g. externally proposed continuations).
 *   lt_rollback_branch: prune branch `uid` (not the root) and its descendants,
 *     freeing their KV slots; its parent forgets the child.
 *   lt_commit_branch: commit the token of `uid`, which must be a child of the
 *     root, WITHOUT full-depth verification (logged with source 3); every
 *     branch outside its subtree is pruned and it becomes the root.  The old
 *     root has not run all R loop iterations yet, and later rows attend to
 *     its position at every depth, so it stays in the table as a retiring
 *     entry (parent -2 in lt_read_branch_table): it keeps iterating with the
 *     batch and taking its readouts (which write its coda cache rows), decides
 *     nothing, and leaves after its R-th iteration.
 * Errors: LT_ERR_ARG for an unknown uid, the root, a retiring entry, or
 * (commit) a non-child; LT_ERR_STATE when no decode is in progress.
 */
int lt_rollback_branch(lt_handle* h, int32_t uid);
int lt_commit_branch(lt_handle* h, int32_t uid);
/* Commit log of the last generate / decode calls: token, source (1 first
 * proposal, 2 second, 0 drawn at full depth) and 1-based step of each commit. */
int lt_read_log(lt_handle* h, int32_t* h_tok, int32_t* h_src, int32_t* h_step, int n);
/* Branch rows logged per step, [n_steps][max_branches][4] = (uid, slot, pos,
 * depth) sorted by uid, unused entries -1. */
int lt_read_trace(lt_handle* h, int32_t* h_trace, int n_steps);
/* Committed tokens and their KV slots (arrays of max_ctx ints). */
int lt_read_committed(lt_handle* h, int32_t* h_tokens, int32_t* h_slots, int* h_len);
/* Branch table, [12][max_branches]: alive, uid, parent uid, slot, pos, token,
 * depth, x1, x2, gate, child1 uid, child2 uid. */
int lt_read_branch_table(lt_handle* h, int32_t* h_table);
/* Last pass's readout rows: logits and processed probabilities [max_branches]
 * [vocab], argmax [max_branches].  Any pointer may be NULL; h_rows unused. */
int lt_read_readouts(lt_handle* h, float* h_logits, float* h_probs, int32_t* h_arg,
                     int32_t* h_rows);
/* Per-step timing of the next n_steps passes of the current decode (starting
 * one like lt_decode_step if needed), run without the CUDA graph and without
 * programmatic dependent launch, with CUDA events around every GEMM and
 * attention launch on the handle's stream.  Bytes are algorithmic: weights,
 * activation rows and results for GEMMs; (pos+2) K and V rows per row and
 * shared-block layer for the KV. */
typedef struct {
  int steps;
  int rows;                 /* active rows summed over the steps */
  double step_ms;           /* summed step times */
  double gemm_core_ms, gemm_core_bytes;  /* shared-block layer GEMMs */
  int gemm_core_launches;
  double gemm_other_ms;     /* prelude / coda / LM-head GEMMs */
  int gemm_other_launches;
  double gemm_other_bytes;
  double attn_ms;           /* attention + split combine */
  int attn_launches;
  double kv_bytes;          /* KV read + written by the shared-block layers */
  double weight_bytes_core; /* one pass of the shared block's GEMM weights */
} lt_profile;
int lt_profile_steps(lt_handle* h, int ar_mode, int n_steps, lt_profile* out);
/*
 * In-graph timing of the weight-streaming GEMM: the shared-block GEMMs of one
 * decode pass (per layer QKV, O + residual, gate/up + SwiGLU, down + residual;
 * LoopSpec page sections 1 and 2.2: the one batched pass of the shared block's
 * weights per step) are captured alone in a CUDA graph, in the decode step's
 * order and launch configuration (programmatic dependent launch between them),
 * over the rows of the handle's last step, and replayed n_iters times with
 * CUDA events on the handle's stream around the replays.  Attention and the
 * other kernels of a step are left out, so the GEMMs run back to back.
 * h_out (host, 3 doubles): [0] ms per replay, [1] algorithmic bytes per replay
 * (weights, activation rows, fp32 results), [2] GEMM launches per replay.
 * The epilogues overwrite the hidden states: the decode state is reset
 * (prefill again).  Synchronises the stream.  Errors: LT_ERR_ARG, LT_ERR_STATE
 * (weights not loaded), LT_ERR_CUDA, LT_ERR_DEVICE_CHECK.
 */
int lt_profile_gemms(lt_handle* h, int n_iters, double* h_out);

/* Static facts of a handle (captures the step graph if not done yet). */
typedef struct {
  int kernels_per_step;     /* kernel launches in one decode step (graph nodes) */
  int gemm_grid;            /* CTAs of the shared-block GEMMs (one per SM) */
  int n_tags;               /* readout depths */
  int kv_slots;
  double workspace_bytes;
  double weight_bytes_core, weight_bytes_prelude_coda, weight_bytes_head;
} lt_info;
int lt_get_info(lt_handle* h, lt_info* out);

/*
 * One shared-block pass over caller-specified rows (the mixed-depth step of
 * sections 1 / 2.2 in isolation, for kernel sweeps): row i sits at loop depth
 * h_depth[i] in 1..R and position h_pos[i]; it attends over the slots
 * d_lists[h_list_off[i] + j], j = 0..h_pos[i] (device int32; the last one is its
 * own slot, where its K/V rows are written) in the cache planes of its depth.
 * d_hidden [n_rows][d_model] fp32 (device) holds H^(r-1) on entry and H^(r)
 * after all n_core layers on return.  n_rows <= max_branches.  iters > 1 or
 * h_ms != NULL: the pass is captured once as a CUDA graph and replayed iters
 * times (each replay continues from the previous output), h_ms[k] = replay k's
 * time in ms (CUDA events on the handle's stream).  Resets any decode state.
 */
int lt_block_pass(lt_handle* h, int n_rows, const int32_t* h_depth, const int32_t* h_pos,
                  const int32_t* d_lists, const int32_t* h_list_off, float* d_hidden, int iters,
                  float* h_ms);
/* KV pool of a handle, for callers that fill caches (sweeps, tests): layout
 * [plane][slot][K|V][d_model] in the model dtype; the plane of shared-block
 * layer l at depth r is plane_core0 + l * R + (r - 1). */
int lt_kv_pool(lt_handle* h, void** d_pool, size_t* bytes, int* n_planes, int* n_slots,
               int* plane_core0);
int lt_reset(lt_handle* h);
const char* lt_last_error(const lt_handle* h);
void lt_destroy(lt_handle* h);

/*
 * Total variation between two readouts of the same positions (depth
 * selection, LoopSpec page, section 2.4, Eq. 7 and section 3.1, Fig. 3:
 * E_X[TV(p_r, p_R)] over positions, fitted by a power law, sets d1 and d2
 * through Eq. 8).  Row i of each input holds raw readout logits (e.g. the
 * d_logits of lt_prefill at depths r and R); both rows get the readout
 * processing of a decode step (temperature T, top-p, normalisation; section
 * 2.1) and d_tv[i] = 1/2 sum_j |p_a(j) - p_b(j)|.  T = 0: one-hot argmax
 * readouts, so d_tv[i] = 1 where the argmaxes differ, else 0.
 *   d_za, d_zb  device fp32, row i at d_za + i * stride_a (elements), V entries;
 *               OVERWRITTEN with the processed distributions when T > 0;
 *               the two inputs must not overlap.
 *   d_tv        device fp32 [n].
 * Asynchronous on `stream`.  Errors: LT_ERR_ARG (null pointer with n > 0,
 * V <= 0, T < 0, top_p <= 0, a stride below V), LT_ERR_CUDA (launch).
 */
int lt_readout_tv(float* d_za, long long stride_a, float* d_zb, long long stride_b, int n, int V,
                  float T, float top_p, float* d_tv, void* stream);

/*
 * Calibration of the copy screen on a committed text (CopyLoop card,
 * kongchang.com: copied continuations are scored at a shallow loop depth, and
 * a light calibration sets the threshold that admits them to the full-depth
 * verification; the copy_* fields of lt_decode_config use the same lookup and
 * score).  For each position t of d_tokens[0..n-1]:
 *   d_tok[t]    the first token the decoder's copy lookup proposes after the
 *               prefix d_tokens[0..t], all of it committed: the end e of the
 *               earlier occurrence (k-1 <= e <= t-1) whose backward match with
 *               the prefix's end is longest (>= k, capped at match_cap; the
 *               most recent on ties) gives d_tokens[e+1]; -1 when none;
 *   d_score[t]  its screen score, softmax of d_z1 row t at T = 1, taken at
 *               that token (-1 when none);
 *   d_accept[t] the probability that full depth accepts it as a one-hot
 *               draft: T = 0, 1 if it is the argmax of d_zR row t (lowest index
 *               on ties), else 0; T > 0, its probability after the readout
 *               processing of d_zR row t (temperature T, top-p, normalisation);
 *               0 when none.
 *   d_z1, d_zR  device fp32 logits, row t at base + t * stride (elements, >= V):
 *               the depth-d1 and full-depth readouts of position t (e.g. the
 *               d_logits of lt_prefill); d_zR is OVERWRITTEN with the processed
 *               distribution when T > 0.
 *   d_tokens, d_tok (device int32 [n]), d_score, d_accept (device fp32 [n]).
 * Asynchronous on `stream`; allocates nothing.  Errors: LT_ERR_ARG (null
 * pointer with n > 0, V <= 0, k < 1, match_cap < k, T < 0, top_p outside
 * (0, 1], a stride below V), LT_ERR_CUDA (launch).
 */
int lt_copy_screen_scores(const int32_t* d_tokens, int n, int k, int match_cap,
                          const float* d_z1, long long stride1, float* d_zR, long long strideR,
                          int V, float T, float top_p, int32_t* d_tok, float* d_score,
                          float* d_accept, void* stream);

/*
 * Self-test of the bounded waits (a test hook; the pages have no counterpart).
 * Every pipeline wait in the library gives up after ~1 s, records
 * DEV_TIMEOUT (1) and lets its kernel return, so a lost arrival ends in an
 * error status instead of a hung GPU.  This call launches one warp that
 * waits, through the same wait routine, on an mbarrier phase nothing
 * completes, then a trivial kernel.  h_out (host, 3 ints): [0] the status
 * the waiting kernel reported (1 = gave up), [1] 1 if the following kernel
 * ran (the context stayed usable), [2] the wait's duration in ms.
 * Synchronises `stream`.  Errors: LT_ERR_ARG (null h_out), LT_ERR_CUDA.
 */
int lt_selftest_wait(int32_t* h_out, void* stream);

/*
 * Stand-alone weight-streaming GEMM of the shared block (tcgen05 + TMEM + TMA):
 *   d_y[i][n] = sum_k d_x[i][k] * d_w[n][k],  i < ncols, n < n_out.
 * This is the contraction every shared-block layer runs once per decode step
 * over all active rows (LoopSpec page, sections 1 and 2.2: all branches advance
 * the shared block together in one batch).
 *   dtype   LT_BF16 (bf16 operands, fp32 accumulate) or LT_F32 (tf32 operands).
 *   d_w     [n_out][k] row-major (nn.Linear layout), 16-byte aligned, k*elem % 16 == 0.
 *   d_x     [ncols][k] row-major, same alignment; ncols in {8, 16, 32, 64}.
 *   d_y     [ncols][n_out] fp32.
 *   d_scratch  >= lt_gemm_scratch_bytes() bytes of device memory (an error
 *              word, reduction tables and fp32 partials); its contents are
 *              overwritten.
 * The call synchronises `stream` before returning.  The result for row i does
 * not depend on the other rows' values (the MMA always spans ncols columns).
 * Errors: LT_ERR_ARG / LT_ERR_SHAPE (arguments), LT_ERR_CAPACITY (scratch too
 * small), LT_ERR_CUDA (a runtime call failed), LT_ERR_DEVICE_CHECK (a bounded
 * wait inside the kernel gave up after ~1 s; d_y is then not a valid result).
 */
int lt_gemm_scratch_bytes(int dtype, int n_out, int k, int ncols, size_t* bytes);
int lt_gemm_rows(int dtype, const void* d_w, const void* d_x, float* d_y, int n_out, int k,
                 int ncols, void* d_scratch, size_t scratch_bytes, void* stream);

/*
 * Allocation-free variant of lt_gemm_rows, for callers that cannot allocate
 * device memory (a graph or memory pool owns every allocation, a plug-in gets
 * a stream but no allocator, or another framework has reserved the device).
 * The paper has no counterpart: this is a deployment convenience.
 *   - bf16 only (dtype must be LT_BF16; LT_F32 returns LT_ERR_ARG);
 *   - its scratch (reduction tables + fp32 partials) is one static device
 *     array of LT_NOALLOC_SCRATCH_BYTES inside the library, present on every
 *     device that loads the library until the process exits; sizes whose
 *     scratch would exceed it return LT_ERR_CAPACITY (e.g. n_out 49152 with
 *     ncols 64);
 *   - the first call on a device resolves the device addresses of the array
 *     and of a static error word (cudaGetSymbolAddress), so that first call
 *     must come before any stream capture; the addresses are kept for the
 *     life of the process and assume the device's primary context is not
 *     reset (cudaDeviceReset) in between;
 *   - every call shares the array and the error word: calls that overlap on
 *     the GPU (other streams, other threads) race; serialise them.  Each call
 *     clears the error word before its launch; a completed GEMM writes every
 *     partial its reduction reads, so nothing else needs clearing;
 *   - it calls no cudaMalloc / cudaFree and no allocating library routine;
 *   - every call copies its small reduction tables from the host and reads
 *     the error word back, synchronising `stream` before it returns.
 * Arguments, result and errors as lt_gemm_rows (LT_ERR_DEVICE_CHECK when a
 * bounded wait of the kernel gave up).
 */
#define LT_NOALLOC_SCRATCH_BYTES (8u << 20)
int lt_gemm_rows_noalloc(int dtype, const void* d_w, const void* d_x, float* d_y, int n_out,
                         int k, int ncols, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LOOPED_SPEC_H */
