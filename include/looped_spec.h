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
 *   d_scratch  >= lt_gemm_scratch_bytes() bytes of device memory (reduction
 *              tables and fp32 partials); its contents are overwritten.
 * The call synchronises `stream` before returning.  The result for row i does
 * not depend on the other rows' values (the MMA always spans ncols columns).
 */
int lt_gemm_scratch_bytes(int dtype, int n_out, int k, int ncols, size_t* bytes);
int lt_gemm_rows(int dtype, const void* d_w, const void* d_x, float* d_y, int n_out, int k,
                 int ncols, void* d_scratch, size_t scratch_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LOOPED_SPEC_H */
