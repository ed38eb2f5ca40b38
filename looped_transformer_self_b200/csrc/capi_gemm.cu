// C-ABI entry points for the stand-alone weight-streaming GEMM.
#include <string.h>

#include <vector>

#include "../../include/looped_spec.h"
#include "gemm.cuh"

namespace lt {

__global__ void k_reduce_rows(const float* __restrict__ part, GemmShape s, int ncols,
                              float* __restrict__ y) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int i = blockIdx.y;
  if (n < s.n_out) y[(size_t)i * s.n_out + n] = sk_reduce(part, s, ncols, i, n);
}

static int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace lt

using namespace lt;

extern "C" int lt_gemm_scratch_bytes(int dtype, int n_out, int k, int ncols, size_t* bytes) {
  if (!bytes || n_out <= 0 || k <= 0) return LT_ERR_ARG;
  GemmShape s;
  gemm_plan(n_out, k, dtype == LT_F32, ncols, sm_count(), &s, nullptr, nullptr);
  *bytes = 256 /* error word */ + align256((size_t)gemm_table_ints(n_out, k, dtype == LT_F32, ncols, sm_count()) *
                    sizeof(int)) +
           align256(gemm_part_bytes(s, ncols));
  if (dtype == LT_F32) *bytes += 2 * align256((size_t)n_out * k * 4) + 2 * align256((size_t)ncols * k * 4);
  return LT_OK;
}

extern "C" int lt_gemm_rows(int dtype, const void* d_w, const void* d_x, float* d_y, int n_out,
                            int k, int ncols, void* d_scratch, size_t scratch_bytes,
                            void* stream) {
  if (!d_w || !d_x || !d_y || !d_scratch || n_out <= 0 || k <= 0) return LT_ERR_ARG;
  if (ncols != 8 && ncols != 16 && ncols != 32 && ncols != 64) return LT_ERR_SHAPE;
  if (dtype != LT_F32 && dtype != LT_BF16) return LT_ERR_ARG;
  const bool f32 = dtype == LT_F32;
  size_t need = 0;
  lt_gemm_scratch_bytes(dtype, n_out, k, ncols, &need);
  if (scratch_bytes < need) return LT_ERR_CAPACITY;
  GemmShape s;
  gemm_plan(n_out, k, f32, ncols, sm_count(), &s, nullptr, nullptr);
  std::vector<int> tab(gemm_table_ints(n_out, k, f32, ncols, sm_count()));
  gemm_plan(n_out, k, f32, ncols, sm_count(), &s, tab.data(), tab.data() + 2 * s.tiles);
  char* cur = (char*)d_scratch;
  int* d_err = (int*)cur;  // DEV_TIMEOUT when a bounded wait of the GEMM gave up
  cur += 256;
  int* d_tab = (int*)cur;
  cur += align256(tab.size() * sizeof(int));
  float* part = (float*)cur;
  cur += align256(gemm_part_bytes(s, ncols));
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemsetAsync(d_err, 0, sizeof(int), st) != cudaSuccess ||
      cudaMemcpyAsync(d_tab, tab.data(), tab.size() * sizeof(int), cudaMemcpyHostToDevice, st) !=
          cudaSuccess)
    return LT_ERR_CUDA;
  s.tile_c = d_tab;
  s.cta_t0 = d_tab + 2 * s.tiles;
  s.tinfo = reinterpret_cast<const int4*>(d_tab + gemm_tinfo_offset(s));
  GemmOperand tw, tx, twl, txl;
  const void* w_hi = d_w;
  const void* x_hi = d_x;
  if (f32) {  // fp32 operands run as split tf32 (hi + lo pairs)
    float* wh = (float*)cur;
    cur += align256((size_t)n_out * k * 4);
    float* wl = (float*)cur;
    cur += align256((size_t)n_out * k * 4);
    float* xh = (float*)cur;
    cur += align256((size_t)ncols * k * 4);
    float* xl = (float*)cur;
    if (split_tf32((const float*)d_w, wh, wl, (size_t)n_out * k, st) != cudaSuccess ||
        split_tf32((const float*)d_x, xh, xl, (size_t)ncols * k, st) != cudaSuccess)
      return LT_ERR_CUDA;
    w_hi = wh;
    x_hi = xh;
    if (make_operand(&twl, wl, true, n_out, k, GEMM_BM, s.kc) != 0) return LT_ERR_SHAPE;
    if (make_operand(&txl, xl, true, ncols, k, ncols, s.kc) != 0) return LT_ERR_SHAPE;
  }
  if (make_operand(&tw, w_hi, f32, n_out, k, GEMM_BM, s.kc) != 0) return LT_ERR_SHAPE;
  if (make_operand(&tx, x_hi, f32, ncols, k, ncols, s.kc) != 0) return LT_ERR_SHAPE;
  if (!f32) {
    twl = tw;
    txl = tx;
  }
  if (gemm_launch(tw, twl, tx, txl, part, s, ncols, f32 ? 2 : 0, nullptr, d_err, st, false) !=
      cudaSuccess)
    return LT_ERR_CUDA;
  dim3 grid((n_out + 255) / 256, ncols);
  k_reduce_rows<<<grid, 256, 0, st>>>(part, s, ncols, d_y);
  if (cudaGetLastError() != cudaSuccess) return LT_ERR_CUDA;
  // the host copy of the tables must outlive the async copy
  int h_err = 0;
  if (cudaMemcpyAsync(&h_err, d_err, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return LT_ERR_CUDA;
  // a bounded wait gave up: d_y holds no valid result
  return h_err ? LT_ERR_DEVICE_CHECK : LT_OK;
}
