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
  gemm_plan(n_out, k, dtype == LT_F32, sm_count(), &s, nullptr, nullptr);
  *bytes = align256((size_t)(2 * s.tiles + s.grid) * sizeof(int)) + gemm_part_bytes(s, ncols);
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
  gemm_plan(n_out, k, f32, sm_count(), &s, nullptr, nullptr);
  std::vector<int> tab(2 * s.tiles + s.grid);
  gemm_plan(n_out, k, f32, sm_count(), &s, tab.data(), tab.data() + 2 * s.tiles);
  int* d_tab = (int*)d_scratch;
  float* part = (float*)((char*)d_scratch + align256(tab.size() * sizeof(int)));
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemcpyAsync(d_tab, tab.data(), tab.size() * sizeof(int), cudaMemcpyHostToDevice, st) !=
      cudaSuccess)
    return LT_ERR_CUDA;
  s.tile_c = d_tab;
  s.cta_t0 = d_tab + 2 * s.tiles;
  CUtensorMap tw, tx;
  if (make_tmap(&tw, d_w, f32, n_out, k, GEMM_BM) != 0) return LT_ERR_SHAPE;
  if (make_tmap(&tx, d_x, f32, ncols, k, ncols) != 0) return LT_ERR_SHAPE;
  if (gemm_launch(tw, tx, part, s, ncols, f32, nullptr, nullptr, st, false) != cudaSuccess)
    return LT_ERR_CUDA;
  dim3 grid((n_out + 255) / 256, ncols);
  k_reduce_rows<<<grid, 256, 0, st>>>(part, s, ncols, d_y);
  if (cudaGetLastError() != cudaSuccess) return LT_ERR_CUDA;
  // the host copy of the tables must outlive the async copy
  if (cudaStreamSynchronize(st) != cudaSuccess) return LT_ERR_CUDA;
  return LT_OK;
}
