// Allocation-free variant of the stand-alone weight-streaming GEMM.
//
// Some callers cannot call cudaMalloc: code that runs while a memory pool or
// a CUDA graph owns every allocation, plug-ins that are handed a stream but no
// allocator, or processes whose device memory is fully reserved by another
// framework.  lt_gemm_rows_noalloc serves them: instead of a caller-provided
// scratch buffer it uses one fixed array in device global memory that is part
// of the library image (LT_NOALLOC_SCRATCH_BYTES, loaded with the library on
// every device that uses it and held until the process exits).
#include <mutex>
#include <vector>

#include "../../include/looped_spec.h"
#include "gemm.cuh"

namespace lt {

__global__ void k_reduce_rows_na(const float* __restrict__ part, GemmShape s, int ncols,
                                 float* __restrict__ y) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int i = blockIdx.y;
  if (n < s.n_out) y[(size_t)i * s.n_out + n] = sk_reduce(part, s, ncols, i, n);
}

}  // namespace lt

// Scratch of the allocation-free GEMM: reduction tables, then fp32 partials.
// Host code may not use this name as a device address (it is a host-side
// stand-in); the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LT_NOALLOC_SCRATCH_BYTES];
// Error word of the allocation-free GEMM: a bounded wait inside the kernel
// that gives up writes DEV_TIMEOUT here.  Cleared before every launch and read
// back after the call's stream synchronisation (same host-side stand-in rule).
static __device__ __align__(16) int g_noalloc_err;

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
// Device addresses of the two arrays, resolved once per device.  They assume
// the device's primary context lives as long as the process (a
// cudaDeviceReset in between would leave them stale).
void* g_scratch_ptr[kMaxDevices] = {};
int* g_err_ptr[kMaxDevices] = {};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

int sm_count_dev(int dev) {
  int n = 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}
}  // namespace

using namespace lt;

extern "C" int lt_gemm_rows_noalloc(int dtype, const void* d_w, const void* d_x, float* d_y,
                                    int n_out, int k, int ncols, void* stream) {
  if (!d_w || !d_x || !d_y || n_out <= 0 || k <= 0) return LT_ERR_ARG;
  if (dtype != LT_BF16) return LT_ERR_ARG;  // fp32 would need hi/lo copies of the whole matrix
  if (ncols != 8 && ncols != 16 && ncols != 32 && ncols != 64) return LT_ERR_SHAPE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LT_ERR_CUDA;
  void* base = nullptr;
  int* d_err = nullptr;
  {
    // Once per device, with that device current: resolve the arrays' device
    // addresses.  Done by the first call on the device (before any stream capture).
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
      void* p = nullptr;
      void* q = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return LT_ERR_CUDA;
      if (cudaGetSymbolAddress(&q, g_noalloc_err) != cudaSuccess || !q) return LT_ERR_CUDA;
      g_scratch_ptr[dev] = p;
      g_err_ptr[dev] = (int*)q;
    }
    base = g_scratch_ptr[dev];
    d_err = g_err_ptr[dev];
  }
  GemmShape s;
  const int grid_cap = sm_count_dev(dev);
  gemm_plan(n_out, k, false, ncols, grid_cap, &s, nullptr, nullptr);
  std::vector<int> tab(gemm_table_ints(n_out, k, false, ncols, grid_cap));
  gemm_plan(n_out, k, false, ncols, grid_cap, &s, tab.data(), tab.data() + 2 * s.tiles);
  const size_t tab_bytes = align256(tab.size() * sizeof(int));
  const size_t need = tab_bytes + gemm_part_bytes(s, ncols);
  if (need > (size_t)LT_NOALLOC_SCRATCH_BYTES) return LT_ERR_CAPACITY;
  int* d_tab = (int*)base;
  float* part = (float*)((char*)base + tab_bytes);
  cudaStream_t st = (cudaStream_t)stream;
  // A completed GEMM writes every partial the reducer reads, so only the error
  // word needs clearing: a GEMM whose wait gave up leaves earlier calls'
  // partials in the array, and the word is what tells the caller.
  if (cudaMemsetAsync(d_err, 0, sizeof(int), st) != cudaSuccess ||
      cudaMemcpyAsync(d_tab, tab.data(), tab.size() * sizeof(int), cudaMemcpyHostToDevice, st) !=
          cudaSuccess)
    return LT_ERR_CUDA;
  s.tile_c = d_tab;
  s.cta_t0 = d_tab + 2 * s.tiles;
  s.tinfo = reinterpret_cast<const int4*>(d_tab + gemm_tinfo_offset(s));
  GemmOperand tw, tx;
  if (make_operand(&tw, d_w, false, n_out, k, GEMM_BM, s.kc) != 0) return LT_ERR_SHAPE;
  if (make_operand(&tx, d_x, false, ncols, k, ncols, s.kc) != 0) return LT_ERR_SHAPE;
  if (gemm_launch(tw, tw, tx, tx, part, s, ncols, 0, nullptr, d_err, st, false) != cudaSuccess)
    return LT_ERR_CUDA;
  dim3 grid((n_out + 255) / 256, ncols);
  k_reduce_rows_na<<<grid, 256, 0, st>>>(part, s, ncols, d_y);
  if (cudaGetLastError() != cudaSuccess) return LT_ERR_CUDA;
  // the host copy of the tables must outlive the asynchronous copy
  int h_err = 0;
  if (cudaMemcpyAsync(&h_err, d_err, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return LT_ERR_CUDA;
  // a bounded wait gave up: d_y holds no valid result
  return h_err ? LT_ERR_DEVICE_CHECK : LT_OK;
}
