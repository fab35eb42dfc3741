// Allocation-free variant of the block-mask entry point.
//
// Some callers cannot hand this library a scratch buffer: a plugin running
// inside a host framework that owns every byte of device memory and passes the
// plugin only its input and output tensors, or a latency-critical caller that
// must not risk an allocation stalling or failing in the middle of a run.
// This entry point serves them.  Its scratch space lives in one fixed-size
// array compiled into the library: every GPU that loads libtra.so holds that
// array (kMaskStaticScratchBytes) until the process exits, and nothing is ever
// allocated or freed at call time.
//
// Because every call shares that one array, and a call leaves its contents in
// place, two calls whose kernels overlap on the GPU (different streams, or
// different host threads, on the same device) race and may corrupt each
// other's masks.  Calls that follow one another on a single stream are safe.
// Every word of scratch the mask kernels read is written earlier in the same
// call, so nothing has to be cleared between calls.
#include <cuda_runtime.h>

#include <climits>
#include <cstdint>
#include <mutex>


#include "tra_internal.h"

namespace tra {
namespace {

constexpr size_t kMaskStaticScratchBytes = static_cast<size_t>(TRA_MASK_STATIC_SCRATCH_BYTES);

// The scratch array.  In host code this name is only a stand-in for the
// device object: host code must use the address from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_mask_scratch[kMaskStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_mask_scratch on the current device, looked up once per
// device (with that device current) and cached; nullptr on failure.
void* scratch_address() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_mask_scratch);
    if (e != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return nullptr;
    }
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace tra

extern "C" tra_status tra_build_block_mask_noalloc(const float* r, const float* phi, int heads,
                                                   tra_grid grid, tra_tile tile, int block_q,
                                                   int block_k, int vote_threshold, int* row_ptr,
                                                   int* col_idx, long long col_capacity,
                                                   int* nnz, tra_stream_t stream) {
  using namespace tra;
  NvtxRange nvtx_range("tra_build_block_mask_noalloc");
  if (heads < 0 || !grid_ok(grid) || !tile_ok(tile)) return TRA_ERR_INVALID_ARGUMENT;
  if (!block_ok(block_q) || !block_ok(block_k)) return TRA_ERR_UNSUPPORTED;
  if (vote_threshold < 1) return TRA_ERR_INVALID_ARGUMENT;
  if (grid.F > kMaxMaskFrames) return TRA_ERR_UNSUPPORTED;
  if (col_capacity < 0) return TRA_ERR_CAPACITY;
  if (nnz == nullptr) return TRA_ERR_INVALID_ARGUMENT;
  const long long N = static_cast<long long>(grid.F) * grid.H * grid.W;
  const long long nqb = (N + block_q - 1) / block_q, nkb = (N + block_k - 1) / block_k;
  if (heads > 65535 || static_cast<long long>(heads) * nqb * nkb >= INT_MAX)
    return TRA_ERR_UNSUPPORTED;
  const TileLayout L = layout_of(grid, tile);
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (heads == 0 || N == 0) {
    // The empty problem follows tra_build_block_mask_ex exactly: only row_ptr
    // and nnz are written, so only they are checked.
    if (heads > 0 && row_ptr == nullptr) return TRA_ERR_INVALID_ARGUMENT;
    const tra_status dv = check_device({row_ptr, nnz});
    if (dv != TRA_OK) return dv;
    cudaError_t e = cudaSuccess;
    if (heads > 0) e = cudaMemsetAsync(row_ptr, 0, sizeof(int) * heads, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(nnz, 0, sizeof(int), st);
    return status_of(e);
  }
  if (r == nullptr || phi == nullptr || row_ptr == nullptr) return TRA_ERR_INVALID_ARGUMENT;
  if (col_idx == nullptr && col_capacity > 0) return TRA_ERR_INVALID_ARGUMENT;
  // Problems whose scratch would not fit the built-in array are refused.
  if (mask_workspace_bytes(heads, L, block_q, block_k) > kMaskStaticScratchBytes)
    return TRA_ERR_WORKSPACE;
  const tra_status dv = check_device({r, phi, row_ptr, col_idx, nnz});
  if (dv != TRA_OK) return dv;
  void* scratch = scratch_address();
  if (scratch == nullptr) return TRA_ERR_CUDA;
  return status_of(launch_block_mask(r, phi, heads, L, block_q, block_k, vote_threshold, false,
                                     row_ptr, col_idx, col_capacity, nnz, scratch, st));
}
