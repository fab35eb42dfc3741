// Host-side interface between the C ABI (api.cu) and the kernel files.
#pragma once
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>
#include <initializer_list>

#include "tra.h"
#include "layout.cuh"

namespace tra {

constexpr int kMaxFrames = 1024;   // phi / frame tables live in kernel parameters
constexpr int kMaxMaskFrames = 384;  // the mask keeps a 128-query x F threshold table in smem
constexpr int kMaxSide = 16384;    // H, W bound: squared distances stay below 2^30

// Device error word of the current device (a module-scope __device__ int).
int* device_error_word();

// Status of a CUDA runtime result: TRA_OK or TRA_ERR_CUDA (defined in api.cu).
tra_status status_of(cudaError_t e);

// Argument checks shared by the entry points (defined in api.cu).
bool grid_ok(const tra_grid& g);  // sides >= 0, within kMaxFrames / kMaxSide, N <= 2^24
bool tile_ok(const tra_tile& t);  // every tile side >= 1
bool block_ok(int b);             // block sizes 16, 64, 128
TileLayout layout_of(const tra_grid& g, const tra_tile& t);
// TRA_OK when the current device has compute capability 10.x and every
// non-null pointer of `ptrs` is device memory of that device (or managed
// memory); TRA_ERR_DEVICE or TRA_ERR_INVALID_ARGUMENT otherwise.  Host
// pointers are refused here, before any launch, instead of faulting a kernel.
tra_status check_device(std::initializer_list<const void*> ptrs = {});
// NVTX range named after an API call, visible to Nsight tools (no-op without one).
struct NvtxRange {
  explicit NvtxRange(const char* name);
  ~NvtxRange();
};

// permute.cu
cudaError_t launch_permute(const void* src, void* dst, tra_dtype in_dtype, tra_dtype out_dtype,
                           int heads, int d, const TileLayout& L, bool inverse,
                           cudaStream_t stream);

// radius.cu
struct FrameTables {
  float coef[kMaxFrames];  // per query frame t: sqrt(tau / (pi S(t))) (disk), tau / (2 L(t)) (1D)
  float phi[kMaxFrames];   // decay table phi(delta)
};
struct FrameTablesD {
  double c[kMaxFrames];   // per query frame t: 1 / (pi S(t)) (disk) or 1 / (2 L(t)) (1D)
  float phi[kMaxFrames];  // decay table phi(delta)
};
// r = coef[t] * expf(e * H), e = 1/2 (disk) or 1 (1D distance)
cudaError_t launch_budget_radius(const float* H, float* r, float* phi_out, int heads,
                                 const TileLayout& L, const FrameTables& tables, bool line,
                                 cudaStream_t stream);
// shared per-head budget K_h = tau * mean(exp(H)); r = sqrt(K_h c[t]) or K_h c[t]
cudaError_t launch_shared_budget_radius(const float* H, float* r, float* phi_out, int heads,
                                        const TileLayout& L, double tau, bool line,
                                        const FrameTablesD& tables, cudaStream_t stream);
// r = r0 everywhere; phi_out <- tables.phi
cudaError_t launch_fill_radius(float* r, float* phi_out, int heads, const TileLayout& L, float r0,
                               const FrameTables& tables, cudaStream_t stream);

// mask.cu
size_t mask_workspace_bytes(int heads, const TileLayout& L, int block_q, int block_k);
cudaError_t launch_block_mask(const float* r, const float* phi, int heads, const TileLayout& L,
                              int block_q, int block_k, int vote, bool line, int* row_ptr,
                              int* col_idx, long long capacity, int* nnz, void* workspace,
                              cudaStream_t stream);

// attention.cu
struct AttnArgs {
  const void* Q;
  const void* K;
  const void* V;
  void* O;
  float* H;    // entropy (dense only), may be null
  float* lse;  // may be null
  const int* row_ptr;  // sparse only
  const int* col_idx;  // sparse only
  int heads, N, d;
  int block_q, block_k;  // sparse only; dense uses 128-key tiles
  float scale;
  bool dense;
  bool entropy_only;  // H (and LSE) over all keys, no output (V and O unused)
  bool fp8;           // Q and K are E4M3 codes with per-block scales
  const float* q_scales;  // [heads, ceil(N / 128)] (fp8 only)
  const float* k_scales;  // [heads, ceil(N / 128)] (fp8 only)
};
// selftest.cu: one wait on a barrier nothing completes, given up after limit_ns
cudaError_t launch_selftest_wait(unsigned long long limit_ns, int* completed, cudaStream_t stream);
// quant.cu: per (head, block of `block` rows) E4M3 quantization of bf16 X
cudaError_t launch_quantize_e4m3(const void* X, void* Xq, float* scales, int heads, int N, int d,
                                 int block, cudaStream_t stream);
cudaError_t launch_attention(const AttnArgs& a, cudaStream_t stream);

}  // namespace tra
