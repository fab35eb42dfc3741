// C ABI of the Token Radius Attention hot path: argument checks, the host
// side of the budget -> radius tables, and dispatch to the kernels.  Every
// entry point validates first and launches nothing when it returns an error.
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "ptx.cuh"
#include "tra_internal.h"

namespace tra {

NvtxRange::NvtxRange(const char* name) { nvtxRangePushA(name); }
NvtxRange::~NvtxRange() { nvtxRangePop(); }

// Device error word: first code recorded by a kernel whose wait ran out of time.
__device__ int g_device_error = 0;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int* g_err_ptr[kMaxDevices] = {};
int g_cc_ok[kMaxDevices] = {};  // 0 unknown, 1 sm_100, -1 other

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

tra_status status_of(cudaError_t e) {
  if (e == cudaSuccess) return TRA_OK;
  return TRA_ERR_CUDA;
}

tra_status check_device(std::initializer_list<const void*> ptrs) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return TRA_ERR_DEVICE;
  }
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_cc_ok[dev] == 0) {
      int major = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
        cudaGetLastError();
        return TRA_ERR_DEVICE;
      }
      g_cc_ok[dev] = (major == 10) ? 1 : -1;
    }
    if (g_cc_ok[dev] != 1) return TRA_ERR_DEVICE;
  }
  for (const void* p : ptrs) {
    if (p == nullptr) continue;
    cudaPointerAttributes at{};
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
      cudaGetLastError();
      return TRA_ERR_INVALID_ARGUMENT;
    }
    if (at.type == cudaMemoryTypeManaged) continue;
    if (at.type != cudaMemoryTypeDevice || at.device != dev) return TRA_ERR_INVALID_ARGUMENT;
  }
  return TRA_OK;
}

bool grid_ok(const tra_grid& g) {
  return g.F >= 0 && g.H >= 0 && g.W >= 0 && g.F <= kMaxFrames && g.H <= kMaxSide &&
         g.W <= kMaxSide && static_cast<long long>(g.F) * g.H * g.W <= (1LL << 24);
}

bool tile_ok(const tra_tile& t) { return t.t >= 1 && t.y >= 1 && t.x >= 1; }

bool block_ok(int b) { return b == 16 || b == 64 || b == 128; }

TileLayout layout_of(const tra_grid& g, const tra_tile& t) {
  return TileLayout{g.F, g.H, g.W, t.t, t.y, t.x};
}

int* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_err_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_device_error) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_err_ptr[dev] = static_cast<int*>(ptr);
  }
  return g_err_ptr[dev];
}

}  // namespace tra

using namespace tra;

extern "C" {

const char* tra_status_string(tra_status s) {
  switch (s) {
    case TRA_OK: return "ok";
    case TRA_ERR_INVALID_ARGUMENT: return "invalid argument (null, misaligned or host pointer, or bad size)";
    case TRA_ERR_UNSUPPORTED: return "unsupported shape (d, block size or list length)";
    case TRA_ERR_WORKSPACE: return "workspace too small or not 256-byte aligned";
    case TRA_ERR_CAPACITY: return "negative col_idx capacity";
    case TRA_ERR_CUDA: return "CUDA runtime error";
    case TRA_ERR_DEVICE: return "no usable compute capability 10.0 (sm_100a) device";
    case TRA_ERR_TIMEOUT: return "a device-side wait ran out of time";
    case TRA_ERR_BAD_INPUT: return "a kernel met an invalid CSR row (skipped)";
  }
  return "unknown status";
}

int tra_version(void) { return 100; }

tra_status tra_tile_major_permute(const void* X, void* X_tm, tra_dtype in_dtype,
                                  tra_dtype out_dtype, int heads, int d, tra_grid grid,
                                  tra_tile tile, tra_stream_t stream) {
  NvtxRange nvtx_range("tra_tile_major_permute");
  if (heads < 0 || !grid_ok(grid) || !tile_ok(tile)) return TRA_ERR_INVALID_ARGUMENT;
  if ((in_dtype != TRA_BF16 && in_dtype != TRA_F32) || (out_dtype != TRA_BF16 && out_dtype != TRA_F32))
    return TRA_ERR_INVALID_ARGUMENT;
  if (d < 8 || d > 1024 || d % 8 != 0) return TRA_ERR_UNSUPPORTED;
  const long long N = static_cast<long long>(grid.F) * grid.H * grid.W;
  if (heads == 0 || N == 0) return TRA_OK;
  if (heads > 65535) return TRA_ERR_UNSUPPORTED;
  if (X == nullptr || X_tm == nullptr || !aligned16(X) || !aligned16(X_tm))
    return TRA_ERR_INVALID_ARGUMENT;
  if (X == X_tm) return TRA_ERR_INVALID_ARGUMENT;
  const tra_status dv = check_device({X, X_tm});
  if (dv != TRA_OK) return dv;
  return status_of(launch_permute(X, X_tm, in_dtype, out_dtype, heads, d, layout_of(grid, tile),
                                  false, reinterpret_cast<cudaStream_t>(stream)));
}

tra_status tra_inverse_permute(const void* X_tm, void* X, tra_dtype dtype, int heads, int d,
                               tra_grid grid, tra_tile tile, tra_stream_t stream) {
  NvtxRange nvtx_range("tra_inverse_permute");
  if (heads < 0 || !grid_ok(grid) || !tile_ok(tile)) return TRA_ERR_INVALID_ARGUMENT;
  if (dtype != TRA_BF16 && dtype != TRA_F32) return TRA_ERR_INVALID_ARGUMENT;
  if (d < 8 || d > 1024 || d % 8 != 0) return TRA_ERR_UNSUPPORTED;
  const long long N = static_cast<long long>(grid.F) * grid.H * grid.W;
  if (heads == 0 || N == 0) return TRA_OK;
  if (heads > 65535) return TRA_ERR_UNSUPPORTED;
  if (X == nullptr || X_tm == nullptr || !aligned16(X) || !aligned16(X_tm))
    return TRA_ERR_INVALID_ARGUMENT;
  if (X == X_tm) return TRA_ERR_INVALID_ARGUMENT;
  const tra_status dv = check_device({X, X_tm});
  if (dv != TRA_OK) return dv;
  return status_of(launch_permute(X_tm, X, dtype, dtype, heads, d, layout_of(grid, tile), true,
                                  reinterpret_cast<cudaStream_t>(stream)));
}

static tra_status check_attn_common(const void* Q, const void* K, const void* V, void* O,
                                    int heads, int N, int d, float scale) {
  if (heads < 0 || N < 0) return TRA_ERR_INVALID_ARGUMENT;
  if (!(scale > 0.f) || !std::isfinite(scale)) return TRA_ERR_INVALID_ARGUMENT;
  if (d != 64 && d != 128) return TRA_ERR_UNSUPPORTED;
  if (heads == 0 || N == 0) return TRA_OK;
  if (heads > 65535 || N > (1 << 24)) return TRA_ERR_UNSUPPORTED;
  if (!Q || !K || !V || !O) return TRA_ERR_INVALID_ARGUMENT;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return TRA_ERR_INVALID_ARGUMENT;
  return TRA_OK;
}

tra_status tra_dense_attn_entropy(const void* Q, const void* K, const void* V, void* O, float* H,
                                  float* lse, int heads, int N, int d, float scale,
                                  tra_stream_t stream) {
  NvtxRange nvtx_range("tra_dense_attn_entropy");
  tra_status s = check_attn_common(Q, K, V, O, heads, N, d, scale);
  if (s != TRA_OK || heads == 0 || N == 0) return s;
  if (H == nullptr) return TRA_ERR_INVALID_ARGUMENT;
  s = check_device({Q, K, V, O, H, lse});
  if (s != TRA_OK) return s;
  AttnArgs a{};
  a.Q = Q; a.K = K; a.V = V; a.O = O; a.H = H; a.lse = lse;
  a.heads = heads; a.N = N; a.d = d; a.scale = scale; a.dense = true;
  a.block_q = 128; a.block_k = 128;
  return status_of(launch_attention(a, reinterpret_cast<cudaStream_t>(stream)));
}

tra_status tra_attn_entropy(const void* Q, const void* K, float* H, float* lse, int heads, int N,
                            int d, float scale, tra_stream_t stream) {
  NvtxRange nvtx_range("tra_attn_entropy");
  if (heads < 0 || N < 0) return TRA_ERR_INVALID_ARGUMENT;
  if (!(scale > 0.f) || !std::isfinite(scale)) return TRA_ERR_INVALID_ARGUMENT;
  if (d != 64 && d != 128) return TRA_ERR_UNSUPPORTED;
  if (heads == 0 || N == 0) return TRA_OK;
  if (heads > 65535 || N > (1 << 24)) return TRA_ERR_UNSUPPORTED;
  if (!Q || !K || !H || !aligned16(Q) || !aligned16(K)) return TRA_ERR_INVALID_ARGUMENT;
  const tra_status s = check_device({Q, K, H, lse});
  if (s != TRA_OK) return s;
  AttnArgs a{};
  a.Q = Q; a.K = K; a.V = nullptr; a.O = nullptr; a.H = H; a.lse = lse;
  a.heads = heads; a.N = N; a.d = d; a.scale = scale; a.dense = true; a.entropy_only = true;
  a.block_q = 128; a.block_k = 128;
  return status_of(launch_attention(a, reinterpret_cast<cudaStream_t>(stream)));
}

tra_status tra_block_sparse_attn(const void* Q, const void* K, const void* V, void* O, float* lse,
                                 const int* row_ptr, const int* col_idx, int heads, int N, int d,
                                 int block_q, int block_k, float scale, tra_stream_t stream) {
  NvtxRange nvtx_range("tra_block_sparse_attn");
  tra_status s = check_attn_common(Q, K, V, O, heads, N, d, scale);
  if (s != TRA_OK) return s;
  if (!block_ok(block_q) || !block_ok(block_k)) return TRA_ERR_UNSUPPORTED;
  if (heads == 0 || N == 0) return TRA_OK;
  if (row_ptr == nullptr || col_idx == nullptr) return TRA_ERR_INVALID_ARGUMENT;
  const long long nkb = (N + block_k - 1) / block_k;
  // 16-token blocks run on the kernel that merges up to eight query blocks'
  // lists in shared memory (at most 1024 key blocks)
  if (block_q < 128 && (block_q == 16 || block_k == 16) && nkb > 1024) return TRA_ERR_UNSUPPORTED;
  s = check_device({Q, K, V, O, lse, row_ptr, col_idx});
  if (s != TRA_OK) return s;
  AttnArgs a{};
  a.Q = Q; a.K = K; a.V = V; a.O = O; a.H = nullptr; a.lse = lse;
  a.row_ptr = row_ptr; a.col_idx = col_idx;
  a.heads = heads; a.N = N; a.d = d; a.scale = scale; a.dense = false;
  a.block_q = block_q; a.block_k = block_k;
  return status_of(launch_attention(a, reinterpret_cast<cudaStream_t>(stream)));
}

tra_status tra_quantize_e4m3(const void* X, void* Xq, float* scales, int heads, int N, int d,
                             int block, tra_stream_t stream) {
  NvtxRange nvtx_range("tra_quantize_e4m3");
  if (heads < 0 || N < 0) return TRA_ERR_INVALID_ARGUMENT;
  if ((d != 64 && d != 128) || (block != 64 && block != 128)) return TRA_ERR_UNSUPPORTED;
  if (heads == 0 || N == 0) return TRA_OK;
  if (heads > 65535 || N > (1 << 24)) return TRA_ERR_UNSUPPORTED;
  if (!X || !Xq || !scales || !aligned16(X) || !aligned16(Xq)) return TRA_ERR_INVALID_ARGUMENT;
  const tra_status dv = check_device({X, Xq, scales});
  if (dv != TRA_OK) return dv;
  return status_of(launch_quantize_e4m3(X, Xq, scales, heads, N, d, block,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

tra_status tra_block_sparse_attn_fp8(const void* Q8, const float* q_scales, const void* K8,
                                     const float* k_scales, const void* V, void* O, float* lse,
                                     const int* row_ptr, const int* col_idx, int heads, int N,
                                     int d, int block_q, int block_k, float scale,
                                     tra_stream_t stream) {
  NvtxRange nvtx_range("tra_block_sparse_attn_fp8");
  tra_status s = check_attn_common(Q8, K8, V, O, heads, N, d, scale);
  if (s != TRA_OK) return s;
  if (d != 128 || block_q != 128 || block_k != 128) return TRA_ERR_UNSUPPORTED;
  if (heads == 0 || N == 0) return TRA_OK;
  if (!row_ptr || !col_idx || !q_scales || !k_scales) return TRA_ERR_INVALID_ARGUMENT;
  s = check_device({Q8, q_scales, K8, k_scales, V, O, lse, row_ptr, col_idx});
  if (s != TRA_OK) return s;
  AttnArgs a{};
  a.Q = Q8; a.K = K8; a.V = V; a.O = O; a.H = nullptr; a.lse = lse;
  a.row_ptr = row_ptr; a.col_idx = col_idx;
  a.heads = heads; a.N = N; a.d = d; a.scale = scale; a.dense = false;
  a.block_q = 128; a.block_k = 128;
  a.fp8 = true; a.q_scales = q_scales; a.k_scales = k_scales;
  return status_of(launch_attention(a, reinterpret_cast<cudaStream_t>(stream)));
}

tra_status tra_budget_radius_ex(const float* H, float* r, float* phi_out, int heads,
                                tra_grid grid, tra_tile tile, float tau, float gamma,
                                tra_budget budget, tra_metric metric, tra_stream_t stream) {
  NvtxRange nvtx_range("tra_budget_radius_ex");
  if (heads < 0 || !grid_ok(grid) || !tile_ok(tile)) return TRA_ERR_INVALID_ARGUMENT;
  if (!(tau >= 0.f) || !std::isfinite(tau) || !(gamma >= 0.f) || !std::isfinite(gamma))
    return TRA_ERR_INVALID_ARGUMENT;
  if (budget != TRA_BUDGET_ENTROPY && budget != TRA_BUDGET_SHARED) return TRA_ERR_INVALID_ARGUMENT;
  if (metric != TRA_METRIC_DISK && metric != TRA_METRIC_LINE) return TRA_ERR_INVALID_ARGUMENT;
  const long long N = static_cast<long long>(grid.F) * grid.H * grid.W;
  if (N == 0) return TRA_OK;
  if (heads == 0 && phi_out == nullptr) return TRA_OK;
  if (heads > 0 && (H == nullptr || r == nullptr)) return TRA_ERR_INVALID_ARGUMENT;
  if (heads > 65535) return TRA_ERR_UNSUPPORTED;
  const tra_status dv = check_device({H, r, phi_out});
  if (dv != TRA_OK) return dv;
  const bool line = metric == TRA_METRIC_LINE;
  // phi(delta) = exp(-gamma delta); per query frame t the disk uses
  // S(t) = sum_t' phi(|t'-t|)^2 and the 1D distance L(t) = sum_t' phi(|t'-t|);
  // all in double, rounded once.
  const int F = grid.F;
  double phid[kMaxFrames];
  double per_frame[kMaxFrames];  // 1 / (pi S(t)) or 1 / (2 L(t))
  for (int k = 0; k < F; ++k) phid[k] = std::exp(-static_cast<double>(gamma) * k);
  for (int t = 0; t < F; ++t) {
    double acc = 0.0;
    for (int tp = 0; tp < F; ++tp) {
      const double f = phid[tp > t ? tp - t : t - tp];
      acc += line ? f : f * f;
    }
    per_frame[t] = line ? 1.0 / (2.0 * acc) : 1.0 / (M_PI * acc);
  }
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const TileLayout Lt = layout_of(grid, tile);
  if (budget == TRA_BUDGET_ENTROPY) {
    static thread_local FrameTables tab;
    for (int k = 0; k < F; ++k) tab.phi[k] = static_cast<float>(phid[k]);
    for (int t = 0; t < F; ++t) {
      const double c = static_cast<double>(tau) * per_frame[t];
      tab.coef[t] = static_cast<float>(line ? c : std::sqrt(c));
    }
    return status_of(launch_budget_radius(H, r, phi_out, heads, Lt, tab, line, st));
  }
  static thread_local FrameTablesD tabd;
  for (int k = 0; k < F; ++k) tabd.phi[k] = static_cast<float>(phid[k]);
  for (int t = 0; t < F; ++t) tabd.c[t] = per_frame[t];
  if (heads == 0) {
    // only the decay table is asked for
    static thread_local FrameTables tab;
    for (int k = 0; k < F; ++k) tab.phi[k] = tabd.phi[k];
    return status_of(launch_fill_radius(nullptr, phi_out, 0, Lt, 0.f, tab, st));
  }
  return status_of(launch_shared_budget_radius(H, r, phi_out, heads, Lt, static_cast<double>(tau),
                                               line, tabd, st));
}

tra_status tra_budget_radius(const float* H, float* r, float* phi_out, int heads, tra_grid grid,
                             tra_tile tile, float tau, float gamma, tra_stream_t stream) {
  return tra_budget_radius_ex(H, r, phi_out, heads, grid, tile, tau, gamma, TRA_BUDGET_ENTROPY,
                              TRA_METRIC_DISK, stream);
}

tra_status tra_radial_radius(float* r, float* phi_out, int heads, tra_grid grid, tra_tile tile,
                             float r0, tra_metric metric, tra_stream_t stream) {
  NvtxRange nvtx_range("tra_radial_radius");
  if (heads < 0 || !grid_ok(grid) || !tile_ok(tile)) return TRA_ERR_INVALID_ARGUMENT;
  if (!(r0 >= 0.f)) return TRA_ERR_INVALID_ARGUMENT;  // NaN and negative radii
  if (metric != TRA_METRIC_DISK && metric != TRA_METRIC_LINE) return TRA_ERR_INVALID_ARGUMENT;
  const long long N = static_cast<long long>(grid.F) * grid.H * grid.W;
  if (N == 0) return TRA_OK;
  if (heads == 0 && phi_out == nullptr) return TRA_OK;
  if (heads > 0 && r == nullptr) return TRA_ERR_INVALID_ARGUMENT;
  if (heads > 65535) return TRA_ERR_UNSUPPORTED;
  const tra_status dv = check_device({r, phi_out});
  if (dv != TRA_OK) return dv;
  // band b = floor(log2(delta + 1)); window factor 2^(-b/2) (disk: the area
  // halves per band) or 2^(-b) (1D: the length halves per band)
  static thread_local FrameTables tab;
  for (int k = 0; k < grid.F; ++k) {
    int b = 0;
    while ((static_cast<unsigned>(k) + 1u) >> (b + 1)) ++b;
    const double f = metric == TRA_METRIC_LINE ? std::ldexp(1.0, -b) : std::pow(2.0, -0.5 * b);
    tab.phi[k] = static_cast<float>(f);
    tab.coef[k] = 0.f;
  }
  return status_of(launch_fill_radius(heads > 0 ? r : nullptr, phi_out, heads,
                                      layout_of(grid, tile), r0, tab,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

size_t tra_mask_workspace_size(int heads, tra_grid grid, tra_tile tile, int block_q, int block_k) {
  if (heads < 0 || !grid_ok(grid) || !tile_ok(tile) || !block_ok(block_q) || !block_ok(block_k))
    return 0;
  return mask_workspace_bytes(heads, layout_of(grid, tile), block_q, block_k);
}

size_t tra_workspace_size(int heads, tra_grid grid, int block_q, int block_k) {
  return tra_mask_workspace_size(heads, grid, tra_tile{1, 4, 4}, block_q, block_k);
}

tra_status tra_build_block_mask_ex(const float* r, const float* phi, int heads, tra_grid grid,
                                   tra_tile tile, int block_q, int block_k, int vote_threshold,
                                   tra_metric metric, int* row_ptr, int* col_idx,
                                   long long col_capacity, int* nnz, void* workspace,
                                   size_t workspace_bytes, tra_stream_t stream) {
  NvtxRange nvtx_range("tra_build_block_mask_ex");
  if (heads < 0 || !grid_ok(grid) || !tile_ok(tile)) return TRA_ERR_INVALID_ARGUMENT;
  if (metric != TRA_METRIC_DISK && metric != TRA_METRIC_LINE) return TRA_ERR_INVALID_ARGUMENT;
  if (!block_ok(block_q) || !block_ok(block_k)) return TRA_ERR_UNSUPPORTED;
  if (vote_threshold < 1) return TRA_ERR_INVALID_ARGUMENT;
  if (grid.F > kMaxMaskFrames) return TRA_ERR_UNSUPPORTED;
  if (col_capacity < 0) return TRA_ERR_CAPACITY;
  if (nnz == nullptr) return TRA_ERR_INVALID_ARGUMENT;
  const long long N = static_cast<long long>(grid.F) * grid.H * grid.W;
  const long long nqb = (N + block_q - 1) / block_q, nkb = (N + block_k - 1) / block_k;
  if (heads > 65535 || static_cast<long long>(heads) * nqb * nkb >= INT_MAX) return TRA_ERR_UNSUPPORTED;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (heads == 0 || N == 0) {
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
  const size_t need = mask_workspace_bytes(heads, layout_of(grid, tile), block_q, block_k);
  if (workspace == nullptr || workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return TRA_ERR_WORKSPACE;
  const tra_status dv = check_device({r, phi, row_ptr, col_idx, nnz, workspace});
  if (dv != TRA_OK) return dv;
  return status_of(launch_block_mask(r, phi, heads, layout_of(grid, tile), block_q, block_k,
                                     vote_threshold, metric == TRA_METRIC_LINE, row_ptr,
                                     col_idx, col_capacity, nnz, workspace, st));
}

tra_status tra_build_block_mask(const float* r, const float* phi, int heads, tra_grid grid,
                                tra_tile tile, int block_q, int block_k, int vote_threshold,
                                int* row_ptr, int* col_idx, long long col_capacity, int* nnz,
                                void* workspace, size_t workspace_bytes, tra_stream_t stream) {
  return tra_build_block_mask_ex(r, phi, heads, grid, tile, block_q, block_k, vote_threshold,
                                 TRA_METRIC_DISK, row_ptr, col_idx, col_capacity, nnz, workspace,
                                 workspace_bytes, stream);
}

tra_status tra_selftest_wait_timeout(int limit_ms, int* completed, tra_stream_t stream) {
  if (limit_ms < 1 || limit_ms > 2000) return TRA_ERR_INVALID_ARGUMENT;
  if (completed != nullptr && !aligned16(completed)) return TRA_ERR_INVALID_ARGUMENT;
  const tra_status dv = check_device({completed});
  if (dv != TRA_OK) return dv;
  return status_of(launch_selftest_wait(static_cast<unsigned long long>(limit_ms) * 1000000ull,
                                        completed, reinterpret_cast<cudaStream_t>(stream)));
}

tra_status tra_get_device_error(int* code, tra_stream_t stream) {
  if (code == nullptr) return TRA_ERR_INVALID_ARGUMENT;
  *code = 0;
  const tra_status dv = check_device();
  if (dv != TRA_OK) return dv;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return TRA_ERR_CUDA;
  }
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return TRA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return TRA_ERR_CUDA;
  }
  *code = v;
  if (v == 0) return TRA_OK;
  return (v == kErrBadCsr || v == kErrIndex) ? TRA_ERR_BAD_INPUT : TRA_ERR_TIMEOUT;
}

}  // extern "C"
