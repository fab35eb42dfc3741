// Entropy -> budget -> radius (Token Radius Attention summary, §2 Insight I:
// B_i = tau * exp(H_i) / N; Insight II: the budget becomes a query-centred
// radius, scaled per key frame by phi(delta) = exp(-gamma * delta)).
//
// Equal-area reading: the disks of all key frames hold K_i = B_i * N tokens,
// K_i = pi * r_i^2 * S(t_i) with S(t) = sum_t' phi(|t' - t|)^2, hence
//   r_i = sqrt(tau / (pi * S(t_i))) * exp(H_i / 2).
// The per-frame factor sqrt(tau / (pi * S(t))) is formed on the host in double
// and rounded once; the kernel multiplies it by expf(0.5 * H).  Elementwise,
// HBM-bound (8 bytes per query).
//
// Variants (the ablations of the summary's §4, and Radial Attention's static
// window):
//  - 1D distance: equal length, K_i = 2 r_i L(t_i) with L(t) = sum_t' phi(|t'-t|),
//    r_i = (tau / (2 L(t_i))) * exp(H_i); same kernel, exponent 1 instead of 1/2.
//  - shared budget: one CTA per head sums exp(H_i) in double, K_h = tau * mean,
//    and every query gets sqrt(K_h / (pi S(t))) (or K_h / (2 L(t))), evaluated
//    in double and rounded once.
//  - Radial's static window: r_i = r0 for every query, with the band table
//    phi_R(delta) = 2^(-b/2) (disk) or 2^(-b) (1D), b = floor(log2(delta + 1)).
#include "check.cuh"
#include "tra_internal.h"

namespace tra {
namespace {

__global__ void budget_radius_kernel(const float* __restrict__ H, float* __restrict__ r,
                                     float* __restrict__ phi_out, int N, long long total,
                                     TileLayout L, float hexp,
                                     const __grid_constant__ FrameTables tab, int* err) {
  if (phi_out != nullptr && blockIdx.x == 0) {
    for (int t = threadIdx.x; t < L.F; t += blockDim.x) phi_out[t] = tab.phi[t];
  }
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += stride) {
    const int p = static_cast<int>(i % N);
    const int t = tile_major_coord(L, p).t;
    if (!in_bounds(t, L.F, err)) continue;
    r[i] = tab.coef[t] * expf(hexp * __ldg(H + i));
  }
}

constexpr int kSharedThreads = 1024;

// grid = heads.  K_h = tau * (sum_i exp(H_i)) / N in double (fixed reduction
// order: per-thread strided sums, then a warp tree and a tree over warps).
__global__ void __launch_bounds__(kSharedThreads)
shared_budget_kernel(const float* __restrict__ H, float* __restrict__ r,
                     float* __restrict__ phi_out, int N, TileLayout L, double tau, bool line,
                     const __grid_constant__ FrameTablesD tab, int* err) {
  __shared__ double s_part[kSharedThreads / 32];
  const int h = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (phi_out != nullptr && h == 0) {
    for (int t = tid; t < L.F; t += kSharedThreads) phi_out[t] = tab.phi[t];
  }
  const float* Hh = H + static_cast<size_t>(h) * N;
  double acc = 0.0;
  for (int i = tid; i < N; i += kSharedThreads) acc += exp(static_cast<double>(__ldg(Hh + i)));
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) s_part[warp] = acc;
  __syncthreads();
  if (warp == 0) {
    double v = s_part[lane];
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) s_part[0] = v;
  }
  __syncthreads();
  const double K = tau * (s_part[0] / static_cast<double>(N));
  float* rh = r + static_cast<size_t>(h) * N;
  for (int i = tid; i < N; i += kSharedThreads) {
    const int t = tile_major_coord(L, i).t;
    if (!in_bounds(t, L.F, err)) continue;
    const double c = tab.c[t];
    rh[i] = static_cast<float>(line ? K * c : sqrt(K * c));
  }
}

__global__ void fill_radius_kernel(float* __restrict__ r, long long total, float r0,
                                   float* __restrict__ phi_out, int F,
                                   const __grid_constant__ FrameTables tab) {
  if (phi_out != nullptr && blockIdx.x == 0) {
    for (int t = threadIdx.x; t < F; t += blockDim.x) phi_out[t] = tab.phi[t];
  }
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += stride)
    r[i] = r0;
}

long long elementwise_blocks(long long total) {
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long blocks = (total + 255) / 256;
  if (blocks > 8LL * sms) blocks = 8LL * sms;
  if (blocks < 1) blocks = 1;
  return blocks;
}

}  // namespace

cudaError_t launch_budget_radius(const float* H, float* r, float* phi_out, int heads,
                                 const TileLayout& L, const FrameTables& tables, bool line,
                                 cudaStream_t stream) {
  const int N = L.F * L.H * L.W;
  const long long total = static_cast<long long>(heads) * N;
  const long long blocks = elementwise_blocks(total);
  budget_radius_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(
      H, r, phi_out, N, total, L, line ? 1.0f : 0.5f, tables, device_error_word());
  return cudaGetLastError();
}

cudaError_t launch_shared_budget_radius(const float* H, float* r, float* phi_out, int heads,
                                        const TileLayout& L, double tau, bool line,
                                        const FrameTablesD& tables, cudaStream_t stream) {
  const int N = L.F * L.H * L.W;
  shared_budget_kernel<<<heads, kSharedThreads, 0, stream>>>(H, r, phi_out, N, L, tau, line,
                                                             tables, device_error_word());
  return cudaGetLastError();
}

cudaError_t launch_fill_radius(float* r, float* phi_out, int heads, const TileLayout& L, float r0,
                               const FrameTables& tables, cudaStream_t stream) {
  const long long total = static_cast<long long>(heads) * L.F * L.H * L.W;
  const long long blocks = elementwise_blocks(total);
  fill_radius_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(r, total, r0, phi_out, L.F,
                                                                   tables);
  return cudaGetLastError();
}

}  // namespace tra
