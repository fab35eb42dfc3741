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
#include "tra_internal.h"

namespace tra {
namespace {

__global__ void budget_radius_kernel(const float* __restrict__ H, float* __restrict__ r,
                                     float* __restrict__ phi_out, int N, long long total,
                                     TileLayout L, const __grid_constant__ FrameTables tab) {
  if (phi_out != nullptr && blockIdx.x == 0) {
    for (int t = threadIdx.x; t < L.F; t += blockDim.x) phi_out[t] = tab.phi[t];
  }
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += stride) {
    const int p = static_cast<int>(i % N);
    const int t = tile_major_coord(L, p).t;
    r[i] = tab.coef[t] * expf(0.5f * __ldg(H + i));
  }
}

}  // namespace

cudaError_t launch_budget_radius(const float* H, float* r, float* phi_out, int heads,
                                 const TileLayout& L, const FrameTables& tables,
                                 cudaStream_t stream) {
  const int N = L.F * L.H * L.W;
  const long long total = static_cast<long long>(heads) * N;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long blocks = (total + 255) / 256;
  if (blocks > 8LL * sms) blocks = 8LL * sms;
  if (blocks < 1) blocks = 1;
  budget_radius_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(H, r, phi_out, N, total, L,
                                                                     tables);
  return cudaGetLastError();
}

}  // namespace tra
