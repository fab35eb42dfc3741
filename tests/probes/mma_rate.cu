// Measurement: how long one tcgen05.mma kind::f16 (bf16 in, fp32 in tensor
// memory, cta_group::1, K = 16) takes for M = 64 and M = 128 at N = 64, 128
// and 256.  It decides whether 64-row query blocks could run as exact-work
// M = 64 tiles instead of two blocks per 128-row tile.
// One CTA per SM; thread 0 issues R MMAs back to back into one TMEM
// accumulator, commits once, waits (bounded), clock64 around it.
#include <cstdio>
#include <cstdint>
#include <vector>
#include <algorithm>
#include <cuda_runtime.h>
#include "ptx.cuh"
using namespace tra;

__global__ void __launch_bounds__(128, 1) rate_kernel(int M, int N, int R, long long* cyc, int* err) {
  extern __shared__ uint8_t raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar_storage;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int tid = threadIdx.x;
  // A: 128 rows x 128 B, B: 256 rows x 128 B  (48 KB); fill with small values
  uint32_t* w = reinterpret_cast<uint32_t*>(smem);
  for (int i = tid; i < (48 * 1024) / 4; i += 128) w[i] = 0x3c003c00u;  // bf16 pairs ~ 0.0078
  const uint32_t bar = smem_u32(&bar_storage);
  if (tid == 0) { mbar_init(bar, 1); fence_barrier_init(); abort_flag = 0; }
  if (tid < 32) { tmem_alloc(smem_u32(&tmem_slot), 512); tmem_relinquish(); }
  fence_proxy_async_smem();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const uint32_t sA = smem_u32(smem), sB = sA + 16 * 1024;
  if (tid == 0) {
    const uint32_t idesc = idesc_bf16_f32(M, N, 0, 0);
    const long long t0 = clock64();
    for (int r = 0; r < R; ++r) {
      const int k = r & 3;
      const uint64_t a = smem_desc_sw128(sA + k * 32, 16, 1024);
      const uint64_t b = smem_desc_sw128(sB + k * 32, 16, 1024);
      mma_bf16_ss(tmem, a, b, idesc, r > 0 ? 1u : 0u);
    }
    mma_commit(bar);
    mbar_wait(bar, 0, &abort_flag, err, 1, 2000000000ull);
    const long long t1 = clock64();
    cyc[blockIdx.x] = t1 - t0;
  }
  __syncthreads();
  if (tid < 32) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

int main() {
  int sms = 0; cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
  long long* d_cyc; int* d_err;
  cudaMalloc(&d_cyc, sizeof(long long) * sms); cudaMalloc(&d_err, 4); cudaMemset(d_err, 0, 4);
  const int smem = 120 * 1024;  // one CTA per SM
  cudaFuncSetAttribute(rate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const int R = 8192;
  int cfg[][2] = {{128, 128}, {64, 128}, {128, 256}, {64, 256}, {128, 64}, {64, 64}};
  for (int rep = 0; rep < 2; ++rep)
  for (auto& c : cfg) {
    rate_kernel<<<sms, 128, smem>>>(c[0], c[1], R, d_cyc, d_err);
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) { printf("error %s\n", cudaGetErrorString(e)); return 1; }
    std::vector<long long> h(sms); cudaMemcpy(h.data(), d_cyc, sizeof(long long) * sms, cudaMemcpyDeviceToHost);
    int herr; cudaMemcpy(&herr, d_err, 4, cudaMemcpyDeviceToHost);
    std::sort(h.begin(), h.end());
    const double med = h[sms / 2];
    const double macs = double(c[0]) * c[1] * 16 * R;
    printf("M=%3d N=%3d: %8.0f clk per CTA (median), %6.1f clk/MMA, %7.1f MAC/clk/SM  err=%d\n", c[0], c[1], med, med / R, macs / med, herr);
  }
  return 0;
}
