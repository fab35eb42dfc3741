// Per-block E4M3 quantization of Q and K for the FP8 score path (the block-
// sparse call with QK^T on the tensor cores' 8-bit kind).
//
// For every head and every block of `block` consecutive rows of a bf16
// [heads, N, d] tensor: amax = max |x| over the block, scale = amax / 448
// (rounded to fp32; 1 when the block is all zero), and each element becomes
// the nearest OCP FP8 E4M3 value to x / scale (IEEE division, ties to even,
// saturating at +-448).  One CTA per (block, head); the block (at most
// 128 x 128 bf16 = 32 KiB) stays in registers between the two passes.
// HBM-bound: 2 bytes read and 1 byte written per element.
#include <cuda_bf16.h>

#include "tra_internal.h"

namespace tra {
namespace {

constexpr int kQuantThreads = 256;
constexpr int kQuantChunks = 8;  // 16-byte chunks (8 bf16) held per thread: 128 x 128 / 8 / 256

// two fp32 -> two E4M3 bytes, element a at the lower address
__device__ __forceinline__ uint16_t to_e4m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
  return r;
}

__global__ void __launch_bounds__(kQuantThreads)
    quant_e4m3_kernel(const __nv_bfloat16* __restrict__ X, uint8_t* __restrict__ Xq,
                      float* __restrict__ scales, int N, int d, int block, int nblk) {
  __shared__ float s_amax[kQuantThreads / 32];
  const int b = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const int row0 = b * block;
  const int rows = min(block, N - row0);
  const int cpr = d / 8;                 // chunks per row
  const int nchunk = rows * cpr;
  const size_t base = (static_cast<size_t>(h) * N + row0) * d;
  uint4 v[kQuantChunks];
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < kQuantChunks; ++k) {
    const int c = tid + k * kQuantThreads;
    if (c < nchunk) {
      v[k] = __ldg(reinterpret_cast<const uint4*>(X + base) + c);
      const __nv_bfloat162* e = reinterpret_cast<const __nv_bfloat162*>(&v[k]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(e[i]);
        amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
  }
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((tid & 31) == 0) s_amax[tid >> 5] = amax;
  __syncthreads();
  if (tid < 32) {
    float a = tid < kQuantThreads / 32 ? s_amax[tid] : 0.f;
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (tid == 0) s_amax[0] = a;
  }
  __syncthreads();
  const float am = s_amax[0];
  const float sc = am > 0.f ? __fdiv_rn(am, 448.f) : 1.f;
  if (tid == 0) scales[static_cast<size_t>(h) * nblk + b] = sc;
#pragma unroll
  for (int k = 0; k < kQuantChunks; ++k) {
    const int c = tid + k * kQuantThreads;
    if (c < nchunk) {
      const __nv_bfloat162* e = reinterpret_cast<const __nv_bfloat162*>(&v[k]);
      uint32_t w[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float2 f0 = __bfloat1622float2(e[2 * i]), f1 = __bfloat1622float2(e[2 * i + 1]);
        const uint16_t lo = to_e4m3x2(__fdiv_rn(f0.x, sc), __fdiv_rn(f0.y, sc));
        const uint16_t hi = to_e4m3x2(__fdiv_rn(f1.x, sc), __fdiv_rn(f1.y, sc));
        w[i] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
      }
      reinterpret_cast<uint2*>(Xq + base)[c] = make_uint2(w[0], w[1]);
    }
  }
}

}  // namespace

cudaError_t launch_quantize_e4m3(const void* X, void* Xq, float* scales, int heads, int N, int d,
                                 int block, cudaStream_t stream) {
  const int nblk = (N + block - 1) / block;
  quant_e4m3_kernel<<<dim3(nblk, heads), kQuantThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(X), static_cast<uint8_t*>(Xq), scales, N, d, block, nblk);
  return cudaGetLastError();
}

}  // namespace tra
