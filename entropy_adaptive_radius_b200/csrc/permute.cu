// Tile-major permutation and its inverse (Token Radius Attention summary,
// §2 "TRA pipeline", tile-major layout).  A pure HBM copy: every row of d
// elements moves once, 16-byte vectors on both sides.  Each warp owns 32
// consecutive tile-major positions; lane l decodes position l once and the
// warp then streams the 32 rows with lanes spread over the row's 8-element
// chunks, so a warp instruction moves 512 contiguous bytes of output.
#include <cuda_bf16.h>

#include "check.cuh"
#include "tra_internal.h"

namespace tra {
namespace {

template <typename T>
struct Chunk;  // 8 consecutive elements
template <>
struct Chunk<__nv_bfloat16> {
  uint4 v;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { v = __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ __forceinline__ void store(__nv_bfloat16* p) const { *reinterpret_cast<uint4*>(p) = v; }
  __device__ __forceinline__ void to_float(float (&f)[8]) const {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = __bfloat1622float2(h[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
  __device__ __forceinline__ void from_float(const float (&f)[8]) {
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  }
};
template <>
struct Chunk<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ void store(float* p) const {
    reinterpret_cast<float4*>(p)[0] = a;
    reinterpret_cast<float4*>(p)[1] = b;
  }
  __device__ __forceinline__ void to_float(float (&f)[8]) const {
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
  __device__ __forceinline__ void from_float(const float (&f)[8]) {
    a = make_float4(f[0], f[1], f[2], f[3]);
    b = make_float4(f[4], f[5], f[6], f[7]);
  }
};

template <typename Tin, typename Tout>
__device__ __forceinline__ void move_chunk(const Tin* src, Tout* dst) {
  Chunk<Tin> c;
  c.load(src);
  if constexpr (sizeof(Tin) == sizeof(Tout)) {
    Chunk<Tout>& o = reinterpret_cast<Chunk<Tout>&>(c);
    o.store(dst);
  } else {
    float f[8];
    c.to_float(f);
    Chunk<Tout> o;
    o.from_float(f);
    o.store(dst);
  }
}

constexpr int kWarps = 8;
constexpr int kRowsPerWarp = 32;
constexpr int kUnroll = 4;

// grid: (ceil(N / (kWarps*32)), heads).  Forward: dst[p] = src[pi(p)];
// inverse: dst[pi(p)] = src[p].
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kWarps * 32) permute_kernel(const Tin* __restrict__ src,
                                                              Tout* __restrict__ dst, int N, int d,
                                                              TileLayout L, int inverse, int* err) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p0 = (blockIdx.x * kWarps + warp) * kRowsPerWarp;
  if (p0 >= N) return;
  const int h = blockIdx.y;
  const int p = p0 + lane;
  const int mine = (p < N) ? tile_major_source(L, p) : 0;
  const int rows = min(kRowsPerWarp, N - p0);
  const int cpr = d >> 3;  // chunks per row
  const int total = rows * cpr;
  const size_t head_off = static_cast<size_t>(h) * N * d;
  for (int base = 0; base < total; base += 32 * kUnroll) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int c = base + u * 32 + lane;
      const int rr = c / cpr;
      const int cc = c - rr * cpr;
      const int other = __shfl_sync(0xffffffffu, mine, rr < 32 ? rr : 0);
      const int srow = inverse ? p0 + rr : other;
      const int drow = inverse ? other : p0 + rr;
      if (c < total && in_bounds(srow, N, err) && in_bounds(drow, N, err)) {
        move_chunk<Tin, Tout>(src + head_off + static_cast<size_t>(srow) * d + cc * 8,
                              dst + head_off + static_cast<size_t>(drow) * d + cc * 8);
      }
    }
  }
}

template <typename Tin, typename Tout>
cudaError_t launch_typed(const void* src, void* dst, int heads, int d, const TileLayout& L,
                         bool inverse, cudaStream_t stream) {
  const int N = L.F * L.H * L.W;
  const dim3 grid((N + kWarps * kRowsPerWarp - 1) / (kWarps * kRowsPerWarp), heads);
  permute_kernel<Tin, Tout><<<grid, kWarps * 32, 0, stream>>>(
      static_cast<const Tin*>(src), static_cast<Tout*>(dst), N, d, L, inverse ? 1 : 0,
      device_error_word());
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_permute(const void* src, void* dst, tra_dtype in_dtype, tra_dtype out_dtype,
                           int heads, int d, const TileLayout& L, bool inverse,
                           cudaStream_t stream) {
  if (in_dtype == TRA_BF16 && out_dtype == TRA_BF16)
    return launch_typed<__nv_bfloat16, __nv_bfloat16>(src, dst, heads, d, L, inverse, stream);
  if (in_dtype == TRA_F32 && out_dtype == TRA_BF16)
    return launch_typed<float, __nv_bfloat16>(src, dst, heads, d, L, inverse, stream);
  if (in_dtype == TRA_BF16 && out_dtype == TRA_F32)
    return launch_typed<__nv_bfloat16, float>(src, dst, heads, d, L, inverse, stream);
  return launch_typed<float, float>(src, dst, heads, d, L, inverse, stream);
}

}  // namespace tra
