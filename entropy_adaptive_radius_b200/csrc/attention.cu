// Attention on tcgen05 tensor cores: the dense warm-up pass with per-query
// entropy, and exact block-sparse attention over a CSR block list.
//
// Token Radius Attention summary (gist.science 2608.02504): §2 "TRA pipeline"
// step 1 (entropy of every query from a dense warm-up pass), §3 contribution 3
// (fused entropy kernel), efficient execution (block-sparse attention over the
// kept query-block x key-block pairs, reused across sparse steps).
//
// Three kernels, each with one CTA per (128-row query tile, head):
//   attn_dual_kernel  the dense pass and block-sparse attention with 64- or
//                     128-token blocks: two softmax warpgroups split the key
//                     blocks, separate K / V producers and QK / PV issuers
//                     (described at the kernel);
//   attn_kernel       block-sparse attention when a block is 16 tokens (up to
//                     eight query blocks per tile, their lists merged in shared
//                     memory): one softmax warpgroup;
//   entropy_kernel    the entropy-only pass (no PV, no output).
// In all of them thread i of a softmax warpgroup owns query row i (TMEM lane
// i): it reads the score tile S_j and keeps the running max m, Z = sum 2^(u-m)
// and A = sum 2^(u-m) (u-m) (u = s * log2 e).  The two attention kernels also
// write P_j (bf16) to shared memory in the MMA's swizzled layout, rescale O
// when the max grows by more than 2^8, and finally write O / Z; all three
// write the entropy H = ln Z - ln 2 * A / Z (dense and entropy-only) and
// LSE = ln 2 * (m + log2 Z).  The tensor cores compute the next score tile
// while the softmax of the current one runs.
//
// attn_kernel's warp roles: warp 0 TMA producer (Q once, then K and V into a
// 2-stage ring), warp 1 MMA issuer (S_j into one of two TMEM score buffers,
// O += P_j V_j), warp 2 tensor-memory allocation, warps 4..7 softmax.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <climits>
#include <cmath>
#include <mutex>

#include "ptx.cuh"
#include "tra_internal.h"

namespace tra {
namespace {

constexpr int BM = 128;                    // query rows per CTA
constexpr int kThreads = 256;              // 8 warps
constexpr int kMaxUnion = 1024;            // key blocks of a merged list
constexpr int kMaxGroups = 8;              // query blocks per CTA (128 / 16)
constexpr float kRescaleLog2 = 8.0f;       // lazy rescale threshold (log2 units)
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;

__host__ __device__ constexpr int pow2_at_least(int x) {
  int p = 32;
  while (p < x) p <<= 1;
  return p;
}

template <int D, int BK>
struct Cfg {
  static constexpr int NS = 2;                          // K and V ring depth
  static constexpr int KCH = D / 64;                    // 128-byte groups of a Q/K/V row
  static constexpr int PCH = (BK + 63) / 64;            // 128-byte groups of a P row
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BK * D * 2;
  static constexpr int P_BYTES = PCH * BM * 128;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr int OFF_P = OFF_V + NS * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int NUM_BARS = 1 + 4 * NS + 6;
  static constexpr int OFF_MISC = OFF_BAR + 256;
  static constexpr int OFF_LIST = OFF_MISC + 64;
  static constexpr int OFF_QBMAP = OFF_LIST + kMaxUnion * 4;
  static constexpr int USED = OFF_QBMAP + kMaxGroups * 32 * 4;
  static constexpr int TMEM_COLS = pow2_at_least(2 * BK + D);
  // 512 tensor-memory columns fill an SM: make sure a second CTA cannot be
  // co-resident (it would only wait for the first to free the columns).
  static constexpr int SMEM = (TMEM_COLS == 512 && USED < 120 * 1024 ? 120 * 1024 : USED) + 1024;
  static_assert(Q_BYTES % 1024 == 0 && KV_BYTES % 1024 == 0, "swizzle atoms need 1 KiB alignment");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(NUM_BARS * 8 <= 256, "barrier area");
};

struct Params {
  int N, nqb, nkb, bq, G;
  float scale_log2;
  const int* row_ptr;
  const int* col_idx;
  const float* q_scales;  // FP8 scores: per (head, query block) scale of Q
  const float* k_scales;  // FP8 scores: per (head, key block) scale of K
  __nv_bfloat16* O;
  float* H;
  float* lse;
  int* err;
};

__device__ __forceinline__ void tmem_ld16f(uint32_t taddr, float* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]),
        "=f"(v[7]), "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]),
        "=f"(v[14]), "=f"(v[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st16f(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]),
      "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]),
      "f"(v[15])
      : "memory");
}

// 2^x on the MUFU unit (flushes subnormal results to zero; 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ void tmem_ld32f(uint32_t taddr, float* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]),
        "=f"(v[7]), "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]),
        "=f"(v[14]), "=f"(v[15]), "=f"(v[16]), "=f"(v[17]), "=f"(v[18]), "=f"(v[19]),
        "=f"(v[20]), "=f"(v[21]), "=f"(v[22]), "=f"(v[23]), "=f"(v[24]), "=f"(v[25]),
        "=f"(v[26]), "=f"(v[27]), "=f"(v[28]), "=f"(v[29]), "=f"(v[30]), "=f"(v[31])
      : "r"(taddr)
      : "memory");
}

template <int N>
__device__ __forceinline__ void freg_fence(float* v) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+f"(v[i]));
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// Bounded wait that ignores the abort flag (used to drain copies in flight).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const unsigned long long t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > 500000000ull) break;
  }
}

template <int D, int BK, bool DENSE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const Params p) {
  using C = Cfg<D, BK>;
  constexpr int NS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sK = sbase + C::OFF_K;
  const uint32_t sV = sbase + C::OFF_V;
  const uint32_t sP = sbase + C::OFF_P;
  const uint32_t bars = sbase + C::OFF_BAR;
  const uint32_t bar_q = bars;
  auto k_full = [&](int s) { return bars + 8u * (1 + s); };
  auto k_empty = [&](int s) { return bars + 8u * (1 + NS + s); };
  auto v_full = [&](int s) { return bars + 8u * (1 + 2 * NS + s); };
  auto v_empty = [&](int s) { return bars + 8u * (1 + 3 * NS + s); };
  auto s_full = [&](int b) { return bars + 8u * (1 + 4 * NS + b); };
  auto s_free = [&](int b) { return bars + 8u * (3 + 4 * NS + b); };
  const uint32_t p_full = bars + 8u * (5 + 4 * NS);
  const uint32_t pv_done = bars + 8u * (6 + 4 * NS);
  volatile int* misc = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
  // misc[0] tmem base, misc[1] abort, misc[2] block count, misc[3] CSR start
  volatile int* abort = misc + 1;
  int* list = reinterpret_cast<int*>(smem + C::OFF_LIST);
  uint32_t* qbmap = reinterpret_cast<uint32_t*>(smem + C::OFF_QBMAP);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int qt = blockIdx.x, h = blockIdx.y;

  if (tid == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full(b), 1);
      mbar_init(s_free(b), 128);
    }
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    fence_barrier_init();
    misc[1] = 0;
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(const_cast<int*>(misc)), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 32) {
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
  }

  // ---- key-block list of this CTA
  if constexpr (DENSE) {
    if (tid == 0) misc[2] = p.nkb;
  } else {
    const int* rp = p.row_ptr + static_cast<size_t>(h) * (p.nqb + 1);
    if (p.G == 1) {
      if (tid == 0) {
        const int st = rp[qt], en = rp[qt + 1];
        int n = en - st;
        if (st < 0 || n < 0 || n > p.nkb) {
          n = 0;
          atomicCAS(p.err, 0, kErrBadCsr);
        }
        misc[2] = n;
        misc[3] = st;
      }
    } else {
      const int nkbw = (p.nkb + 31) >> 5;
      for (int i = tid; i < kMaxGroups * 32; i += kThreads) qbmap[i] = 0u;
      __syncthreads();
      for (int g = 0; g < p.G; ++g) {
        const int qb = qt * p.G + g;
        if (qb >= p.nqb) break;
        const int st = rp[qb], en = rp[qb + 1];
        if (st < 0 || en - st < 0 || en - st > p.nkb) {
          if (tid == 0) atomicCAS(p.err, 0, kErrBadCsr);
          continue;
        }
        for (int e = st + tid; e < en; e += kThreads) {
          const int kb = p.col_idx[e];
          if (kb >= 0 && kb < p.nkb) atomicOr(&qbmap[g * 32 + (kb >> 5)], 1u << (kb & 31));
        }
      }
      __syncthreads();
      if (warp == 0) {
        int run = 0;
        for (int base = 0; base < nkbw; base += 32) {
          const int w = base + lane;
          uint32_t word = 0;
          if (w < nkbw)
            for (int g = 0; g < p.G; ++g) word |= qbmap[g * 32 + w];
          const int c = __popc(word);
          int incl = c;
          for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
          }
          int pos = run + incl - c;
          while (word) {
            const int b = __ffs(word) - 1;
            word &= word - 1;
            list[pos++] = w * 32 + b;
          }
          run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) misc[2] = run;
      }
    }
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);
  const int nblk = misc[2];
  const int csr_start = misc[3];

  auto kb_at = [&](int j) -> int {
    if constexpr (DENSE) {
      return j;
    } else {
      return p.G == 1 ? __ldg(p.col_idx + csr_start + j) : list[j];
    }
  };

  if (warp == 0) {
    // ===================================================== TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_q, C::Q_BYTES);
#pragma unroll
      for (int c = 0; c < C::KCH; ++c) tma_load_3d(sQ + c * (BM * 128), &tmQ, c * 64, qt * BM, h, bar_q);
      int issued = 0;
      for (int j = 0; j < nblk; ++j) {
        const int s = j % NS;
        const uint32_t ph = (j / NS) & 1;
        const int kb = kb_at(j);
        if (!mbar_wait(k_empty(s), ph ^ 1u, abort, p.err, kErrWaitKEmpty)) break;
        mbar_arrive_expect_tx(k_full(s), C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d(sK + s * C::KV_BYTES + c * (BK * 128), &tmK, c * 64, kb * BK, h, k_full(s));
        if (!mbar_wait(v_empty(s), ph ^ 1u, abort, p.err, kErrWaitVEmpty)) {
          issued = -(j + 1);  // K of block j in flight, V not
          break;
        }
        mbar_arrive_expect_tx(v_full(s), C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d(sV + s * C::KV_BYTES + c * (BK * 128), &tmV, c * 64, kb * BK, h, v_full(s));
        issued = j + 1;
      }
      if (*abort) {
        // let every copy still in flight land before the CTA can exit
        drain_wait(bar_q, 0);
        const int kdone = issued >= 0 ? issued : -issued;
        const int vdone = issued >= 0 ? issued : -issued - 1;
        for (int j = (kdone > NS ? kdone - NS : 0); j < kdone; ++j)
          drain_wait(k_full(j % NS), (j / NS) & 1);
        for (int j = (vdone > NS ? vdone - NS : 0); j < vdone; ++j)
          drain_wait(v_full(j % NS), (j / NS) & 1);
      }
    }
  } else if (warp == 1) {
    // ===================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescQK = idesc_bf16_f32(BM, BK, 0, 0);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(BM, D, 0, 1);
      const uint32_t tO = tmem + 2 * BK;
      auto issue_pv = [&](int i) -> bool {
        const int s = i % NS;
        if (!mbar_wait(p_full, i & 1, abort, p.err, kErrWaitPFull)) return false;
        if (!mbar_wait(v_full(s), (i / NS) & 1, abort, p.err, kErrWaitVFull)) return false;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < BK / 16; ++k) {
          const uint64_t a = smem_desc_sw128(sP + (k >> 2) * (BM * 128) + (k & 3) * 32, 16, 1024);
          const uint64_t b = smem_desc_sw128(sV + s * C::KV_BYTES + k * 16 * 128, BK * 128, 1024);
          mma_bf16_ss(tO, a, b, kIdescPV, (i > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(v_empty(s));
        mma_commit(pv_done);
        return true;
      };
      bool ok = mbar_wait(bar_q, 0, abort, p.err, kErrWaitQ);
      for (int j = 0; ok && j < nblk; ++j) {
        const int s = j % NS;
        const int b = j & 1;
        if (!mbar_wait(k_full(s), (j / NS) & 1, abort, p.err, kErrWaitKFull)) { ok = false; break; }
        if (!mbar_wait(s_free(b), ((j >> 1) & 1) ^ 1u, abort, p.err, kErrWaitSFree)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tS = tmem + b * BK;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t a = smem_desc_sw128(sQ + (k >> 2) * (BM * 128) + (k & 3) * 32, 16, 1024);
          const uint64_t bd =
              smem_desc_sw128(sK + s * C::KV_BYTES + (k >> 2) * (BK * 128) + (k & 3) * 32, 16, 1024);
          mma_bf16_ss(tS, a, bd, kIdescQK, k > 0 ? 1u : 0u);
        }
        mma_commit(k_empty(s));
        mma_commit(s_full(b));
        if (j > 0 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && nblk > 0) ok = issue_pv(nblk - 1);
      if (!ok) {
        // wait for every MMA issued so far before tensor memory is freed
        const uint32_t drain = bars + 8u * (C::NUM_BARS);
        mbar_init(drain, 1);
        fence_barrier_init();
        mma_commit(drain);
        drain_wait(drain, 0);
      }
    }
  } else if (warp >= 4) {
    // ===================================================== softmax / epilogue
    const int row = tid - 128;
    const uint32_t tl = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int qpos = qt * BM + row;
    const bool valid_row = qpos < p.N;
    const int g = DENSE ? 0 : row / p.bq;
    float m_ref = -INFINITY, Z = 0.f, A = 0.f;
    bool ok = true;
    float sv[BK];
    for (int j = 0; j < nblk; ++j) {
      const int b = j & 1;
      const int kb = kb_at(j);
      ok = mbar_wait(s_full(b), (j >> 1) & 1, abort, p.err, kErrWaitSFull);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      if constexpr (BK % 32 == 0) {
#pragma unroll
        for (int c = 0; c < BK / 32; ++c) tmem_ld32f(tmem + tl + b * BK + c * 32, sv + c * 32);
      } else {
#pragma unroll
        for (int c = 0; c < BK / 16; ++c) tmem_ld16f(tmem + tl + b * BK + c * 16, sv + c * 16);
      }
      tmem_wait_ld();
      freg_fence<BK>(sv);
      tc_fence_before();
      mbar_arrive(s_free(b));

      int nvalid = p.N - kb * BK;
      if constexpr (!DENSE) {
        if (kb < 0 || kb >= p.nkb) nvalid = 0;
        else if (p.G > 1 && !((qbmap[g * 32 + (kb >> 5)] >> (kb & 31)) & 1u)) nvalid = 0;
      }
      // Running max with lazy rescale: the reference m_ref moves only when the
      // block max exceeds it by more than 2^8; then Z, A (and O, below) are
      // scaled by alpha = 2^(m_ref - m_new).
      float alpha = 1.f;
      bool o_rescale = false;
      auto update_max = [&](float bmax) {
        const float m_new = fmaxf(m_ref, bmax);
        if (m_new > m_ref + kRescaleLog2) {
          if (m_ref != -INFINITY) {
            alpha = ex2_approx(m_ref - m_new);
            A = alpha * (A + (m_ref - m_new) * Z);
            Z *= alpha;
            o_rescale = j > 0;
          }
          m_ref = m_new;
        }
      };
      uint32_t pk[BK / 2];  // P_j as packed bf16 pairs
      if (__all_sync(0xffffffffu, nvalid >= BK)) {
        // Unmasked block (every row of the warp sees all BK keys).
        // Row max of the raw scores (scale > 0 commutes with max): four
        // independent chains of 3-input max.
        float mx[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) mx[i] = fmaxf(sv[i], sv[4 + i]);
#pragma unroll
        for (int c = 8; c < BK; c += 8) {
#pragma unroll
          for (int i = 0; i < 4; ++i) mx[i] = fmax3(mx[i], sv[c + i], sv[c + 4 + i]);
        }
        update_max(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2);
        // m_ref is finite here.  x = s * scale * log2(e) - m_ref, p = 2^x,
        // Z += p, A += p * x, two lanes per instruction, four partial sums.
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 nm2 = make_float2(-m_ref, -m_ref);
        float2 z2[4], a2[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) z2[i] = a2[i] = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < BK / 2; ++c) {
          const float2 x = __ffma2_rn(make_float2(sv[2 * c], sv[2 * c + 1]), sc2, nm2);
          const float2 pr = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          z2[c & 3] = __fadd2_rn(z2[c & 3], pr);
          if constexpr (DENSE) a2[c & 3] = __ffma2_rn(pr, x, a2[c & 3]);
          pk[c] = pack_bf16(pr.x, pr.y);
        }
        const float2 zz = __fadd2_rn(__fadd2_rn(z2[0], z2[1]), __fadd2_rn(z2[2], z2[3]));
        Z += zz.x + zz.y;
        if constexpr (DENSE) {
          const float2 aa = __fadd2_rn(__fadd2_rn(a2[0], a2[1]), __fadd2_rn(a2[2], a2[3]));
          A += aa.x + aa.y;
        }
      } else if (__all_sync(0xffffffffu, nvalid <= 0)) {
        // No row of the warp keeps this block: P = 0, statistics unchanged.
#pragma unroll
        for (int c = 0; c < BK / 2; ++c) pk[c] = 0u;
      } else {
        // Partly masked block (the last, partial key block, or rows of a
        // merged list that do not keep this block): masked keys get -inf.
        float bm0 = -INFINITY, bm1 = -INFINITY;
#pragma unroll
        for (int c = 0; c < BK; c += 2) {
          const float u0 = c < nvalid ? sv[c] * p.scale_log2 : -INFINITY;
          const float u1 = c + 1 < nvalid ? sv[c + 1] * p.scale_log2 : -INFINITY;
          sv[c] = u0;
          sv[c + 1] = u1;
          bm0 = fmaxf(bm0, u0);
          bm1 = fmaxf(bm1, u1);
        }
        update_max(fmaxf(bm0, bm1));
        const float mc = (m_ref == -INFINITY) ? 0.f : m_ref;
        float zs0 = 0.f, zs1 = 0.f, as0 = 0.f, as1 = 0.f;
#pragma unroll
        for (int c = 0; c < BK / 2; ++c) {
          const float x0 = sv[2 * c] - mc, x1 = sv[2 * c + 1] - mc;
          const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          zs0 += p0;
          zs1 += p1;
          if constexpr (DENSE) {
            as0 += p0 > 0.f ? p0 * x0 : 0.f;
            as1 += p1 > 0.f ? p1 * x1 : 0.f;
          }
          pk[c] = pack_bf16(p0, p1);
        }
        Z += zs0 + zs1;
        A += as0 + as1;
      }

      if (j > 0) {
        ok = mbar_wait(pv_done, (j - 1) & 1, abort, p.err, kErrWaitPVDone);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      tc_fence_after();
      if (__any_sync(0xffffffffu, o_rescale)) {
        const float a = o_rescale ? alpha : 1.f;
#pragma unroll
        for (int c = 0; c < D; c += 16) {
          float o[16];
          tmem_ld16f(tmem + tl + 2 * BK + c, o);
          tmem_wait_ld();
          freg_fence<16>(o);
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] *= a;
          tmem_st16f(tmem + tl + 2 * BK + c, o);
        }
        tmem_wait_st();
      }
#pragma unroll
      for (int c8 = 0; c8 < BK / 8; ++c8) {
        const uint32_t addr = sP + (c8 >> 3) * (BM * 128) + row * 128 + (((c8 & 7) ^ (row & 7)) << 4);
        st_shared_v4(addr, pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && nblk > 0) {
      ok = mbar_wait(pv_done, (nblk - 1) & 1, abort, p.err, kErrWaitPVDone);
      ok = __all_sync(0xffffffffu, ok);
    }
    tc_fence_after();
    const float inv = Z > 0.f ? 1.f / Z : 0.f;
    __nv_bfloat16* orow = p.O + (static_cast<size_t>(h) * p.N + (valid_row ? qpos : 0)) * D;
    if (ok && nblk > 0) {
#pragma unroll
      for (int c = 0; c < D; c += 16) {
        float o[16];
        tmem_ld16f(tmem + tl + 2 * BK + c, o);
        tmem_wait_ld();
        freg_fence<16>(o);
        if (valid_row) {
          uint4 w0, w1;
          w0.x = pack_bf16(o[0] * inv, o[1] * inv);
          w0.y = pack_bf16(o[2] * inv, o[3] * inv);
          w0.z = pack_bf16(o[4] * inv, o[5] * inv);
          w0.w = pack_bf16(o[6] * inv, o[7] * inv);
          w1.x = pack_bf16(o[8] * inv, o[9] * inv);
          w1.y = pack_bf16(o[10] * inv, o[11] * inv);
          w1.z = pack_bf16(o[12] * inv, o[13] * inv);
          w1.w = pack_bf16(o[14] * inv, o[15] * inv);
          reinterpret_cast<uint4*>(orow + c)[0] = w0;
          reinterpret_cast<uint4*>(orow + c)[1] = w1;
        }
      }
    } else if (valid_row) {
      for (int c = 0; c < D; c += 8) reinterpret_cast<uint4*>(orow + c)[0] = make_uint4(0, 0, 0, 0);
    }
    if (valid_row) {
      const size_t idx = static_cast<size_t>(h) * p.N + qpos;
      if (DENSE && p.H != nullptr) p.H[idx] = Z > 0.f ? logf(Z) - kLn2 * (A / Z) : NAN;
      if (p.lse != nullptr) p.lse[idx] = Z > 0.f ? kLn2 * (m_ref + log2f(Z)) : -INFINITY;
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Two-warpgroup kernel: the dense pass and block-sparse attention with 64- or
// 128-token blocks (16-token blocks use attn_kernel above).
//
// The CTA owns one 128-row query tile.  Its key-block list is split between
// two softmax warpgroups: warpgroup w (warps 4w .. 4w+3) takes blocks
// j = w, w + 2, w + 4, ... with its own TMEM score tile S_w, its own TMEM output
// accumulator O_w, its own bf16 P_w buffer in shared memory and its own
// running statistics (m_w, Z_w, A_w).  Each warpgroup therefore has two block
// periods of tensor-core work to hide one softmax iteration, and each
// scheduler has two softmax warps to issue from.  QK^T runs two blocks ahead
// of PV (S_{j+2} as soon as warpgroup j mod 2 has read S_j), so a score tile
// is ready when its warpgroup finishes the previous one.  K and V
// have separate producer warps so that prefetching K never waits behind a V
// slot that is still in use.  At the end the two partial results are merged
// exactly:
//   m = max(m_0, m_1),  a_w = 2^(m_w - m),  Z = a_0 Z_0 + a_1 Z_1,
//   A = sum_w a_w (A_w + (m_w - m) Z_w),      O = (a_0 O_0 + a_1 O_1) / Z.
// Warps: 0..7 softmax, 8 Q/K producer (and tensor-memory allocation), 9 QK
// issuer, 10 V producer, 11 PV issuer.  QK and PV are issued by two threads,
// each in block order and each sleeping in its own barrier waits, so neither
// stream holds back the other and no warp spins on the softmax warps' issue
// slots.  The third warpgroup (warps 8..11) hands registers to the two
// softmax warpgroups (setmaxnreg): 168 per thread at launch, 56 for the
// producers and issuers, 224 for the softmax.
//
// Key blocks of 64 tokens are taken two at a time: a "super-block" of 128
// keys is the next two entries of the CTA's key-block list, each loaded into
// half of a K/V stage (a missing second entry loads rows past N, which read as
// zeros).  When query blocks have 64 rows the CTA's 128 rows hold two query
// blocks; its list is the merge of their two CSR rows, and each row leaves
// out the entries its own query block does not keep.  The prologue counts the
// merge from bitmaps of both rows (all threads) and, up to 384 entries, writes
// it to shared memory with membership bits; the softmax reads its entries
// there (and walks the two rows beyond that size), the producers and issuers
// walk the merge themselves, in the same order.  With two 64-key entries a
// warp (64 rows of one query block) keeps each half of a super-block whole or
// not at all, except in the sequence's last key block: an unkept half is left
// out of the row max and takes no exponentials (its P is stored as zeros).
// ---------------------------------------------------------------------------

constexpr int kDualThreads = 384;  // 12 warps
constexpr int kDualKWarp = 8;
constexpr int kDualQKWarp = 9;
constexpr int kDualVWarp = 10;
constexpr int kDualPVWarp = 11;
// Register split.  The CTA is launched with kDualLaunchRegs per thread (the
// host refuses to launch a build that allocated anything else); the split
// hands exactly that pool out again, so setmaxnreg.inc never waits.
constexpr int kDualLaunchRegs = 168;
constexpr int kDualRegsOther = 56;
constexpr int kDualRegsSoftmax = 224;
static_assert(256 * kDualRegsSoftmax + 128 * kDualRegsOther == kDualThreads * kDualLaunchRegs,
              "register split must equal the launch pool");
static_assert(2 * kDualRegsSoftmax * 32 + kDualRegsOther * 32 <= 16384,
              "per-scheduler register file: two softmax warps and one other warp");

template <int D, bool FP8 = false>
struct DualCfg {
  static constexpr int BK = 128;  // keys per super-block
  static constexpr int NS = 2;
  static constexpr int QE = FP8 ? 1 : 2;       // bytes per Q / K element
  static constexpr int QKCH = D * QE / 128;    // 128-byte chunks of a Q / K row
  static constexpr int QKX = 128 / QE;         // elements per chunk (TMA box width)
  static constexpr int KSTEPS = D * QE / 32;   // MMA K-steps of QK^T (32 bytes each)
  static constexpr int KCH = D / 64;           // 128-byte chunks of a V row (bf16)
  static constexpr int Q_BYTES = BM * D * QE;
  static constexpr int K_BYTES = BK * D * QE;  // one K stage
  static constexpr int KV_BYTES = BK * D * 2;  // one V stage
  static constexpr int P_BYTES = 2 * BM * 128;  // one P_w buffer (128 rows x 128 keys bf16)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * K_BYTES;
  static constexpr int OFF_P = OFF_V + NS * KV_BYTES;  // P_0, P_1
  static constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
  static constexpr int NUM_BARS = 1 + 4 * NS + 8 + 2;
  static constexpr int OFF_MISC = OFF_BAR + 256;
  // merged key-block list of a tile's two query blocks (entries with their
  // membership bits), when it has at most kUnionCap entries
  static constexpr int kUnionCap = 384;
  static constexpr int OFF_LIST = OFF_MISC + 64;
  static constexpr int USED = OFF_LIST + kUnionCap * 4;
  static constexpr int SMEM = (USED < 120 * 1024 ? 120 * 1024 : USED) + 1024;
  static constexpr int TMEM_COLS = 512;  // S_0, S_1 (128 each), O_0, O_1 (D each)
  static_assert(2 * BK + 2 * D <= TMEM_COLS, "tensor memory");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(NUM_BARS * 8 <= 256, "barrier area");
  static_assert(!FP8 || D == 128, "FP8 scores: one 128-byte E4M3 row per query / key");
  static_assert(Q_BYTES % 1024 == 0 && K_BYTES % 1024 == 0, "swizzle atoms need 1 KiB alignment");
};

__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Walks the ascending union of up to two CSR rows (a, b), one entry per call:
// returns the key block (-1 once both rows are exhausted) and sets `mem` to
// bit 0 if the entry is in row a, bit 1 if it is in row b.
struct ListWalker {
  const int* a;
  const int* b;
  int na, nb, ia, ib;
  __device__ __forceinline__ int next(uint32_t& mem) {
    const int va = ia < na ? __ldg(a + ia) : INT_MAX;
    const int vb = ib < nb ? __ldg(b + ib) : INT_MAX;
    if (va == INT_MAX && vb == INT_MAX) {
      mem = 0u;
      return -1;
    }
    if (va < vb) {
      ++ia;
      mem = 1u;
      return va;
    }
    if (vb < va) {
      ++ib;
      mem = 2u;
      return vb;
    }
    ++ia;
    ++ib;
    mem = 3u;
    return va;
  }
};

template <int D, int BKS, bool DENSE, bool FP8 = false, bool SINGLE = true>
__global__ void __launch_bounds__(kDualThreads, 1)
    attn_dual_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const Params p) {
  using C = DualCfg<D, FP8>;
  static_assert(!FP8 || (BKS == 128 && !DENSE), "FP8 scores: block-sparse, 128-key blocks");
  constexpr int NS = C::NS;
  constexpr int BK = C::BK;
  constexpr int E = BK / BKS;  // list entries per super-block (1 or 2)
  static_assert(BKS == 64 || BKS == 128, "key block size");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sK = sbase + C::OFF_K;
  const uint32_t sV = sbase + C::OFF_V;
  const uint32_t sP = sbase + C::OFF_P;
  const uint32_t bars = sbase + C::OFF_BAR;
  const uint32_t bar_q = bars;
  auto k_full = [&](int s) { return bars + 8u * (1 + s); };
  auto k_empty = [&](int s) { return bars + 8u * (1 + NS + s); };
  auto v_full = [&](int s) { return bars + 8u * (1 + 2 * NS + s); };
  auto v_empty = [&](int s) { return bars + 8u * (1 + 3 * NS + s); };
  auto s_full = [&](int w) { return bars + 8u * (1 + 4 * NS + w); };
  auto s_free = [&](int w) { return bars + 8u * (3 + 4 * NS + w); };
  auto p_full = [&](int w) { return bars + 8u * (5 + 4 * NS + w); };
  auto pv_done = [&](int w) { return bars + 8u * (7 + 4 * NS + w); };
  const uint32_t drain_qk = bars + 8u * (9 + 4 * NS);
  const uint32_t drain_pv = bars + 8u * (10 + 4 * NS);
  volatile int* misc = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
  volatile int* abort = misc + 1;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int qt = blockIdx.x, h = blockIdx.y;

  if (tid == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(s_full(w), 1);
      mbar_init(s_free(w), 128);
      mbar_init(p_full(w), 128);
      mbar_init(pv_done(w), 1);
    }
    mbar_init(drain_qk, 1);
    mbar_init(drain_pv, 1);
    fence_barrier_init();
    misc[1] = 0;
    // misc[2] super-blocks, misc[3..6] start / length of CSR rows a and b
    if constexpr (DENSE) {
      misc[2] = p.nkb;
      misc[3] = 0; misc[4] = p.nkb; misc[5] = 0; misc[6] = 0;
    } else {
      const int* rp = p.row_ptr + static_cast<size_t>(h) * (p.nqb + 1);
      int st[2] = {0, 0}, n[2] = {0, 0};
      for (int g = 0; g < p.G; ++g) {
        const int qb = qt * p.G + g;
        if (qb >= p.nqb) break;
        st[g] = rp[qb];
        n[g] = rp[qb + 1] - st[g];
        if (st[g] < 0 || n[g] < 0 || n[g] > p.nkb) {
          n[g] = 0;
          if (p.err) atomicCAS(p.err, 0, kErrBadCsr);
        }
      }
      // two query blocks: the union's length is set below, by all threads
      misc[2] = (n[0] + E - 1) / E;
      misc[3] = st[0]; misc[4] = n[0]; misc[5] = st[1]; misc[6] = n[1];
      misc[7] = 0;
      misc[8] = 0;   // 1: the merged list is in shared memory
      misc[10] = 0;  // malformed rows (bit 0: A, bit 1: B)
    }
  }
  if (warp == kDualKWarp) {
    tmem_alloc(smem_u32(const_cast<int*>(misc)), C::TMEM_COLS);
    tmem_relinquish();
    if (lane == 0) {
      tma_prefetch_map(&tmQ);
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
    }
  }
  __syncthreads();
  if constexpr (!DENSE) {
    if (misc[6] > 0) {
      // Merged list of two ascending CSR rows A and B.  Its length is
      // |A| + |B| - |A and B|, counted in parallel from bitmaps of A's and B's
      // key blocks in P_0 and P_1 (free until the first probabilities are
      // stored; each holds 262144 bits, the largest nKB).  A list of at most
      // kUnionCap entries is then written out in order, with membership bits,
      // so the softmax reads its entries instead of walking the two rows.
      // The same pass checks that each row is strictly ascending within
      // [0, nKB): the softmax and the producers would otherwise disagree on
      // the list, and one malformed row would spoil the other block's output.
      // A malformed row is skipped (and reported), like a bad start or length.
      static_assert(C::P_BYTES * 8 >= (1 << 24) / 64, "key-block bitmap");
      const int* a = p.col_idx + misc[3];
      const int* b = p.col_idx + misc[5];
      uint32_t* bma = reinterpret_cast<uint32_t*>(smem + C::OFF_P);
      uint32_t* bmb = reinterpret_cast<uint32_t*>(smem + C::OFF_P + C::P_BYTES);
      const int nw = (p.nkb + 31) >> 5;
      // bitmaps of rows A (na entries) and B (nb entries) and their common
      // entries (misc[7]); returns the malformed-row bits (misc[10])
      auto build_bitmaps = [&](int na, int nb) -> uint32_t {
        for (int i = tid; i < nw; i += kDualThreads) {
          bma[i] = 0u;
          bmb[i] = 0u;
        }
        __syncthreads();
        uint32_t bad = 0u;
        for (int i = tid; i < na; i += kDualThreads) {
          const int kb = __ldg(a + i);
          if (kb < 0 || kb >= p.nkb || (i + 1 < na && __ldg(a + i + 1) <= kb)) bad |= 1u;
          else atomicOr(bma + (kb >> 5), 1u << (kb & 31));
        }
        __syncthreads();
        int both = 0;
        for (int i = tid; i < nb; i += kDualThreads) {
          const int kb = __ldg(b + i);
          if (kb < 0 || kb >= p.nkb || (i + 1 < nb && __ldg(b + i + 1) <= kb)) {
            bad |= 2u;
          } else {
            both += static_cast<int>((bma[kb >> 5] >> (kb & 31)) & 1u);
            atomicOr(bmb + (kb >> 5), 1u << (kb & 31));
          }
        }
        both = __reduce_add_sync(0xffffffffu, both);
        bad = __reduce_or_sync(0xffffffffu, bad);
        if (lane == 0 && both > 0) atomicAdd(const_cast<int*>(misc + 7), both);
        if (lane == 0 && bad != 0u) atomicOr(const_cast<int*>(misc + 10), static_cast<int>(bad));
        __syncthreads();
        return static_cast<uint32_t>(misc[10]);
      };
      const uint32_t bad = build_bitmaps(misc[4], misc[6]);
      if (bad != 0u) {
        __syncthreads();  // every thread has read misc[10]
        if (tid == 0) {
          if (bad & 1u) misc[4] = 0;
          if (bad & 2u) misc[6] = 0;
          misc[2] = (misc[4] + E - 1) / E;  // the tile's one remaining row (or none)
          misc[7] = 0;
          misc[10] = 0;
          if (p.err) atomicCAS(p.err, 0, kErrBadCsr);
        }
        __syncthreads();
        // A skipped, B kept: B alone goes through the merged list (its
        // entries carry B's membership bit)
        if (misc[6] > 0) build_bitmaps(0, misc[6]);
      }
      if (misc[6] > 0) {
        const int ulen = misc[4] + misc[6] - misc[7];
        if (tid == 0) {
          misc[2] = (ulen + E - 1) / E;
          misc[9] = ulen;
        }
        if (ulen <= C::kUnionCap && warp == 0) {
          // warp 0 writes the set bits of A | B in ascending order, 32 words a round
          uint32_t* list = reinterpret_cast<uint32_t*>(smem + C::OFF_LIST);
          int run = 0;
          for (int base = 0; base < nw; base += 32) {
            const int wd = base + lane;
            const uint32_t wa = wd < nw ? bma[wd] : 0u, wb = wd < nw ? bmb[wd] : 0u;
            uint32_t word = wa | wb;
            const int cnt = __popc(word);
            int incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const int v = __shfl_up_sync(0xffffffffu, incl, o);
              if (lane >= o) incl += v;
            }
            int pos = run + incl - cnt;
            while (word) {
              const int bit = __ffs(word) - 1;
              word &= word - 1;
              const uint32_t mem = ((wa >> bit) & 1u) | (((wb >> bit) & 1u) << 1);
              if (pos < C::kUnionCap) list[pos] = static_cast<uint32_t>(wd * 32 + bit) | (mem << 30);
              ++pos;
            }
            run += __shfl_sync(0xffffffffu, incl, 31);
          }
          if (lane == 0) misc[8] = 1;
        }
        __syncthreads();
      }
    }
  }
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);
  const int nblk = misc[2];  // super-blocks
  // a walker over this CTA's key-block list (dense: 0 .. nkb-1)
  auto make_walker = [&]() {
    return ListWalker{p.col_idx + misc[3], p.col_idx + misc[5], misc[4], misc[6], 0, 0};
  };
  auto next_entry = [&](ListWalker& wk, int& dense_next, uint32_t& mem) -> int {
    if constexpr (DENSE) {
      mem = 1u;
      return dense_next < p.nkb ? dense_next++ : -1;
    } else {
      return wk.next(mem);
    }
  };

  if (warp >= 8) {
  // warpgroup 2 gives registers back (all four warps, same instruction)
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kDualRegsOther));
  if (warp == kDualKWarp) {
    // ===================================================== Q / K producer
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_q, C::Q_BYTES);
#pragma unroll
      for (int c = 0; c < C::QKCH; ++c)
        tma_load_3d(sQ + c * (BM * 128), &tmQ, c * C::QKX, qt * BM, h, bar_q);
      int issued = 0;
      ListWalker wk = make_walker();
      int dn = 0;
      for (int j = 0; j < nblk; ++j) {
        const int s = j % NS;
        if (!mbar_wait(k_empty(s), ((j / NS) & 1) ^ 1u, abort, p.err, kErrWaitKEmpty)) break;
        mbar_arrive_expect_tx(k_full(s), C::K_BYTES);
#pragma unroll
        for (int e = 0; e < E; ++e) {
          uint32_t mem;
          const int kb = next_entry(wk, dn, mem);
          const int row0 = kb >= 0 ? kb * BKS : p.N;  // past N: zeros
#pragma unroll
          for (int c = 0; c < C::QKCH; ++c)
            tma_load_3d(sK + s * C::K_BYTES + c * (BK * 128) + e * BKS * 128, &tmK, c * C::QKX,
                        row0, h, k_full(s));
        }
        issued = j + 1;
      }
      if (*abort) {
        drain_wait(bar_q, 0);
        for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j)
          drain_wait(k_full(j % NS), (j / NS) & 1);
      }
    }
  } else if (warp == kDualVWarp) {
    // ===================================================== V producer
    if (lane == 0) {
      int issued = 0;
      ListWalker wk = make_walker();
      int dn = 0;
      for (int j = 0; j < nblk; ++j) {
        const int s = j % NS;
        if (!mbar_wait(v_empty(s), ((j / NS) & 1) ^ 1u, abort, p.err, kErrWaitVEmpty)) break;
        mbar_arrive_expect_tx(v_full(s), C::KV_BYTES);
#pragma unroll
        for (int e = 0; e < E; ++e) {
          uint32_t mem;
          const int kb = next_entry(wk, dn, mem);
          const int row0 = kb >= 0 ? kb * BKS : p.N;
#pragma unroll
          for (int c = 0; c < C::KCH; ++c)
            tma_load_3d(sV + s * C::KV_BYTES + c * (BK * 128) + e * BKS * 128, &tmV, c * 64, row0,
                        h, v_full(s));
        }
        issued = j + 1;
      }
      if (*abort) {
        for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j)
          drain_wait(v_full(j % NS), (j / NS) & 1);
      }
    }
  } else if (warp == kDualQKWarp) {
    // ===================================================== QK issuer (block order)
    // QK_j needs K_j and the release of S_{j mod 2} by block j - 2's softmax.
    if (lane == 0) {
      constexpr uint32_t kIdescQK = FP8 ? idesc_e4m3_f32(BM, BK) : idesc_bf16_f32(BM, BK, 0, 0);
      bool ok = mbar_wait(bar_q, 0, abort, p.err, kErrWaitQ);
      for (int j = 0; ok && j < nblk; ++j) {
        const int s = j % NS, w = j & 1, i = j >> 1;
        ok = mbar_wait(k_full(s), (j / NS) & 1, abort, p.err, kErrWaitKFull) &&
             mbar_wait(s_free(w), (i & 1) ^ 1u, abort, p.err, kErrWaitSFree);
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = tmem + w * BK;
        // K-steps of 32 bytes (16 bf16 or 32 E4M3 elements) along the rows
#pragma unroll
        for (int k = 0; k < C::KSTEPS; ++k) {
          const uint64_t a = smem_desc_sw128(sQ + (k >> 2) * (BM * 128) + (k & 3) * 32, 16, 1024);
          const uint64_t bd =
              smem_desc_sw128(sK + s * C::K_BYTES + (k >> 2) * (BK * 128) + (k & 3) * 32, 16, 1024);
          if constexpr (FP8) {
            mma_f8_ss(tS, a, bd, kIdescQK, k > 0 ? 1u : 0u);
          } else {
            mma_bf16_ss(tS, a, bd, kIdescQK, k > 0 ? 1u : 0u);
          }
        }
        mma_commit(k_empty(s));
        mma_commit(s_full(w));
      }
      if (!ok) {
        mma_commit(drain_qk);
        drain_wait(drain_qk, 0);
      }
    }
  } else if (warp == kDualPVWarp) {
    // ===================================================== PV issuer (block order)
    // PV_j needs P_j from warpgroup j mod 2 and V_j.
    if (lane == 0) {
      constexpr uint32_t kIdescPV = idesc_bf16_f32(BM, D, 0, 1);
      bool ok = true;
      for (int j = 0; ok && j < nblk; ++j) {
        const int s = j % NS, w = j & 1, i = j >> 1;
        ok = mbar_wait(p_full(w), i & 1, abort, p.err, kErrWaitPFull) &&
             mbar_wait(v_full(s), (j / NS) & 1, abort, p.err, kErrWaitVFull);
        if (!ok) break;
        tc_fence_after();
        const uint32_t tO = tmem + 2 * BK + w * D;
        const uint32_t pw = sP + w * C::P_BYTES;
#pragma unroll
        for (int k = 0; k < BK / 16; ++k) {
          const uint64_t a = smem_desc_sw128(pw + (k >> 2) * (BM * 128) + (k & 3) * 32, 16, 1024);
          const uint64_t b = smem_desc_sw128(sV + s * C::KV_BYTES + k * 16 * 128, BK * 128, 1024);
          mma_bf16_ss(tO, a, b, kIdescPV, (i > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(v_empty(s));
        mma_commit(pv_done(w));
      }
      if (!ok) {
        mma_commit(drain_pv);
        drain_wait(drain_pv, 0);
      }
    }
  }
  } else {
    // ===================================================== softmax warpgroups (warps 0..7)
    // take the registers warpgroup 2 gave back (waits until it has)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kDualRegsSoftmax));
    const int w = warp >> 2;                  // warpgroup 0 or 1
    const int row = tid & 127;                // query row = TMEM lane
    const uint32_t tl = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + tl + w * BK;
    const uint32_t tO = tmem + tl + 2 * BK + w * D;
    const uint32_t pw = sP + w * C::P_BYTES;
    const int qpos = qt * BM + row;
    const bool valid_row = qpos < p.N;
    const int nmine = (nblk + 1 - w) >> 1;    // blocks of this warpgroup
    float m_ref = -INFINITY, Z = 0.f, A = 0.f;
    bool ok = true;
    float sv[BK];
    // P_w row `row`: 128-byte swizzled K-major rows, two 64-key halves of
    // 128 rows each; chunk c8 (8 keys, 16 bytes) lands at prow + poff[c8]
    const uint32_t prow = pw + row * 128;
    uint32_t poff[BK / 8];
#pragma unroll
    for (int c8 = 0; c8 < BK / 8; ++c8) poff[c8] = (c8 >> 3) * (BM * 128) + (((c8 & 7) ^ (row & 7)) << 4);
    // this thread's walk of the key-block list, and its query block within
    // the CTA (rows 64g .. 64g+63 when two 64-row query blocks share it)
    ListWalker wk = make_walker();
    int dn = 0, sb_done = 0;
    const uint32_t my_bit = SINGLE ? 1u : (1u << (row >> 6));
    // One query block per CTA and one list entry per super-block (128-row
    // query blocks, 128-key blocks, and the dense pass): every row keeps every
    // entry, so entry j is simply the j-th list element (one load, no walk)
    constexpr bool kDirect = (E == 1) && (DENSE || SINGLE);
    const int* my_list = p.col_idx + misc[3];
    // Otherwise entry j * E + e comes from: the tile's one CSR row (read
    // directly, entries of query block A), or the merged list in shared
    // memory, or, when that list would not fit, a walk of the two rows.
    const bool one_row = SINGLE || misc[6] == 0;
    const int n_row = misc[4];
    const bool use_list = !one_row && misc[8] != 0;
    const int ulen = misc[9];
    const uint32_t* s_list = reinterpret_cast<const uint32_t*>(smem + C::OFF_LIST);
    // FP8 scores carry the query block's and the key block's scale
    float q_sl2 = p.scale_log2;
    if constexpr (FP8) q_sl2 *= __ldg(p.q_scales + static_cast<size_t>(h) * p.nqb + qt);
    for (int i = 0; i < nmine; ++i) {
      const int j = 2 * i + w;
      // valid keys of each entry of super-block j for this row
      int nv[E];
      float sl2 = q_sl2;
      if constexpr (kDirect) {
        const int kb = DENSE ? j : __ldg(my_list + j);
        const bool kb_ok = kb >= 0 && kb < p.nkb;
        nv[0] = kb_ok ? min(BKS, p.N - kb * BKS) : 0;
        if constexpr (FP8) {
          if (kb_ok) sl2 *= __ldg(p.k_scales + static_cast<size_t>(h) * p.nkb + kb);
        }
      } else if (one_row) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int idx = j * E + e;
          const int kb = idx < n_row ? __ldg(my_list + idx) : -1;
          const bool keep = kb >= 0 && kb < p.nkb && (my_bit & 1u) != 0u;
          nv[e] = keep ? min(BKS, p.N - kb * BKS) : 0;
        }
      } else if (use_list) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int idx = j * E + e;
          const uint32_t ent = idx < ulen ? s_list[idx] : 0xFFFFFFFFu;
          const int kb = ent == 0xFFFFFFFFu ? -1 : static_cast<int>(ent & 0x3FFFFFFFu);
          const bool keep = kb >= 0 && kb < p.nkb && ((ent >> 30) & my_bit) != 0u;
          nv[e] = keep ? min(BKS, p.N - kb * BKS) : 0;
        }
      } else {
        // walk the merged list, skipping the other warpgroup's super-blocks
        for (; sb_done < j; ++sb_done) {
#pragma unroll
          for (int e = 0; e < E; ++e) {
            uint32_t mem;
            next_entry(wk, dn, mem);
          }
        }
#pragma unroll
        for (int e = 0; e < E; ++e) {
          uint32_t mem;
          const int kb = next_entry(wk, dn, mem);
          const bool keep = kb >= 0 && kb < p.nkb && (mem & my_bit) != 0u;
          nv[e] = keep ? min(BKS, p.N - kb * BKS) : 0;
        }
        ++sb_done;
      }
      ok = mbar_wait(s_full(w), i & 1, abort, p.err, kErrWaitSFull);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < BK / 32; ++c) tmem_ld32f(tS + c * 32, sv + c * 32);
      tmem_wait_ld();
      freg_fence<BK>(sv);
      tc_fence_before();
      mbar_arrive(s_free(w));   // S_w may now receive this warpgroup's next QK

      // key c of the super-block is valid for this row iff c - BKS*e < nv[e]
      bool all_valid = true, any_valid = false;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        all_valid = all_valid && nv[e] >= BKS;
        any_valid = any_valid || nv[e] > 0;
      }
      float alpha = 1.f;
      bool o_rescale = false;
      auto update_max = [&](float bmax) {
        const float m_new = fmaxf(m_ref, bmax);
        if (m_new > m_ref + kRescaleLog2) {
          if (m_ref != -INFINITY) {
            alpha = ex2_approx(m_ref - m_new);
            A = alpha * (A + (m_ref - m_new) * Z);
            Z *= alpha;
            o_rescale = i > 0;
          }
          m_ref = m_new;
        }
      };
      // Three cases, warp-uniform: every key of the block valid for the whole
      // warp (fast path), none valid (P = 0), or a partly valid tail block.
      // (with one query block per tile every row has the same valid keys)
      const int mode = kDirect ? (all_valid ? 0 : (any_valid ? 2 : 1))
                       : (__all_sync(0xffffffffu, all_valid)
                              ? 0
                              : (__all_sync(0xffffffffu, !any_valid) ? 1 : 2));
      auto wait_prev_pv = [&]() -> bool {
        // P_w and O_w are free once this warpgroup's previous PV has completed
        if (i > 0) {
          const bool done = mbar_wait(pv_done(w), (i - 1) & 1, abort, p.err, kErrWaitPVDone);
          if (!__all_sync(0xffffffffu, done)) return false;
        }
        tc_fence_after();
        return true;
      };
      auto rescale_o = [&]() {
        if (__any_sync(0xffffffffu, o_rescale)) {
          const float a = o_rescale ? alpha : 1.f;
#pragma unroll
          for (int c = 0; c < D; c += 16) {
            float o[16];
            tmem_ld16f(tO + c, o);
            tmem_wait_ld();
            freg_fence<16>(o);
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] *= a;
            tmem_st16f(tO + c, o);
          }
          tmem_wait_st();
        }
      };
      if (mode == 1) {
        // no key of this block is valid: P = 0, statistics unchanged
        if (!wait_prev_pv()) { ok = false; break; }
#pragma unroll
        for (int c8 = 0; c8 < BK / 8; ++c8) st_shared_v4(prow + poff[c8], 0u, 0u, 0u, 0u);
      } else {
        // Two 64-key entries: each half of the super-block is kept whole or
        // not at all by this warp's query block, except in the sequence's last
        // key block.  Whole halves need no per-key mask: an unkept half is left
        // out of the max and gets offset -inf below (x = -inf, p = 0).
        bool halves = false;
        bool keep_half[E];
#pragma unroll
        for (int e = 0; e < E; ++e) keep_half[e] = true;
        if constexpr (E == 2) {
          halves = (nv[0] == 0 || nv[0] == BKS) && (nv[1] == 0 || nv[1] == BKS);
          if (halves) {
            keep_half[0] = nv[0] > 0;
            keep_half[1] = nv[1] > 0;
          }
        }
        if (mode == 2 && !halves) {
          // partly valid: invalid keys (past N, or not kept by this row's
          // query block) get a huge negative score, so p = 0 and p * x = 0
          // without special cases; a row with no valid key leaves its
          // statistics alone (below)
#pragma unroll
          for (int c = 0; c < BK; ++c) sv[c] = (c % BKS) < nv[c / BKS] ? sv[c] : -1e30f;
        }
        {
          // row max: 16 independent chains of 3-input max, then a small tree
          // (per 64-key half with two entries)
          float bmax;
          if constexpr (E == 2) {
            float hm[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              float mx[16];
#pragma unroll
              for (int q = 0; q < 16; ++q) {
                mx[q] = fmax3(sv[64 * e + q], sv[64 * e + 16 + q], sv[64 * e + 32 + q]);
                mx[q] = fmaxf(mx[q], sv[64 * e + 48 + q]);
              }
#pragma unroll
              for (int q = 0; q < 5; ++q) mx[q] = fmax3(mx[3 * q], mx[3 * q + 1], mx[3 * q + 2]);
              hm[e] = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[15]));
              if (!keep_half[e]) hm[e] = -INFINITY;
            }
            bmax = fmaxf(hm[0], hm[1]);
          } else {
            float mx[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              mx[q] = fmax3(sv[q], sv[16 + q], sv[32 + q]);
              mx[q] = fmax3(mx[q], sv[48 + q], sv[64 + q]);
              mx[q] = fmax3(mx[q], sv[80 + q], sv[96 + q]);
              mx[q] = fmaxf(mx[q], sv[112 + q]);
            }
#pragma unroll
            for (int q = 0; q < 5; ++q) mx[q] = fmax3(mx[3 * q], mx[3 * q + 1], mx[3 * q + 2]);
            bmax = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[15]));
          }
          if (any_valid) update_max(bmax * sl2);
        }
        // x = s * scale * log2(e) - m_ref, p = 2^x, Z += p, A += p * x, two
        // lanes per instruction (m_ref is -inf only for a row with no valid
        // key yet, whose p are then all 0); an unkept half's offset is -inf
        const float2 sc2 = make_float2(sl2, sl2);
        const float mc = (m_ref == -INFINITY) ? 0.f : m_ref;
        float2 nmh[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const float o = keep_half[e] ? -mc : -INFINITY;
          nmh[e] = make_float2(o, o);
        }
        float2 z2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        float2 a2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        auto pair = [&](int c) -> uint32_t {
          const float2 x = __ffma2_rn(make_float2(sv[2 * c], sv[2 * c + 1]), sc2, nmh[(2 * c) / BKS]);
          const float2 pr = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          z2[c & 1] = __fadd2_rn(z2[c & 1], pr);
          if constexpr (DENSE) a2[c & 1] = __ffma2_rn(pr, x, a2[c & 1]);
          return pack_bf16(pr.x, pr.y);
        };
        // the first half of the keys into registers while this warpgroup's
        // previous PV (which reads P_w) finishes on the tensor cores
        // (with two 64-key entries the halves are the entries: an unkept one
        // takes no exponentials, its P is stored as zeros)
        bool skip_first = false, skip_rest = false;
        if constexpr (E == 2) {
          skip_first = !keep_half[0];
          skip_rest = !keep_half[1];
        }
        uint32_t first[BK / 4];
        if (skip_first) {
#pragma unroll
          for (int c = 0; c < BK / 4; ++c) first[c] = 0u;
        } else {
#pragma unroll
          for (int c = 0; c < BK / 4; ++c) first[c] = pair(c);
        }
        if (!wait_prev_pv()) { ok = false; break; }
        rescale_o();
#pragma unroll
        for (int c8 = 0; c8 < BK / 16; ++c8)
          st_shared_v4(prow + poff[c8], first[4 * c8], first[4 * c8 + 1], first[4 * c8 + 2],
                       first[4 * c8 + 3]);
        // the rest: computed and stored 8 keys at a time
        if (skip_rest) {
#pragma unroll
          for (int c8 = BK / 16; c8 < BK / 8; ++c8) st_shared_v4(prow + poff[c8], 0u, 0u, 0u, 0u);
        } else {
#pragma unroll
          for (int c8 = BK / 16; c8 < BK / 8; ++c8) {
            const uint32_t a = pair(4 * c8), b = pair(4 * c8 + 1);
            const uint32_t c = pair(4 * c8 + 2), d = pair(4 * c8 + 3);
            st_shared_v4(prow + poff[c8], a, b, c, d);
          }
        }
        const float2 zz = __fadd2_rn(z2[0], z2[1]);
        Z += zz.x + zz.y;
        if constexpr (DENSE) {
          const float2 aa = __fadd2_rn(a2[0], a2[1]);
          A += aa.x + aa.y;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full(w));
    }
    // ---- merge the two warpgroups' partial results
    if (ok && nmine > 0) {
      ok = mbar_wait(pv_done(w), (nmine - 1) & 1, abort, p.err, kErrWaitPVDone);
      ok = __all_sync(0xffffffffu, ok);
    }
    float* st = reinterpret_cast<float*>(smem + C::OFF_P + w * C::P_BYTES);  // P_w is free now
    st[row] = m_ref;
    st[128 + row] = Z;
    st[256 + row] = A;
    tc_fence_before();
    named_barrier_sync(1, 256);
    tc_fence_after();
    const float* so = reinterpret_cast<const float*>(smem + C::OFF_P + (1 - w) * C::P_BYTES);
    const float m_o = so[row], Z_o = so[128 + row], A_o = so[256 + row];
    const float m0 = w == 0 ? m_ref : m_o, m1 = w == 0 ? m_o : m_ref;
    const float Z0 = w == 0 ? Z : Z_o, Z1 = w == 0 ? Z_o : Z;
    const float A0 = w == 0 ? A : A_o, A1 = w == 0 ? A_o : A;
    const float m = fmaxf(m0, m1);
    const float a0 = (m0 == -INFINITY) ? 0.f : ex2_approx(m0 - m);
    const float a1 = (m1 == -INFINITY) ? 0.f : ex2_approx(m1 - m);
    const float Zt = a0 * Z0 + a1 * Z1;
    float At = 0.f;
    if (a0 > 0.f) At += a0 * (A0 + (m0 - m) * Z0);
    if (a1 > 0.f) At += a1 * (A1 + (m1 - m) * Z1);
    const float inv = Zt > 0.f ? 1.f / Zt : 0.f;
    const int n0 = (nblk + 1) >> 1, n1 = nblk >> 1;
    const bool use0 = ok && n0 > 0, use1 = ok && n1 > 0;
    const float c0 = use0 ? a0 * inv : 0.f, c1 = use1 ? a1 * inv : 0.f;
    __nv_bfloat16* orow = p.O + (static_cast<size_t>(h) * p.N + (valid_row ? qpos : 0)) * D;
    // warpgroup w writes output columns [w * D/2, (w + 1) * D/2): all of its
    // TMEM loads are issued before one wait
    constexpr int kOutChunks = D / 32;  // 16-column chunks per warpgroup
    float o0[kOutChunks][16], o1[kOutChunks][16];
#pragma unroll
    for (int k = 0; k < kOutChunks; ++k) {
      const int c = w * (D / 2) + 16 * k;
      if (use0) tmem_ld16f(tmem + tl + 2 * BK + c, o0[k]);
      if (use1) tmem_ld16f(tmem + tl + 2 * BK + D + c, o1[k]);
    }
    tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < kOutChunks; ++k) {
      const int c = w * (D / 2) + 16 * k;
      if (use0) freg_fence<16>(o0[k]);
      if (use1) freg_fence<16>(o1[k]);
      float* o = o0[k];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float x0 = use0 ? o0[k][e] * c0 : 0.f;
        const float x1 = use1 ? o1[k][e] * c1 : 0.f;
        o[e] = x0 + x1;
      }
      if (valid_row) {
        uint4 w0, w1;
        w0.x = pack_bf16(o[0], o[1]);
        w0.y = pack_bf16(o[2], o[3]);
        w0.z = pack_bf16(o[4], o[5]);
        w0.w = pack_bf16(o[6], o[7]);
        w1.x = pack_bf16(o[8], o[9]);
        w1.y = pack_bf16(o[10], o[11]);
        w1.z = pack_bf16(o[12], o[13]);
        w1.w = pack_bf16(o[14], o[15]);
        reinterpret_cast<uint4*>(orow + c)[0] = w0;
        reinterpret_cast<uint4*>(orow + c)[1] = w1;
      }
    }
    if (w == 0 && valid_row) {
      const size_t idx = static_cast<size_t>(h) * p.N + qpos;
      if (DENSE && p.H != nullptr) p.H[idx] = Zt > 0.f ? logf(Zt) - kLn2 * (At / Zt) : NAN;
      if (p.lse != nullptr) p.lse[idx] = Zt > 0.f ? kLn2 * (m + log2f(Zt)) : -INFINITY;
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == kDualKWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Entropy-only pass: H and LSE of every query over all N keys, without the
// PV product or the output (an entropy refresh that needs no dense output).
//
// With no output accumulator the 512 TMEM columns hold four score tiles, one
// per softmax warpgroup: warpgroup w takes key blocks j = w, w + 4, ... and
// reads its tile in two halves of 64 scores, so that four warpgroups fit the
// register file (setmaxnreg: 104 per softmax thread, 64 for the producer /
// MMA warpgroup) and each scheduler has four softmax warps to issue from.  K
// has a 4-stage ring.  Per score the softmax does one packed FMA
// (x = s * scale * log2 e - m), one ex2 and half of a packed add (Z) and of a
// packed FMA (A): the MUFU unit bounds it, the tensor cores run at half their
// dense-pass load.  The four warpgroups' (m, Z, A) are merged exactly at the
// end.  Warps: 0..15 softmax, 16 Q/K producer (and tensor-memory allocation),
// 17 MMA, 18 and 19 idle (they complete the fifth warpgroup).
// ---------------------------------------------------------------------------

constexpr int kEntThreads = 640;  // 20 warps
constexpr int kEntWarpgroups = 4; // softmax warpgroups (warps 0..15)
constexpr int kEntKWarp = 16;
constexpr int kEntMmaWarp = 17;
// Registers: launched at 96 per thread (640 x 96 = 61440); the softmax
// warpgroups take 104, the producer / MMA warpgroup gives back to 64:
// 4 x 128 x 104 + 128 x 64 = 61440.
constexpr int kEntRegsLaunch = 96;
constexpr int kEntRegsSoftmax = 104;
constexpr int kEntRegsOther = 64;
static_assert(kEntWarpgroups * 128 * kEntRegsSoftmax + 128 * kEntRegsOther ==
                  kEntThreads * kEntRegsLaunch, "register split");

template <int D>
struct EntCfg {
  static constexpr int BK = 128;
  static constexpr int NS = 4;
  static constexpr int KCH = D / 64;
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BK * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_ST = OFF_K + NS * KV_BYTES;  // merge statistics, 4 x 3 x 128 fp32
  static constexpr int OFF_BAR = OFF_ST + kEntWarpgroups * 3 * BM * 4;
  static constexpr int NUM_BARS = 1 + 2 * NS + 8 + 1;
  static constexpr int OFF_MISC = OFF_BAR + 256;
  static constexpr int USED = OFF_MISC + 64;
  static constexpr int SMEM = (USED < 120 * 1024 ? 120 * 1024 : USED) + 1024;
  static constexpr int TMEM_COLS = 512;  // one 128-column score tile per warpgroup
  static_assert(kEntWarpgroups * BK <= TMEM_COLS, "tensor memory");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(NUM_BARS * 8 <= 256, "barrier area");
};

template <int D>
__global__ void __launch_bounds__(kEntThreads, 1)
    entropy_kernel(const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmK, const Params p) {
  using C = EntCfg<D>;
  constexpr int NS = C::NS;
  constexpr int BK = C::BK;
  constexpr int WG = kEntWarpgroups;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sK = sbase + C::OFF_K;
  const uint32_t bars = sbase + C::OFF_BAR;
  const uint32_t bar_q = bars;
  auto k_full = [&](int s) { return bars + 8u * (1 + s); };
  auto k_empty = [&](int s) { return bars + 8u * (1 + NS + s); };
  auto s_full = [&](int w) { return bars + 8u * (1 + 2 * NS + w); };
  auto s_free = [&](int w) { return bars + 8u * (5 + 2 * NS + w); };
  const uint32_t drain_bar = bars + 8u * (9 + 2 * NS);
  volatile int* misc = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
  volatile int* abort = misc + 1;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int qt = blockIdx.x, h = blockIdx.y;
  const int nblk = p.nkb;

  if (tid == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
    }
    for (int w = 0; w < WG; ++w) {
      mbar_init(s_full(w), 1);
      mbar_init(s_free(w), 128);
    }
    mbar_init(drain_bar, 1);
    fence_barrier_init();
    misc[1] = 0;
  }
  if (warp == kEntKWarp) {
    tmem_alloc(smem_u32(const_cast<int*>(misc)), C::TMEM_COLS);
    tmem_relinquish();
    if (lane == 0) {
      tma_prefetch_map(&tmQ);
      tma_prefetch_map(&tmK);
    }
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(misc[0]);

  if (warp >= 4 * WG) {
  // the producer / MMA warpgroup gives registers back (all four warps)
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kEntRegsOther));
  if (warp == kEntKWarp) {
    // ===================================================== Q / K producer
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_q, C::Q_BYTES);
#pragma unroll
      for (int c = 0; c < C::KCH; ++c) tma_load_3d(sQ + c * (BM * 128), &tmQ, c * 64, qt * BM, h, bar_q);
      int issued = 0;
      for (int j = 0; j < nblk; ++j) {
        const int s = j % NS;
        if (!mbar_wait(k_empty(s), ((j / NS) & 1) ^ 1u, abort, p.err, kErrWaitKEmpty)) break;
        mbar_arrive_expect_tx(k_full(s), C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < C::KCH; ++c)
          tma_load_3d(sK + s * C::KV_BYTES + c * (BK * 128), &tmK, c * 64, j * BK, h, k_full(s));
        issued = j + 1;
      }
      if (*abort) {
        drain_wait(bar_q, 0);
        for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j)
          drain_wait(k_full(j % NS), (j / NS) & 1);
      }
    }
  } else if (warp == kEntMmaWarp) {
    // ===================================================== MMA issuer (QK only, in block order)
    // block j goes to warpgroup j mod 4 and its score tile S_{j mod 4}
    if (lane == 0) {
      constexpr uint32_t kIdescQK = idesc_bf16_f32(BM, BK, 0, 0);
      bool ok = mbar_wait(bar_q, 0, abort, p.err, kErrWaitQ);
      for (int j = 0; ok && j < nblk; ++j) {
        const int s = j % NS, w = j % WG, u = j / WG;
        ok = mbar_wait(k_full(s), (j / NS) & 1, abort, p.err, kErrWaitKFull) &&
             mbar_wait(s_free(w), (u & 1) ^ 1u, abort, p.err, kErrWaitSFree);
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = tmem + w * BK;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t a = smem_desc_sw128(sQ + (k >> 2) * (BM * 128) + (k & 3) * 32, 16, 1024);
          const uint64_t bd =
              smem_desc_sw128(sK + s * C::KV_BYTES + (k >> 2) * (BK * 128) + (k & 3) * 32, 16, 1024);
          mma_bf16_ss(tS, a, bd, kIdescQK, k > 0 ? 1u : 0u);
        }
        mma_commit(k_empty(s));
        mma_commit(s_full(w));
      }
      if (!ok) {
        mma_commit(drain_bar);
        drain_wait(drain_bar, 0);
      }
    }
  }
  } else {
    // ===================================================== softmax statistics (warps 0..15)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kEntRegsSoftmax));
    const int w = warp >> 2;
    const int row = tid & 127;
    const uint32_t tl = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + tl + w * BK;
    const int qpos = qt * BM + row;
    const int nmine = nblk > w ? (nblk - 1 - w) / WG + 1 : 0;
    float m_ref = -INFINITY, Z = 0.f, A = 0.f;
    bool ok = true;
    for (int i = 0; i < nmine; ++i) {
      const int j = WG * i + w;
      ok = mbar_wait(s_full(w), i & 1, abort, p.err, kErrWaitSFull);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int nvalid = min(BK, p.N - j * BK);  // keys past N (zero rows) are excluded
      // the score row in two halves of 64 (registers for four warpgroups);
      // S_w is released once both halves are in registers
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float sv[BK / 2];
        tmem_ld32f(tS + hh * (BK / 2), sv);
        tmem_ld32f(tS + hh * (BK / 2) + 32, sv + 32);
        tmem_wait_ld();
        freg_fence<BK / 2>(sv);
        if (hh == 1) {
          tc_fence_before();
          mbar_arrive(s_free(w));
        }
        if (nvalid < BK) {
#pragma unroll
          for (int c = 0; c < BK / 2; ++c) sv[c] = hh * (BK / 2) + c < nvalid ? sv[c] : -1e30f;
        }
        {
          float mx[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            mx[q] = fmax3(sv[q], sv[16 + q], sv[32 + q]);
            mx[q] = fmaxf(mx[q], sv[48 + q]);
          }
#pragma unroll
          for (int q = 0; q < 5; ++q) mx[q] = fmax3(mx[3 * q], mx[3 * q + 1], mx[3 * q + 2]);
          const float bmax = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[15])) *
                             p.scale_log2;
          const float m_new = fmaxf(m_ref, bmax);
          if (m_new > m_ref + kRescaleLog2) {
            if (m_ref != -INFINITY) {
              const float alpha = ex2_approx(m_ref - m_new);
              A = alpha * (A + (m_ref - m_new) * Z);
              Z *= alpha;
            }
            m_ref = m_new;
          }
        }
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 nm2 = make_float2(-m_ref, -m_ref);
        float2 z2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        float2 a2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < BK / 4; ++c) {
          const float2 x = __ffma2_rn(make_float2(sv[2 * c], sv[2 * c + 1]), sc2, nm2);
          const float2 pr = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          z2[c & 1] = __fadd2_rn(z2[c & 1], pr);
          a2[c & 1] = __ffma2_rn(pr, x, a2[c & 1]);
        }
        const float2 zz = __fadd2_rn(z2[0], z2[1]);
        const float2 aa = __fadd2_rn(a2[0], a2[1]);
        Z += zz.x + zz.y;
        A += aa.x + aa.y;
      }
    }
    // ---- merge the four warpgroups' statistics; warpgroup 0 writes H and LSE
    float* st = reinterpret_cast<float*>(smem + C::OFF_ST);
    st[(w * 3 + 0) * BM + row] = ok ? m_ref : -INFINITY;
    st[(w * 3 + 1) * BM + row] = ok ? Z : 0.f;
    st[(w * 3 + 2) * BM + row] = ok ? A : 0.f;
    named_barrier_sync(1, WG * 128);
    if (w == 0 && qpos < p.N) {
      float mw[WG], Zw[WG], Aw[WG];
      float m = -INFINITY;
#pragma unroll
      for (int g = 0; g < WG; ++g) {
        mw[g] = st[(g * 3 + 0) * BM + row];
        Zw[g] = st[(g * 3 + 1) * BM + row];
        Aw[g] = st[(g * 3 + 2) * BM + row];
        m = fmaxf(m, mw[g]);
      }
      float Zt = 0.f, At = 0.f;
#pragma unroll
      for (int g = 0; g < WG; ++g) {
        const float ag = (mw[g] == -INFINITY) ? 0.f : ex2_approx(mw[g] - m);
        if (ag > 0.f) {
          Zt += ag * Zw[g];
          At += ag * (Aw[g] + (mw[g] - m) * Zw[g]);
        }
      }
      const size_t idx = static_cast<size_t>(h) * p.N + qpos;
      p.H[idx] = Zt > 0.f ? logf(Zt) - kLn2 * (At / Zt) : NAN;
      if (p.lse != nullptr) p.lse[idx] = Zt > 0.f ? kLn2 * (m + log2f(Zt)) : -INFINITY;
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == kEntKWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// [heads, N, d] as a 3D tensor (d, N, heads) of bf16 (esize 2) or E4M3 bytes
// (esize 1); boxes of (128 / esize) x rows x 1, i.e. 128-byte rows, 128-byte
// swizzle; rows past N read as zeros.
bool make_map(CUtensorMap* map, const void* base, int d, int N, int heads, int rows,
              int esize = 2) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(heads)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * esize,
                                 static_cast<cuuint64_t>(N) * d * esize};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / esize), static_cast<cuuint32_t>(rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                        3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int BKS, bool DENSE, bool FP8 = false, bool SINGLE = true>
cudaError_t launch_dual(const AttnArgs& a, const Params& prm, cudaStream_t stream) {
  using C = DualCfg<D, FP8>;
  auto kern = attn_dual_kernel<D, BKS, DENSE, FP8, SINGLE>;
  // The kernel's register split assumes exactly kDualLaunchRegs per thread at
  // launch; with any other allocation setmaxnreg.inc could wait forever.
  static const int launch_regs = [kern] {
    cudaFuncAttributes fa{};
    return cudaFuncGetAttributes(&fa, kern) == cudaSuccess ? fa.numRegs : -1;
  }();
  if (launch_regs != kDualLaunchRegs) return cudaErrorInvalidDeviceFunction;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.Q, D, a.N, a.heads, BM, C::QE) ||
      !make_map(&mk, a.K, D, a.N, a.heads, BKS, C::QE) ||
      !make_map(&mv, a.V, D, a.N, a.heads, BKS))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const dim3 grid((a.N + BM - 1) / BM, a.heads);
  kern<<<grid, kDualThreads, C::SMEM, stream>>>(mq, mk, mv, prm);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_entropy(const AttnArgs& a, const Params& prm, cudaStream_t stream) {
  using C = EntCfg<D>;
  CUtensorMap mq, mk;
  if (!make_map(&mq, a.Q, D, a.N, a.heads, BM) || !make_map(&mk, a.K, D, a.N, a.heads, 128))
    return cudaErrorInvalidValue;
  auto kern = entropy_kernel<D>;
  // the setmaxnreg split assumes the launch allocation: refuse any other
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, kern);
  if (e != cudaSuccess) return e;
  if (attr.numRegs != kEntRegsLaunch) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const dim3 grid((a.N + BM - 1) / BM, a.heads);
  kern<<<grid, kEntThreads, C::SMEM, stream>>>(mq, mk, prm);
  return cudaGetLastError();
}

template <int D, int BK, bool DENSE>
cudaError_t launch_cfg(const AttnArgs& a, const Params& prm, cudaStream_t stream) {
  using C = Cfg<D, BK>;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.Q, D, a.N, a.heads, BM) || !make_map(&mk, a.K, D, a.N, a.heads, BK) ||
      !make_map(&mv, a.V, D, a.N, a.heads, BK))
    return cudaErrorInvalidValue;
  auto kern = attn_kernel<D, BK, DENSE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const dim3 grid((a.N + BM - 1) / BM, a.heads);
  kern<<<grid, kThreads, C::SMEM, stream>>>(mq, mk, mv, prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t stream) {
  Params prm;
  prm.N = a.N;
  const int bk = a.dense ? 128 : a.block_k;
  const int bq = a.dense ? 128 : a.block_q;
  prm.nqb = (a.N + bq - 1) / bq;
  prm.nkb = (a.N + bk - 1) / bk;
  prm.bq = bq;
  prm.G = BM / bq;
  prm.scale_log2 = a.scale * kLog2e;
  prm.row_ptr = a.row_ptr;
  prm.col_idx = a.col_idx;
  prm.q_scales = a.q_scales;
  prm.k_scales = a.k_scales;
  prm.O = static_cast<__nv_bfloat16*>(a.O);
  prm.H = a.H;
  prm.lse = a.lse;
  prm.err = device_error_word();
  // Query and key blocks of 64 or 128 tokens (and the dense pass) use the
  // two-warpgroup kernel; 16-token blocks use the single-warpgroup kernel,
  // which merges the lists of up to eight query blocks per CTA.
  if (a.entropy_only) return a.d == 128 ? launch_entropy<128>(a, prm, stream)
                                          : launch_entropy<64>(a, prm, stream);
  // E4M3 Q and K: 128-row query blocks, 128-key blocks, d = 128 (checked by the API)
  if (a.fp8) return launch_dual<128, 128, false, true>(a, prm, stream);
  if (a.dense) {
    if (a.d == 128) return launch_dual<128, 128, true>(a, prm, stream);
    return launch_dual<64, 128, true>(a, prm, stream);
  }
  if ((bq == 128 || bq == 64) && (bk == 128 || bk == 64)) {
    // SINGLE: one query block per 128-row tile
    if (bq == 128) {
      if (a.d == 128)
        return bk == 128 ? launch_dual<128, 128, false, false, true>(a, prm, stream)
                         : launch_dual<128, 64, false, false, true>(a, prm, stream);
      return bk == 128 ? launch_dual<64, 128, false, false, true>(a, prm, stream)
                       : launch_dual<64, 64, false, false, true>(a, prm, stream);
    }
    if (a.d == 128)
      return bk == 128 ? launch_dual<128, 128, false, false, false>(a, prm, stream)
                       : launch_dual<128, 64, false, false, false>(a, prm, stream);
    return bk == 128 ? launch_dual<64, 128, false, false, false>(a, prm, stream)
                     : launch_dual<64, 64, false, false, false>(a, prm, stream);
  }
  if (a.d == 128) {
    if (bk == 128) return launch_cfg<128, 128, false>(a, prm, stream);
    if (bk == 64) return launch_cfg<128, 64, false>(a, prm, stream);
    return launch_cfg<128, 16, false>(a, prm, stream);
  }
  if (bk == 128) return launch_cfg<64, 128, false>(a, prm, stream);
  if (bk == 64) return launch_cfg<64, 64, false>(a, prm, stream);
  return launch_cfg<64, 16, false>(a, prm, stream);
}

}  // namespace tra
