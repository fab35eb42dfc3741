// Fused radius mask -> block-sparse CSR (Token Radius Attention summary, §2
// "TRA pipeline", efficient execution: distance computation, radius compare,
// block pruning and token voting fused into one kernel that emits a regular
// query-block x key-block mask).
//
// Token mask: key j is in query i's support when dx^2 + dy^2 <= R2 with
// R2 = fl32(fl32(r_i * phi[|t_j - t_i|])^2); non-finite radii keep every key.
// Distances are integers, so the compare is done exactly as
// dx^2 + dy^2 <= floor(R2) (R2 clamped to 2^30, above any grid distance).
//
// Four launches:
//  1. footprint: for every key block, the rows (t, y, [x_lo, x_hi]) its tokens
//     cover and per-frame bounding boxes.  A contiguous run of tile-major
//     positions covers, for each (t, y), one contiguous x interval; the kernel
//     verifies this per block and otherwise marks the block for token-by-token
//     testing.
//  2. votes: one CTA per (head, query block).  Each CTA bounds, for every key
//     frame, the union of its queries' disks by a box; a key block whose
//     per-frame boxes miss those boxes has no votes and is pruned (lanes over
//     key blocks).  A survivor is then rejected when no query's disk meets any
//     of its per-frame boxes.  With a vote threshold of 1 and the disk distance
//     the block's complete rectangles (runs of rows of one frame with the same
//     x interval, every lattice position a key) decide exactly: the nearest
//     point of such a rectangle to a query is one of its keys, so one
//     dx^2 + dy^2 test per (query, rectangle) answers.  Otherwise survivors are
//     counted exactly (lanes over queries): for a query and a key row the
//     number of keys inside the disk is the overlap of [x_lo, x_hi] with
//     [x_q - s, x_q + s], s = isqrt(floor(R2) - dy^2); with a vote threshold
//     of 1 an existence test replaces the count.  Above 1, complete
//     rectangles are counted in closed form where the disk misses a
//     rectangle (nothing) or holds all of it (its area), row by row only
//     where the circle cuts it.  Counting stops once the threshold is reached
//     (only "votes >= threshold" is needed).
//  3. scan: exclusive prefix sum of the per-row kept counts -> row_ptr, nnz.
//  4. compact: kept bits -> ascending col_idx.
//
// The 1D-distance variant (the ablation of the summary's §4 that replaces the
// radius mask by a 1D distance) runs the same four launches: the distance of
// two tokens of a frame is the difference of their raster indices
// n = y * W + x, a key is inside when (n_j - n_i)^2 <= R2, and each query
// keeps, per key frame, the index interval [n_i - s, n_i + s] with
// s = isqrt(floor(R2)); boxes and rows are compared as index intervals.
#include "check.cuh"
#include "tra_internal.h"

namespace tra {
namespace {

constexpr int kMaxSeg = 4;   // per-frame boxes kept per key block (more: no pruning)
constexpr int kMaxRect = 4;  // complete rectangles kept per key block (more: row tests)
constexpr int kVoteThreads = 128;
constexpr int kRsqCap = 1 << 30;
constexpr int kReachCap = 1 << 30;  // 1D reach cap: beyond any in-frame index distance (< 2^24)

struct MaskWs {
  uint2* rows;      // [nkb * Bk]: x = t << 16 | y, y = x_lo << 16 | x_hi
  int4* info;       // [nkb]: x = rows (-1: not row-contiguous), y = segments (-1: too many), z = tokens
  int4* segs;       // [nkb * kMaxSeg]: x = t, y = y_lo << 16 | y_hi, z = x_lo << 16 | x_hi
  int4* rects;      // [nkb * kMaxRect]: as segs, every position of the rectangle a key of the block
  uint32_t* bits;   // [heads * nqb * nkbw]
  int* counts;      // [heads * nqb]
  int* err;         // device error word (index checks of the checked build)
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct MaskDims {
  int N, nqb, nkb, nkbw;
};

__host__ __device__ inline MaskDims mask_dims(const TileLayout& L, int bq, int bk) {
  MaskDims m;
  m.N = L.F * L.H * L.W;
  m.nqb = (m.N + bq - 1) / bq;
  m.nkb = (m.N + bk - 1) / bk;
  m.nkbw = (m.nkb + 31) / 32;
  return m;
}

size_t carve(const TileLayout& L, int heads, int bq, int bk, char* base, MaskWs* ws) {
  const MaskDims m = mask_dims(L, bq, bk);
  size_t off = 0;
  const size_t rows = align256(sizeof(uint2) * static_cast<size_t>(m.nkb) * bk);
  const size_t info = align256(sizeof(int4) * static_cast<size_t>(m.nkb));
  const size_t segs = align256(sizeof(int4) * static_cast<size_t>(m.nkb) * kMaxSeg);
  const size_t rects = align256(sizeof(int4) * static_cast<size_t>(m.nkb) * kMaxRect);
  const size_t bits = align256(sizeof(uint32_t) * static_cast<size_t>(heads) * m.nqb * m.nkbw);
  const size_t counts = align256(sizeof(int) * static_cast<size_t>(heads) * m.nqb);
  if (ws) {
    char* q = base + off;
    ws->rows = reinterpret_cast<uint2*>(q);
    ws->info = reinterpret_cast<int4*>(q += rows);
    ws->segs = reinterpret_cast<int4*>(q += info);
    ws->rects = reinterpret_cast<int4*>(q += segs);
    ws->bits = reinterpret_cast<uint32_t*>(q += rects);
    ws->counts = reinterpret_cast<int*>(q += bits);
  }
  return rows + info + segs + rects + bits + counts;
}

// floor(sqrt(m)) for 0 <= m <= 2^30: an estimate from the approximate
// reciprocal square root (within one of the answer for these m), corrected
// exactly with integer squares.
__device__ __forceinline__ int isqrt_floor(int m) {
  const float f = static_cast<float>(m);
  int s = m > 0 ? __float2int_rz(f * rsqrtf(f)) : 0;
  while (s * s > m) --s;
  while ((s + 1) * (s + 1) <= m) ++s;
  return s;
}

// floor(fl32(fl32(r * phi)^2)), clamped to 2^30 (also for +inf and NaN).
__device__ __forceinline__ int radius_sq(float r, float phi) {
  const float R = __fmul_rn(r, phi);
  const float R2 = __fmul_rn(R, R);
  if (!(R2 < 1073741824.0f)) return kRsqCap;
  return __float2int_rz(R2);
}

// floor(sqrt(floor(fl32(fl32(r * phi)^2)))): the largest integer index
// distance inside R, capped at 2^30 (also for +inf and NaN).
__device__ __forceinline__ int line_reach(float r, float phi) {
  const float R = __fmul_rn(r, phi);
  const float R2 = __fmul_rn(R, R);
  if (!(R2 < 1152921504606846976.0f)) return kReachCap;  // 2^60
  const unsigned long long m = __float2ull_rz(R2);
  unsigned long long sq = static_cast<unsigned long long>(sqrt(static_cast<double>(m)));
  while (sq * sq > m) --sq;
  while ((sq + 1) * (sq + 1) <= m) ++sq;
  return sq > static_cast<unsigned long long>(kReachCap) ? kReachCap : static_cast<int>(sq);
}

// ---------------------------------------------------------------- 1. footprint

__global__ void footprint_kernel(TileLayout L, int bk, MaskWs ws) {
  const int nkb = (L.F * L.H * L.W + bk - 1) / bk;
  const int kb = blockIdx.x * blockDim.x + threadIdx.x;
  if (kb >= nkb) return;
  const int N = L.F * L.H * L.W;
  const int p0 = kb * bk, p1 = min(N, p0 + bk);
  uint2* rows = ws.rows + static_cast<size_t>(kb) * bk;
  int4* segs = ws.segs + static_cast<size_t>(kb) * kMaxSeg;
  int nrows = 0, nseg = 0;
  int st[kMaxSeg], sylo[kMaxSeg], syhi[kMaxSeg], sxlo[kMaxSeg], sxhi[kMaxSeg];
  for (int p = p0; p < p1; ++p) {
    const Coord c = tile_major_coord(L, p);
    const uint32_t key = (static_cast<uint32_t>(c.t) << 16) | static_cast<uint32_t>(c.y);
    int f = -1;
    for (int i = nrows - 1; i >= 0; --i) {
      if (rows[i].x == key) { f = i; break; }
    }
    if (f < 0) {
      if (!in_bounds(nrows, bk, ws.err)) break;
      rows[nrows] = make_uint2(key, (static_cast<uint32_t>(c.x) << 16) | static_cast<uint32_t>(c.x));
      ++nrows;
    } else {
      const uint2 rw = rows[f];
      const int xlo = min(static_cast<int>(rw.y >> 16), c.x);
      const int xhi = max(static_cast<int>(rw.y & 0xFFFFu), c.x);
      rows[f].y = (static_cast<uint32_t>(xlo) << 16) | static_cast<uint32_t>(xhi);
    }
    if (nseg >= 0) {
      int s = -1;
      for (int i = 0; i < nseg; ++i)
        if (st[i] == c.t) s = i;
      if (s < 0) {
        if (nseg == kMaxSeg) {
          nseg = -1;
        } else {
          s = nseg++;
          st[s] = c.t; sylo[s] = syhi[s] = c.y; sxlo[s] = sxhi[s] = c.x;
        }
      }
      if (s >= 0) {
        sylo[s] = min(sylo[s], c.y); syhi[s] = max(syhi[s], c.y);
        sxlo[s] = min(sxlo[s], c.x); sxhi[s] = max(sxhi[s], c.x);
      }
    }
  }
  // Row-contiguity check: every row's span must be fully covered.
  int span = 0;
  for (int i = 0; i < nrows; ++i) {
    const uint2 rw = rows[i];
    span += static_cast<int>(rw.y & 0xFFFFu) - static_cast<int>(rw.y >> 16) + 1;
  }
  const int tokens = p1 - p0;
  for (int i = 0; i < max(nseg, 0); ++i)
    segs[i] = make_int4(st[i], (sylo[i] << 16) | syhi[i], (sxlo[i] << 16) | sxhi[i], 0);
  // Complete rectangles: consecutive rows of one frame with consecutive y and
  // the same x interval.  With contiguous rows every position of such a
  // rectangle is a key of the block, so a disk meets a key of the block iff
  // it meets one of the rectangles.
  int nrect = -1;
  if (span == tokens) {
    int4* rects = ws.rects + static_cast<size_t>(kb) * kMaxRect;
    nrect = 0;
    int ct = -1, cylo = 0, cyhi = 0, cx = 0;
    for (int i = 0; i <= nrows && nrect >= 0; ++i) {
      int t = -1, y = 0, xr = 0;
      if (i < nrows) {
        t = static_cast<int>(rows[i].x >> 16);
        y = static_cast<int>(rows[i].x & 0xFFFFu);
        xr = static_cast<int>(rows[i].y);
        if (t == ct && y == cyhi + 1 && xr == cx) {
          cyhi = y;
          continue;
        }
      }
      if (ct >= 0) {  // close the current rectangle
        if (nrect == kMaxRect) {
          nrect = -1;
          break;
        }
        rects[nrect++] = make_int4(ct, (cylo << 16) | cyhi, cx, 0);
      }
      ct = t; cylo = cyhi = y; cx = xr;
    }
  }
  ws.info[kb] = make_int4(span == tokens ? nrows : -1, nseg, tokens, nrect);
}

// -------------------------------------------------------------------- 2. votes

// grid (nqb, heads), kVoteThreads threads.  Dynamic smem: F * 128 ints
// (floor of each query's fp32 squared radius in each key frame) + 4 * F ints
// (per-frame union boxes of the disks).
//
// Exact phase: a warp takes one candidate key block; lane l holds queries
// l, l+32, l+64, l+96; the warp walks the block's rows (t, y, [x_lo, x_hi])
// and, per row, counts for each of its queries the keys of the row inside the
// query's disk: with m = floor(R2) - dy^2 >= 0 they are the x in [x_lo, x_hi]
// with (x - x_q)^2 <= m.  With a vote threshold of 1 only existence matters:
// the nearest x of the row is tested, and the block is kept at the first row
// where any query has a hit.
//
// LINE = true (1D distance): the table holds each query's reach s per key
// frame, the per-frame "box" is the index interval [min(n - s), max(n + s)],
// a key block's per-frame box becomes the index interval
// [y_lo * W + x_lo, y_hi * W + x_hi] (a superset of its tokens' indices) and
// a row (t, y, [x_lo, x_hi]) the interval [y W + x_lo, y W + x_hi].
template <bool LINE>
__global__ void __launch_bounds__(kVoteThreads) votes_kernel(const float* __restrict__ r,
                                                             const float* __restrict__ phi,
                                                             TileLayout L, int bq, int bk, int vote,
                                                             MaskWs ws) {
  extern __shared__ int s_dyn[];
  __shared__ float s_phi[kMaxFrames];
  __shared__ int s_qx[128], s_qy[128], s_qt[128];
  __shared__ float s_qr[128];
  __shared__ int s_count;
  const int N = L.F * L.H * L.W;
  const MaskDims md = mask_dims(L, bq, bk);
  const int qb = blockIdx.x, h = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int F = L.F;
  int* s_rsq = s_dyn;               // [F][128]
  int* bxlo = s_dyn + F * 128;      // [F] each
  int* bxhi = bxlo + F;
  int* bylo = bxlo + 2 * F;
  int* byhi = bxlo + 3 * F;

  for (int t = tid; t < F; t += kVoteThreads) {
    s_phi[t] = phi[t];
    bxlo[t] = INT_MAX; bxhi[t] = INT_MIN; bylo[t] = INT_MAX; byhi[t] = INT_MIN;
  }
  if (tid == 0) s_count = 0;
  const int q0 = qb * bq;
  const int nq = min(bq, N - q0);
  if (tid < 128) {
    if (tid < nq) {
      const Coord c = tile_major_coord(L, q0 + tid);
      float rv = r[static_cast<size_t>(h) * N + q0 + tid];
      if (rv != rv) rv = __int_as_float(0x7f800000);  // NaN keeps every key, like +inf
      s_qx[tid] = c.x; s_qy[tid] = c.y; s_qt[tid] = c.t; s_qr[tid] = rv;
    } else {
      s_qx[tid] = 0; s_qy[tid] = 0; s_qt[tid] = 0; s_qr[tid] = 0.f;
    }
  }
  __syncthreads();

  // Per key frame: each query's integer threshold, and the box containing
  // every query's disk in that frame.
  {
    const bool mine = tid < nq;
    const int qx = s_qx[tid], qy = s_qy[tid], qt = s_qt[tid];
    const float qr = s_qr[tid];
    for (int t = 0; t < F; ++t) {
      const int dt = t > qt ? t - qt : qt - t;
      int xlo = INT_MAX, xhi = INT_MIN, ylo = INT_MAX, yhi = INT_MIN;
      if constexpr (LINE) {
        const int reach = mine ? line_reach(qr, s_phi[dt]) : -1;  // -1: no key ever inside
        s_rsq[t * 128 + tid] = reach;
        if (mine) {
          const int qn = qy * L.W + qx;
          xlo = qn - reach; xhi = qn + reach; ylo = 0; yhi = 0;
        }
      } else {
        const int rsq = mine ? radius_sq(qr, s_phi[dt]) : -1;  // -1: no key ever inside
        s_rsq[t * 128 + tid] = rsq;
        if (mine) {
          const int sq = isqrt_floor(rsq);
          xlo = qx - sq; xhi = qx + sq; ylo = qy - sq; yhi = qy + sq;
        }
      }
      xlo = __reduce_min_sync(0xffffffffu, xlo);
      xhi = __reduce_max_sync(0xffffffffu, xhi);
      ylo = __reduce_min_sync(0xffffffffu, ylo);
      yhi = __reduce_max_sync(0xffffffffu, yhi);
      if (lane == 0 && xlo != INT_MAX) {
        atomicMin(&bxlo[t], xlo); atomicMax(&bxhi[t], xhi);
        atomicMin(&bylo[t], ylo); atomicMax(&byhi[t], yhi);
      }
    }
  }
  __syncthreads();

  const bool exists = (vote == 1);
  // this lane's queries
  int qx[4], qy[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    qx[k] = s_qx[lane + 32 * k];
    qy[k] = s_qy[lane + 32 * k];
    if constexpr (LINE) qx[k] += qy[k] * L.W;  // raster index n = y W + x
  }
  uint32_t* bits_row = ws.bits + (static_cast<size_t>(h) * md.nqb + qb) * md.nkbw;
  int my_count = 0;
  for (int w = warp; w < md.nkbw; w += kVoteThreads / 32) {
    // prune, lanes over key blocks
    const int kb = w * 32 + lane;
    bool survive = false;
    int4 info = make_int4(0, 0, 0, 0);
    if (kb < md.nkb) {
      info = ws.info[kb];
      if (info.y < 0) {
        survive = true;
      } else {
        const int4* sg = ws.segs + static_cast<size_t>(kb) * kMaxSeg;
        for (int i = 0; i < info.y && !survive; ++i) {
          const int4 s = sg[i];
          if (!in_bounds(s.x, F, ws.err)) continue;
          const int ylo = s.y >> 16, yhi = s.y & 0xFFFF, xlo = s.z >> 16, xhi = s.z & 0xFFFF;
          if constexpr (LINE) {
            const int nlo = ylo * L.W + xlo, nhi = yhi * L.W + xhi;
            survive = nlo <= bxhi[s.x] && nhi >= bxlo[s.x];
          } else {
            survive = ylo <= byhi[s.x] && yhi >= bylo[s.x] && xlo <= bxhi[s.x] && xhi >= bxlo[s.x];
          }
        }
      }
    }
    uint32_t cand = __ballot_sync(0xffffffffu, survive);
    uint32_t word = 0;
    // exact votes, lanes over queries, rows of the key block in turn
    while (cand) {
      const int b = __ffs(cand) - 1;
      cand &= cand - 1;
      const int kb2 = w * 32 + b;
      const int nrows = __shfl_sync(0xffffffffu, info.x, b);
      const int nseg = __shfl_sync(0xffffffffu, info.y, b);
      const int nrect = __shfl_sync(0xffffffffu, info.w, b);
      bool keep = false;
      if constexpr (!LINE) {
        // vote threshold 1 and complete rectangles: the disk / rectangle test
        // is exact (the nearest lattice point of a rectangle to the query is
        // one of its keys), so it decides the block without row tests
        if (exists && nrect >= 0) {
          const int4* rc = ws.rects + static_cast<size_t>(kb2) * kMaxRect;
          bool hit = false;
          for (int i = 0; i < nrect; ++i) {
            const int4 rr = rc[i];
            if (!in_bounds(rr.x, F, ws.err)) continue;
            const int* rs = s_rsq + rr.x * 128 + lane;
            const int ylo = rr.y >> 16, yhi = rr.y & 0xFFFF;
            const int xlo = rr.z >> 16, xhi = rr.z & 0xFFFF;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int lim = rs[32 * k];
              const int dx = max(0, max(xlo - qx[k], qx[k] - xhi));
              const int dy = max(0, max(ylo - qy[k], qy[k] - yhi));
              hit |= (lim >= 0) & (dx * dx + dy * dy <= lim);
            }
          }
          if (__any_sync(0xffffffffu, hit)) word |= 1u << b;
          continue;
        }
        // vote threshold above 1 and complete rectangles: per rectangle, the
        // queries whose disk holds it whole (its farthest corner inside: the
        // disk is convex) add its area at once, and each query whose circle
        // cuts it (nearest point inside, farthest corner outside) at least
        // one vote; the warp stops as soon as that lower bound reaches the
        // threshold.  Otherwise the cut queries are counted row by row,
        // again stopping at the threshold.
        if (!exists && nrect >= 0) {
          const int4* rc = ws.rects + static_cast<size_t>(kb2) * kMaxRect;
          int votes = 0;
          for (int i = 0; i < nrect && !keep; ++i) {
            const int4 rr = rc[i];
            if (!in_bounds(rr.x, F, ws.err)) continue;
            const int* rs = s_rsq + rr.x * 128 + lane;
            const int ylo = rr.y >> 16, yhi = rr.y & 0xFFFF;
            const int xlo = rr.z >> 16, xhi = rr.z & 0xFFFF;
            const int area = (yhi - ylo + 1) * (xhi - xlo + 1);
            int cnt = 0, own = 0, lim[4];
            uint32_t cut = 0u;  // bit k: query k's circle cuts the rectangle
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              lim[k] = rs[32 * k];
              const int dxn = max(0, max(xlo - qx[k], qx[k] - xhi));
              const int dyn = max(0, max(ylo - qy[k], qy[k] - yhi));
              const int dxf = max(qx[k] - xlo, xhi - qx[k]);
              const int dyf = max(qy[k] - ylo, yhi - qy[k]);
              const bool meets = lim[k] >= 0 && dxn * dxn + dyn * dyn <= lim[k];
              const bool whole = meets && dxf * dxf + dyf * dyf <= lim[k];
              cnt += whole ? area : 0;
              cut |= (meets && !whole) ? (1u << k) : 0u;
              // a cut query has at least one vote in the rectangle: the
              // rectangle's nearest point to it is one of its keys, inside
              own += (meets && !whole) ? 1 : 0;
            }
            votes += __reduce_add_sync(0xffffffffu, cnt);
            keep = votes >= vote;
            // exact votes so far plus one per cut query: enough to keep the block
            if (!keep) keep = votes + __reduce_add_sync(0xffffffffu, own) >= vote;
            if (keep || !__any_sync(0xffffffffu, cut != 0u)) continue;
            for (int y = ylo; y <= yhi && !keep; ++y) {
              int row_cnt = 0;
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int dy = y - qy[k];
                const int m = lim[k] - dy * dy;
                if (((cut >> k) & 1u) && m >= 0) {
                  const int sq = isqrt_floor(m);
                  const int lo = max(xlo, qx[k] - sq), hi = min(xhi, qx[k] + sq);
                  if (hi >= lo) row_cnt += hi - lo + 1;
                }
              }
              votes += __reduce_add_sync(0xffffffffu, row_cnt);
              keep = votes >= vote;
            }
          }
          if (keep) word |= 1u << b;
          continue;
        }
      }
      // Exact rejection first: if no query's disk (interval) meets any of the
      // block's per-frame boxes, no key of the block is inside any support.
      // One test per (query, box) instead of one per (query, row).
      if (nseg > 0) {
        const int4* sg = ws.segs + static_cast<size_t>(kb2) * kMaxSeg;
        bool hit = false;
        for (int i = 0; i < nseg; ++i) {
          const int4 sgm = sg[i];
          if (!in_bounds(sgm.x, F, ws.err)) continue;
          const int* rs = s_rsq + sgm.x * 128 + lane;
          const int ylo = sgm.y >> 16, yhi = sgm.y & 0xFFFF;
          const int xlo = sgm.z >> 16, xhi = sgm.z & 0xFFFF;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int lim = rs[32 * k];
            if constexpr (LINE) {
              const int nlo = ylo * L.W + xlo, nhi = yhi * L.W + xhi;
              const int dn = max(0, max(nlo - qx[k], qx[k] - nhi));
              hit |= (lim >= 0) & (dn <= lim);
            } else {
              const int dx = max(0, max(xlo - qx[k], qx[k] - xhi));
              const int dy = max(0, max(ylo - qy[k], qy[k] - yhi));
              hit |= (lim >= 0) & (dx * dx + dy * dy <= lim);
            }
          }
        }
        if (!__any_sync(0xffffffffu, hit)) continue;  // not kept: no votes at all
      }
      if (nrows >= 0) {
        const uint2* rows = ws.rows + static_cast<size_t>(kb2) * bk;
        int votes = 0;
        for (int i = 0; i < nrows; ++i) {
          const uint2 rw = rows[i];
          const int t = static_cast<int>(rw.x >> 16);
          if (!in_bounds(t, F, ws.err)) continue;
          const int y = static_cast<int>(rw.x & 0xFFFFu);
          const int xlo = static_cast<int>(rw.y >> 16);
          const int xhi = static_cast<int>(rw.y & 0xFFFFu);
          const int* rs = s_rsq + t * 128 + lane;
          if constexpr (LINE) {
            const int nlo = y * L.W + xlo, nhi = y * L.W + xhi;
            if (exists) {
              bool hit = false;
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int reach = rs[32 * k];
                const int dn = max(0, max(nlo - qx[k], qx[k] - nhi));
                hit |= (reach >= 0) & (dn <= reach);
              }
              if (__any_sync(0xffffffffu, hit)) { keep = true; break; }
            } else {
              int cnt = 0;
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int reach = rs[32 * k];
                if (reach >= 0) {
                  const int lo = max(nlo, qx[k] - reach), hi = min(nhi, qx[k] + reach);
                  if (hi >= lo) cnt += hi - lo + 1;
                }
              }
              votes += __reduce_add_sync(0xffffffffu, cnt);
              if (votes >= vote) { keep = true; break; }
            }
          } else if (exists) {
            bool hit = false;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int dy = y - qy[k];
              const int m = rs[32 * k] - dy * dy;
              const int dx = max(0, max(xlo - qx[k], qx[k] - xhi));
              hit |= (m >= 0) & (dx * dx <= m);
            }
            if (__any_sync(0xffffffffu, hit)) { keep = true; break; }
          } else {
            int cnt = 0;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int dy = y - qy[k];
              const int m = rs[32 * k] - dy * dy;
              if (m >= 0) {
                const int sq = isqrt_floor(m);
                const int lo = max(xlo, qx[k] - sq), hi = min(xhi, qx[k] + sq);
                if (hi >= lo) cnt += hi - lo + 1;
              }
            }
            votes += __reduce_add_sync(0xffffffffu, cnt);
            if (votes >= vote) { keep = true; break; }
          }
        }
      } else {
        // key block whose rows are not contiguous: token by token
        int votes = 0;
        const int p1 = min(N, (kb2 + 1) * bk);
        for (int pp = kb2 * bk; pp < p1 && !keep; ++pp) {
          const Coord c = tile_major_coord(L, pp);
          if (!in_bounds(c.t, F, ws.err)) continue;
          const int* rs = s_rsq + c.t * 128 + lane;
          int cnt = 0;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if constexpr (LINE) {
              const int dn = abs(c.y * L.W + c.x - qx[k]);
              cnt += (rs[32 * k] >= 0 && dn <= rs[32 * k]) ? 1 : 0;
            } else {
              const int dx = c.x - qx[k], dy = c.y - qy[k];
              cnt += (dx * dx + dy * dy <= rs[32 * k]) ? 1 : 0;
            }
          }
          votes += __reduce_add_sync(0xffffffffu, cnt);
          keep = votes >= vote;
        }
      }
      if (keep) word |= 1u << b;
    }
    if (lane == 0) bits_row[w] = word;
    my_count += __popc(word);
  }
  if (lane == 0) atomicAdd(&s_count, my_count);
  __syncthreads();
  if (tid == 0) ws.counts[static_cast<size_t>(h) * md.nqb + qb] = s_count;
}

// --------------------------------------------------------------------- 3. scan

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) scan_kernel(int heads, int nqb, MaskWs ws,
                                                            int* row_ptr, int* nnz) {
  __shared__ long long s_warp[kScanThreads / 32];
  const long long M = static_cast<long long>(heads) * nqb;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long per = (M + kScanThreads - 1) / kScanThreads;
  const long long b = tid * per, e = min(M, b + per);
  long long local = 0;
  for (long long i = b; i < e; ++i) local += ws.counts[i];
  // block exclusive scan of `local`
  long long incl = local;
  for (int o = 1; o < 32; o <<= 1) {
    const long long v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    long long v = s_warp[lane];
    long long vi = v;
    for (int o = 1; o < 32; o <<= 1) {
      const long long u = __shfl_up_sync(0xffffffffu, vi, o);
      if (lane >= o) vi += u;
    }
    s_warp[lane] = vi - v;  // exclusive over warps
  }
  __syncthreads();
  long long run = s_warp[warp] + incl - local;
  for (long long i = b; i < e; ++i) {
    const int h = static_cast<int>(i / nqb);
    const int qb = static_cast<int>(i - static_cast<long long>(h) * nqb);
    row_ptr[static_cast<size_t>(h) * (nqb + 1) + qb] = static_cast<int>(run);
    run += ws.counts[i];
    if (qb == nqb - 1) row_ptr[static_cast<size_t>(h) * (nqb + 1) + nqb] = static_cast<int>(run);
  }
  if (e == M && b < e) *nnz = static_cast<int>(run);
  if (M == 0 && tid == 0) *nnz = 0;
}

// ------------------------------------------------------------------ 4. compact

constexpr int kCompactWarps = 8;

__global__ void __launch_bounds__(kCompactWarps * 32) compact_kernel(int heads, int nqb, int nkbw,
                                                                     MaskWs ws,
                                                                     const int* __restrict__ row_ptr,
                                                                     int* col_idx,
                                                                     long long capacity) {
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kCompactWarps + (threadIdx.x >> 5);
  if (row >= static_cast<long long>(heads) * nqb) return;
  const int h = static_cast<int>(row / nqb);
  const int qb = static_cast<int>(row - static_cast<long long>(h) * nqb);
  long long off = row_ptr[static_cast<size_t>(h) * (nqb + 1) + qb];
  const uint32_t* bits = ws.bits + row * nkbw;
  for (int base = 0; base < nkbw; base += 32) {
    const int w = base + lane;
    uint32_t word = w < nkbw ? bits[w] : 0u;
    const int c = __popc(word);
    int incl = c;
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    long long pos = off + incl - c;
    while (word) {
      const int bit = __ffs(word) - 1;
      word &= word - 1;
      if (pos < capacity) col_idx[pos] = w * 32 + bit;
      ++pos;
    }
    off += __shfl_sync(0xffffffffu, incl, 31);
  }
}

}  // namespace

size_t mask_workspace_bytes(int heads, const TileLayout& L, int block_q, int block_k) {
  return carve(L, heads, block_q, block_k, nullptr, nullptr);
}

cudaError_t launch_block_mask(const float* r, const float* phi, int heads, const TileLayout& L,
                              int block_q, int block_k, int vote, bool line, int* row_ptr,
                              int* col_idx, long long capacity, int* nnz, void* workspace,
                              cudaStream_t stream) {
  MaskWs ws;
  carve(L, heads, block_q, block_k, static_cast<char*>(workspace), &ws);
  ws.err = device_error_word();
  const MaskDims md = mask_dims(L, block_q, block_k);
  footprint_kernel<<<(md.nkb + 127) / 128, 128, 0, stream>>>(L, block_k, ws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t votes_smem = (static_cast<size_t>(L.F) * 128 + 4 * L.F) * sizeof(int);
  auto kernel = line ? votes_kernel<true> : votes_kernel<false>;
  if (votes_smem > 48 * 1024) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(votes_smem));
    if (e != cudaSuccess) return e;
  }
  kernel<<<dim3(md.nqb, heads), kVoteThreads, votes_smem, stream>>>(r, phi, L, block_q, block_k,
                                                                    vote, ws);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  scan_kernel<<<1, kScanThreads, 0, stream>>>(heads, md.nqb, ws, row_ptr, nnz);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long rows = static_cast<long long>(heads) * md.nqb;
  compact_kernel<<<static_cast<unsigned>((rows + kCompactWarps - 1) / kCompactWarps),
                   kCompactWarps * 32, 0, stream>>>(heads, md.nqb, md.nkbw, ws, row_ptr, col_idx,
                                                    capacity);
  return cudaGetLastError();
}

}  // namespace tra
