/*
 * tra.h — C ABI of the Token Radius Attention (TRA) hot path on B200 (sm_100a).
 *
 * The method: "Token Radius Attention for Efficient Video Generation"
 * (summaries at gist.science, paper 2608.02504; section names below follow
 * those pages).  A dense warm-up attention pass also yields every query's
 * softmax entropy H_i; the entropy sets a per-query token budget
 * B_i = tau * exp(H_i) / N (§2 Insight I); the budget becomes a base radius
 * that shrinks with temporal distance by phi(delta) = exp(-gamma * delta)
 * (§2 Insight II); a fused kernel turns the per-token disks into a
 * block-sparse query-block x key-block mask over a tile-major token order
 * (§2 "TRA pipeline", efficient execution); later denoising steps run exact
 * softmax attention over the kept blocks only, reusing the entropy
 * (cross-step reuse).
 *
 * Conventions shared by every call:
 *  - Pointers are DEVICE pointers owned by the caller unless a comment says
 *    otherwise.  The library never allocates device memory; scratch space is
 *    passed in (see tra_mask_workspace_size).  Each call asks the CUDA runtime
 *    where its pointers live and returns TRA_ERR_INVALID_ARGUMENT, launching
 *    nothing, for host memory (pageable or pinned) or memory of another
 *    device; managed memory is accepted.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream) and never synchronises, except tra_get_device_error.
 *  - Every call checks its arguments first and launches nothing when it
 *    returns an error.  heads == 0 or N == 0 is a valid empty problem.
 *  - Tensors are [heads, N, d] with d contiguous (batch folded into heads),
 *    N = F * H * W tokens.  The original token order is (t, y, x) row-major,
 *    token n = (t * H + y) * W + x.
 *  - Calls on distinct streams may run concurrently from several threads.
 *  - A device-side wait that runs out of time (it never should) makes the
 *    kernel record a code in a device error word and return early; the next
 *    tra_get_device_error reports it.  A CSR row that a kernel finds invalid
 *    is skipped (its queries get O = 0, lse = -inf) and recorded the same
 *    way.  No kernel traps.
 *  - Requires a compute capability 10.0 GPU (B200, sm_100a).
 *  - The library looks up the device addresses of its two module-scope
 *    objects (the device error word and the scratch array of
 *    tra_build_block_mask_noalloc) once per device and keeps them.  A
 *    cudaDeviceReset, or anything else that destroys the device's primary
 *    context, while the library is loaded leaves those addresses stale: do
 *    not reset a device between calls into this library.
 */
#ifndef TRA_H_
#define TRA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* tra_stream_t; /* identical to cudaStream_t */

typedef enum {
  TRA_OK = 0,
  TRA_ERR_INVALID_ARGUMENT = 1, /* null, misaligned or host pointer, bad size */
  TRA_ERR_UNSUPPORTED = 2,      /* valid but outside the supported shapes */
  TRA_ERR_WORKSPACE = 3,        /* workspace too small or misaligned */
  TRA_ERR_CAPACITY = 4,         /* col_idx capacity negative */
  TRA_ERR_CUDA = 5,             /* a CUDA runtime call failed (launch, attribute) */
  TRA_ERR_DEVICE = 6,           /* no usable sm_100 device */
  TRA_ERR_TIMEOUT = 7,          /* reported by tra_get_device_error: a wait ran out of time */
  TRA_ERR_BAD_INPUT = 8         /* reported by tra_get_device_error: a kernel met an invalid
                                   CSR row (negative start, or longer than nKB), or (checked
                                   builds only) an index outside what it indexes */
} tra_status;

typedef enum { TRA_BF16 = 0, TRA_F32 = 1 } tra_dtype;

/* Latent video grid: F frames of H x W tokens. */
typedef struct { int F, H, W; } tra_grid;

/* Tile shape of the tile-major order: t frames x y rows x x columns. */
typedef struct { int t, y, x; } tra_tile;

/* Static description of a status code; never NULL. */
const char* tra_status_string(tra_status s);

/* Library version, major * 10000 + minor * 100 + patch. */
int tra_version(void);

/*
 * Tile-major permutation (§2 "TRA pipeline", tile-major layout: tokens are
 * re-ordered so that spatial neighbours are contiguous).
 *
 * X_tm[h, p, :] = X[h, pi(p), :], where pi walks the tiles of `tile` in
 * (frame-tile, tile-row, tile-col) order and, inside a tile, its tokens in
 * (t, y, x) row-major order; tiles at the grid's far edges are truncated, so
 * pi is a bijection on [0, N).
 *   X     [heads, N, d] of in_dtype, original order; read only.
 *   X_tm  [heads, N, d] of out_dtype, tile-major order; written.  Must not
 *         overlap X.  f32 -> bf16 rounds to nearest even.
 *   d     multiple of 8, 8..1024.  X and X_tm 16-byte aligned.
 */
tra_status tra_tile_major_permute(const void* X, void* X_tm, tra_dtype in_dtype,
                                  tra_dtype out_dtype, int heads, int d, tra_grid grid,
                                  tra_tile tile, tra_stream_t stream);

/*
 * Inverse of tra_tile_major_permute: X[h, pi(p), :] = X_tm[h, p, :].
 * Same dtype on both sides; same shape rules.
 */
tra_status tra_inverse_permute(const void* X_tm, void* X, tra_dtype dtype, int heads, int d,
                               tra_grid grid, tra_tile tile, tra_stream_t stream);

/*
 * Dense warm-up attention with per-query entropy (§2 "TRA pipeline" step 1:
 * entropy of every query from the dense warm-up phase; §3 contribution 3:
 * fused entropy kernel).
 *
 * For every head and query i (rows of Q, any fixed token order):
 *   s_ij = scale * q_i . k_j over all N keys j,
 *   O_i  = sum_j softmax(s_i)_j v_j                 (bf16, fp32 accumulation)
 *   H_i  = ln Z_i - (sum_j e^{s_ij} s_ij) / Z_i,  Z_i = sum_j e^{s_ij}
 *                                                 (natural log, fp32)
 *   lse_i = ln Z_i                                 (fp32; optional)
 *   Q, K, V  [heads, N, d] bf16, 16-byte aligned; read only.
 *   O        [heads, N, d] bf16; written.
 *   H        [heads, N] fp32; written.
 *   lse      [heads, N] fp32 or NULL.
 *   d        64 or 128.   scale > 0 and finite (1/sqrt(d) for standard SDPA).
 *   N        1 .. 2^24 (0 is an empty problem).
 * Tensor cores (tcgen05, bf16 in, fp32 accumulators in tensor memory) run
 * QK^T and PV; entropy statistics are kept in fp32 beside the online softmax.
 */
tra_status tra_dense_attn_entropy(const void* Q, const void* K, const void* V, void* O,
                                  float* H, float* lse, int heads, int N, int d, float scale,
                                  tra_stream_t stream);

/*
 * Entropy-only pass: the H_i (and lse_i) of tra_dense_attn_entropy without
 * the PV product and without writing an output.  For refreshing the entropy
 * (and so the mask) at a step whose output comes from the block-sparse call
 * (§2 "TRA pipeline", cross-step reuse: the entropy pattern is stable across
 * denoising steps, so it is recomputed only now and then).
 *   Q, K  [heads, N, d] bf16, 16-byte aligned; read only.
 *   H     [heads, N] fp32; written.    lse  [heads, N] fp32 or NULL.
 *   d 64 or 128; scale > 0 and finite; N 1 .. 2^24.
 */
tra_status tra_attn_entropy(const void* Q, const void* K, float* H, float* lse, int heads, int N,
                            int d, float scale, tra_stream_t stream);

/*
 * Entropy -> budget -> radius (§2 Insight I: B_i = tau * exp(H_i) / N;
 * Insight II and pipeline step 2: budget -> query-specific base radius,
 * per-frame radius r_i * phi(|dt|), phi(delta) = exp(-gamma * delta)).
 *
 * The budget becomes a radius by equal area: the disks of all key frames
 * together hold K_i = B_i * N tokens,
 *   K_i = pi * r_i^2 * S(t_i),   S(t) = sum_{t'=0}^{F-1} phi(|t' - t|)^2,
 * so r_i = sqrt(tau * exp(H_i) / (pi * S(t_i))), with t_i the frame of query i.
 *   H        [heads, N] fp32 in TILE-MAJOR order (as produced by the dense
 *            call on permuted inputs); read only.  +inf gives r = +inf,
 *            NaN gives NaN (the mask keeps every key for either).
 *   r        [heads, N] fp32, tile-major order; written.
 *   phi_out  [F] fp32 or NULL: phi(delta) for delta = 0..F-1, the table the
 *            mask call reads.  Computed in double on the host, rounded once.
 *   tau >= 0 and finite; gamma >= 0 and finite; F <= 1024.
 */
tra_status tra_budget_radius(const float* H, float* r, float* phi_out, int heads, tra_grid grid,
                             tra_tile tile, float tau, float gamma, tra_stream_t stream);

/*
 * Bytes of device scratch space tra_build_block_mask needs for these sizes
 * (0 if the sizes are invalid).  The space must be 256-byte aligned.  The
 * tile is validated like the mask call's; the size itself depends only on
 * heads, N and the block sizes.
 */
size_t tra_mask_workspace_size(int heads, tra_grid grid, tra_tile tile, int block_q, int block_k);

/*
 * The same size without a tile argument: tra_mask_workspace_size with the
 * 1 frame x 4 rows x 4 columns tile, which gives the size for every tile.
 */
size_t tra_workspace_size(int heads, tra_grid grid, int block_q, int block_k);

/*
 * Fused radius mask -> block-sparse CSR (§2 "TRA pipeline", efficient
 * execution: one kernel fuses distance computation, radius comparison, block
 * pruning and token voting, turning the irregular token-level radius mask
 * into a regular block-sparse mask).
 *
 * Token mask: key j is in query i's support when
 *     dx^2 + dy^2 <= R2,   R2 = fl32(R * R),  R = fl32(r_i * phi[|t_j - t_i|])
 * (integer token distances, inclusive compare, rounded fp32 products with no
 * fused multiply-add; a radius of +inf or NaN keeps every key).
 * Blocks are consecutive runs of block_q (block_k) TILE-MAJOR positions, the
 * last one possibly shorter.  votes(qb, kb) = number of token pairs in the
 * support with the query in qb and the key in kb; a block pair is kept when
 * votes >= vote_threshold.  Pruning by per-frame bounding boxes only skips
 * pairs with no votes, so the mask equals the brute-force definition.
 *   r            [heads, N] fp32 tile-major; read only.
 *   phi          [F] fp32 device table (e.g. written by tra_budget_radius).
 *   row_ptr      [heads * (nqb + 1)] int32, nqb = ceil(N / block_q); written.
 *                Row (h, qb) is col_idx[row_ptr[h*(nqb+1)+qb] .. row_ptr[h*(nqb+1)+qb+1]);
 *                offsets are global over all heads (row_ptr[0] = 0).
 *   col_idx      [col_capacity] int32; written: kept kb of each row, ascending.
 *   nnz          [1] int32; written: total kept blocks.  If it exceeds
 *                col_capacity after the call completes, col_idx holds only the
 *                first col_capacity entries (capacity h*nqb*nkb never overflows).
 *   workspace    >= tra_mask_workspace_size(...) bytes, 256-byte aligned.
 *   block_q, block_k in {16, 64, 128};  vote_threshold >= 1;  tile as given
 *   to tra_tile_major_permute;  F <= 384 (TRA_ERR_UNSUPPORTED above);
 *   H, W <= 16384.
 */
tra_status tra_build_block_mask(const float* r, const float* phi, int heads, tra_grid grid,
                                tra_tile tile, int block_q, int block_k, int vote_threshold,
                                int* row_ptr, int* col_idx, long long col_capacity, int* nnz,
                                void* workspace, size_t workspace_bytes, tra_stream_t stream);

/*
 * Size in bytes of the scratch buffer built into the library for
 * tra_build_block_mask_noalloc.  Every GPU that loads the library holds this
 * much device memory until the process exits.
 */
#define TRA_MASK_STATIC_SCRATCH_BYTES (8u * 1024u * 1024u)

/*
 * tra_build_block_mask for callers that cannot allocate or pass scratch
 * memory, such as a plugin that receives only its input and output tensors
 * from a host framework that owns all device memory, or a latency-critical
 * caller that must not allocate mid-run.  The pages have no counterpart for
 * this call: it is a packaging variant of the fused mask above.
 *
 * Inputs, outputs, rules and results are those of tra_build_block_mask; only
 * workspace / workspace_bytes are gone.  Scratch comes from one buffer of
 * TRA_MASK_STATIC_SCRATCH_BYTES compiled into the library (one per device).
 * A problem that needs more (tra_mask_workspace_size(...) larger than that) is
 * refused with TRA_ERR_WORKSPACE before anything is launched.  The call
 * allocates nothing and calls no allocator.
 *
 * The first call on each device looks up the device address of the built-in
 * buffer (cudaGetSymbolAddress, with that device current); make that first
 * call before any stream capture.  All calls on a device share the buffer and
 * leave their data in it: calls whose kernels overlap on the GPU (different
 * streams or host threads) race and corrupt each other's results, so issue
 * them in order on one stream.
 */
tra_status tra_build_block_mask_noalloc(const float* r, const float* phi, int heads,
                                        tra_grid grid, tra_tile tile, int block_q, int block_k,
                                        int vote_threshold, int* row_ptr, int* col_idx,
                                        long long col_capacity, int* nnz, tra_stream_t stream);

/*
 * ---- Mask variants -------------------------------------------------------
 * The ablations of the Token Radius Attention summary (§4 results, ablation
 * study: the entropy-to-budget mapping removed, or the radius mask replaced
 * by a 1D distance) and the static mask of "Radial Attention: O(n log n)
 * Sparse Attention with Energy Decay for Long Video Generation" (abstract:
 * each token attends to spatially nearby tokens, with a window that shrinks
 * with temporal distance and a compute density that decays with it).  They
 * differ from TRA only in where the radius comes from and in the distance;
 * the votes, the CSR and the block-sparse attention are the same.
 */
typedef enum {
  TRA_METRIC_DISK = 0, /* dx^2 + dy^2 in the frame (TRA's radius mask) */
  TRA_METRIC_LINE = 1  /* (n_j - n_i)^2 with the in-frame raster index n = y * W + x */
} tra_metric;

typedef enum {
  TRA_BUDGET_ENTROPY = 0, /* K_i = tau * exp(H_i): TRA's per-query budget */
  TRA_BUDGET_SHARED = 1   /* K_h = mean over the head's queries of tau * exp(H_i),
                             the same budget for every query of head h */
} tra_budget;

/*
 * tra_budget_radius with a choice of budget and distance.
 *   budget   TRA_BUDGET_ENTROPY: K_i = tau * exp(H_i) (tra_budget_radius).
 *            TRA_BUDGET_SHARED: K_h = tau * (sum_i exp(H_i)) / N for every
 *            query of head h, so the head's total budget is unchanged; the
 *            sum runs in double in a fixed order, and each radius is
 *            evaluated in double and rounded once.  One +inf entropy makes
 *            the whole head's radii +inf, one NaN makes them NaN.
 *   metric   TRA_METRIC_DISK: equal area, r = sqrt(K / (pi * S(t))),
 *            S(t) = sum_t' phi(|t' - t|)^2 (as tra_budget_radius).
 *            TRA_METRIC_LINE: equal length, the 1D windows of all key frames
 *            hold K = 2 * r * L(t) tokens, L(t) = sum_t' phi(|t' - t|), so
 *            r = K / (2 * L(t)).
 * Everything else (layouts, phi_out, limits) is as for tra_budget_radius.
 */
tra_status tra_budget_radius_ex(const float* H, float* r, float* phi_out, int heads,
                                tra_grid grid, tra_tile tile, float tau, float gamma,
                                tra_budget budget, tra_metric metric, tra_stream_t stream);

/*
 * Radial Attention's static window as a radius source (no entropy).
 *   r        [heads, N] fp32; written: r0 for every query.
 *   phi_out  [F] fp32 or NULL: the window factor per temporal distance delta,
 *            phi_R(delta) = 2^(-b/2) for TRA_METRIC_DISK and 2^(-b) for
 *            TRA_METRIC_LINE, b = floor(log2(delta + 1)).  Each time the
 *            temporal distance doubles, the window's area (length) halves, so
 *            every band of temporal distances holds the same number of keys
 *            and a query's support grows with log F.
 *   r0 >= 0 (+inf keeps every key); F <= 1024.
 * Feed r and phi_out to tra_build_block_mask_ex with the same metric.
 */
tra_status tra_radial_radius(float* r, float* phi_out, int heads, tra_grid grid, tra_tile tile,
                             float r0, tra_metric metric, tra_stream_t stream);

/*
 * tra_build_block_mask with a choice of distance.  TRA_METRIC_DISK is
 * tra_build_block_mask.  TRA_METRIC_LINE keeps key j for query i when
 *     (n_j - n_i)^2 <= R2,  n = y * W + x,  R2 and R as for the disk,
 * so in each key frame the query keeps the raster-index interval
 * [n_i - s, n_i + s], s = floor(sqrt(floor(R2))), which runs across row
 * ends.  Votes, CSR, workspace and limits are those of tra_build_block_mask.
 */
tra_status tra_build_block_mask_ex(const float* r, const float* phi, int heads, tra_grid grid,
                                   tra_tile tile, int block_q, int block_k, int vote_threshold,
                                   tra_metric metric, int* row_ptr, int* col_idx,
                                   long long col_capacity, int* nnz, void* workspace,
                                   size_t workspace_bytes, tra_stream_t stream);

/*
 * Block-sparse attention over the kept blocks (§2 "TRA pipeline": the
 * block-sparse mask drives a block-sparse attention backend; reuse across
 * sparse steps).  Exact softmax over every token of the kept key blocks of
 * each query's block row; tokens >= N are excluded; a query whose row keeps
 * nothing gets O = 0 and lse = -inf.
 *   Q, K, V   [heads, N, d] bf16 tile-major, 16-byte aligned; read only.
 *   O         [heads, N, d] bf16; written.
 *   lse       [heads, N] fp32 natural-log sum of exponentials, or NULL.
 *   row_ptr, col_idx  CSR as written by tra_build_block_mask for the same
 *             heads, N, block_q, block_k (col_idx ascending, no repeats).
 *             A row whose start is negative or that holds more than nKB
 *             entries is skipped (O = 0, lse = -inf) and reported through
 *             tra_get_device_error (TRA_ERR_BAD_INPUT).  With 64-row query
 *             blocks, where two rows share a tile, a row that is not strictly
 *             ascending within [0, nKB) is skipped and reported the same way;
 *             otherwise an entry outside [0, nKB) adds no keys.
 *   d in {64, 128}; block_q, block_k in {16, 64, 128};  when block_q < 128
 *   and either block is 16 tokens, ceil(N / block_k) <= 1024.  scale > 0 and
 *   finite.
 */
tra_status tra_block_sparse_attn(const void* Q, const void* K, const void* V, void* O,
                                 float* lse, const int* row_ptr, const int* col_idx, int heads,
                                 int N, int d, int block_q, int block_k, float scale,
                                 tra_stream_t stream);

/*
 * ---- FP8 scores -----------------------------------------------------------
 * The block-sparse call with QK^T on the tensor cores' 8-bit (E4M3) kind:
 * same mask, same exact softmax over the kept blocks, PV still in bf16.  The
 * pages fix no precision; the quantization below is this library's reading.
 *
 * Per-block E4M3 quantization of a bf16 tensor.  For every head and every
 * block of `block` consecutive rows: amax = max |x| over the block,
 * scale = fl32(amax / 448) (1 for an all-zero block), and
 * Xq = E4M3(fl32(x / scale)) (OCP FP8 E4M3, ties to even, saturating).
 *   X       [heads, N, d] bf16, 16-byte aligned; read only.
 *   Xq      [heads, N, d] bytes (E4M3 codes), 16-byte aligned; written.
 *   scales  [heads, ceil(N / block)] fp32; written.
 *   d in {64, 128}; block in {64, 128}.
 */
tra_status tra_quantize_e4m3(const void* X, void* Xq, float* scales, int heads, int N, int d,
                             int block, tra_stream_t stream);

/*
 * tra_block_sparse_attn with E4M3 queries and keys: the score of query i and
 * key j is scale * q_scales[i / 128] * k_scales[j / 128] * (q8_i . k8_j),
 * accumulated in fp32 on the tensor cores; the rest is tra_block_sparse_attn.
 *   Q8, K8    [heads, N, 128] E4M3 codes from tra_quantize_e4m3 with block 128.
 *   q_scales, k_scales  [heads, ceil(N / 128)] fp32 from the same call.
 *   V, O, lse, row_ptr, col_idx, scale: as for tra_block_sparse_attn.
 *   d = 128 and block_q = block_k = 128 only (TRA_ERR_UNSUPPORTED otherwise).
 */
tra_status tra_block_sparse_attn_fp8(const void* Q8, const float* q_scales, const void* K8,
                                     const float* k_scales, const void* V, void* O, float* lse,
                                     const int* row_ptr, const int* col_idx, int heads, int N,
                                     int d, int block_q, int block_k, float scale,
                                     tra_stream_t stream);

/*
 * Self-test of failure detection.  Launches one kernel that waits, with the
 * same bounded-wait helper every kernel here uses, on a barrier that nothing
 * ever completes.  After `limit_ms` the wait gives up, the kernel records
 * code 11 in the device error word and returns, so the context stays usable:
 * the next tra_get_device_error returns TRA_ERR_TIMEOUT with *code = 11.
 *   limit_ms   1 .. 2000.
 *   completed  [1] int32 device pointer (16-byte aligned) or NULL; written:
 *              1 if the wait completed (it never should), 0 if it gave up.
 * The other kernels use a limit of 4 s.
 */
tra_status tra_selftest_wait_timeout(int limit_ms, int* completed, tra_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the device error word of the
 * current device.  *code = 0 when no kernel recorded an error; otherwise the
 * first code recorded:
 *    1 .. 9  a wait that ran out of time (1 Q tile, 2 / 3 K / V tile loaded,
 *            4 / 5 K / V stage free, 6 scores ready, 7 score buffer free,
 *            8 probabilities ready, 9 PV product done)  -> TRA_ERR_TIMEOUT
 *    10      an invalid CSR row (negative start, or longer than nKB; the
 *            row is skipped)                              -> TRA_ERR_BAD_INPUT
 *    11      the self-test's wait (tra_selftest_wait_timeout) -> TRA_ERR_TIMEOUT
 *    12      checked builds only (libtra_check.so, compiled with TRA_CHECK): an
 *            index a kernel derived from the layout or from data it read fell
 *            outside what it indexes; the access was skipped -> TRA_ERR_BAD_INPUT
 * Returns TRA_OK when *code == 0, TRA_ERR_CUDA when the stream reported a
 * CUDA error.
 */
tra_status tra_get_device_error(int* code, tra_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TRA_H_ */
