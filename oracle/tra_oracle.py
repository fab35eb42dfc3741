"""CPU oracle of the Token Radius Attention (TRA) hot path.

TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke entry point and the bench's
CPU-baseline leg may import this module.  The library (entropy_adaptive_radius_b200)
never imports it, and it imports nothing from the library: the two share no
code.  Every step here is the plain definition, in float64 unless a step fixes
another precision, with no blocking, fusion or reordering, so that it can be
checked against the pages by eye.

Sources (all are summaries of "Token Radius Attention for Efficient Video
Generation", gist.science paper 2608.02504, in Japanese, Portuguese and Hindi;
section names follow the Japanese page):
  * §2 Insight I: per-query budget  B = tau * exp(H_i) / N  from the attention
    entropy H_i, with no sorting or ranking.
  * §2 Insight II: the budget becomes a spatial radius around the query; the
    radius shrinks with temporal distance by phi(delta) = exp(-gamma * delta).
  * §2 "TRA pipeline": entropy from a dense warm-up pass, budget -> base radius
    -> per-frame radius forming a 2D disk mask; tile-major token order; one
    fused kernel for distance, radius compare, block pruning and token voting
    that turns the token mask into a block-sparse mask; entropy reused across
    denoising steps.

Readings taken where the pages leave a step open:
  R1 scores s_ij = q_i . k_j / sqrt(d); natural logarithm.
  R2 entropy over all N keys of the same head.
  R3 tile-major order: tiles ordered frame-tile, tile-row, tile-col; inside a
     tile (t, y, x) row-major; edge tiles truncated.
  R4 budget -> radius by equal area: the disks of all key frames together hold
     K_i = B_i * N tokens, i.e. K_i = pi * r_i^2 * sum_t' phi(|t' - t_i|)^2, the
     sum running over the frames that exist.
  R5 a key j is inside query i's support when dx^2 + dy^2 <= R^2 with
     R = r_i * phi(|t_j - t_i|); the compare is taken in float32 as
     R32 = fl(r32 * phi32), R2 = fl(R32 * R32), inclusive, with +inf or NaN radii
     keeping every key.
  R6 a vote is one (query, key) token pair inside the support; a block pair is
     kept when its votes reach the vote threshold.
  R7 a kept block pair contributes every one of its tokens to the exact
     softmax; a query whose row keeps nothing gets O = 0 and LSE = -inf.

Mask variants (the ablations of §4 "ablation study", and the static mask of
"Radial Attention: O(n log n) Sparse Attention with Energy Decay for Long
Video Generation", abstract), all through the same token mask and votes:
  R12 shared budget (entropy mapping removed): every query of a head gets the
      budget K_h = mean over the head's queries of tau * exp(H_i), so the
      head's total budget is unchanged; the radius follows from K_h as in R4.
  R13 1D distance (radius masking replaced by a 1D distance): the distance of
      two tokens is the difference of their in-frame raster indices
      n = y * W + x; a key is inside when (n_j - n_i)^2 <= R^2 with R as in R5;
      the budget becomes a radius by equal length,
      K_i = 2 r_i * sum_t' phi(|t' - t_i|).
  R14 Radial's static window: every query has the same base radius r0 (no
      entropy), and the decay table is phi_R(delta) = 2^(-b/2) for the disk
      (2^(-b) for the 1D distance) with b = floor(log2(delta + 1)): each time
      the temporal distance doubles the window's area (length) halves, so every
      band of temporal distances holds the same number of keys and a query's
      support grows with log F (the O(n log n) cost the Radial page states).

FP8 scores (the last "next" row: same mask, QK^T on FP8 tensor cores):
  R16 Q and K are quantized per (head, block of rows) to OCP FP8 E4M3: the
      block's scale is fl32(amax / 448) (1 for an all-zero block) and each
      element becomes the nearest E4M3 value (ties to even, saturating at
      448) to fl32(x / scale); scores are scale_q * scale_k * (q8 . k8) times
      the softmax scale, and everything after the scores is unchanged.  The
      pages say nothing about precision; this is the plainest per-block
      scaled FP8 reading.

Cross-step reuse (§2 "TRA pipeline": the entropy is computed in the dense
warm-up phase and reused by the later sparse steps):
  R15 the first `warmup` steps are dense (output and entropy); every later
      step is sparse with the mask of the last entropy refresh; with
      refresh_every = k > 0, every k-th sparse-phase step also refreshes the
      entropy from its own Q and K, either as a dense step ("dense": dense
      output) or after its sparse output ("entropy": an entropy-only pass);
      the new mask serves the steps after it.
"""
import math

import numpy as np

# ---------------------------------------------------------------------------
# tile-major layout  (§2 "TRA pipeline", tile-major layout; reading R3)
# ---------------------------------------------------------------------------


def tile_major_order(F, H, W, tile=(1, 4, 4)):
    """pi[p] = original index (t*H + y)*W + x of the token at tile-major
    position p.  Built by walking the tiles in order and, inside each tile,
    its tokens in (t, y, x) row-major order."""
    tt, ty, tx = tile
    order = []
    for t0 in range(0, F, tt):
        for y0 in range(0, H, ty):
            for x0 in range(0, W, tx):
                for t in range(t0, min(F, t0 + tt)):
                    for y in range(y0, min(H, y0 + ty)):
                        for x in range(x0, min(W, x0 + tx)):
                            order.append((t * H + y) * W + x)
    return np.array(order, dtype=np.int64)


def token_coords(F, H, W):
    """[N, 3] int64 (x, y, t) of original token n = (t*H + y)*W + x."""
    n = np.arange(F * H * W, dtype=np.int64)
    return np.stack([n % W, (n // W) % H, n // (H * W)], axis=1)


def permute(X, pi):
    """X_tm[h, p, :] = X[h, pi[p], :]."""
    return X[:, pi, :]


def inverse_permute(X_tm, pi):
    """X[h, pi[p], :] = X_tm[h, p, :]."""
    X = np.empty_like(X_tm)
    X[:, pi, :] = X_tm
    return X


# ---------------------------------------------------------------------------
# dense attention and entropy  (§1 dense 3D self-attention; §2 pipeline step 1;
# readings R1, R2)
# ---------------------------------------------------------------------------


def scores(Q, K, scale):
    """s = scale * Q K^T for one head, float64 [Nq, Nk]."""
    return scale * (np.asarray(Q, np.float64) @ np.asarray(K, np.float64).T)


def softmax_attention(Q, K, V, scale, key_mask=None):
    """Exact softmax attention of one head.

    Returns (O [Nq, d], LSE [Nq], P [Nq, Nk]).  `key_mask` (bool [Nq, Nk])
    restricts each query to its kept keys; a row with no kept key has
    O = 0, LSE = -inf and P = 0 (reading R7)."""
    s = scores(Q, K, scale)
    if key_mask is not None:
        s = np.where(key_mask, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    empty = ~np.isfinite(m[:, 0])
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m)
    Z = e.sum(axis=1, keepdims=True)
    P = np.divide(e, Z, out=np.zeros_like(e), where=Z > 0)
    O = P @ np.asarray(V, np.float64)
    with np.errstate(divide="ignore"):
        lse = m[:, 0] + np.log(Z[:, 0])
    lse[empty] = -np.inf
    return O, lse, P


def entropy_from_probs(P):
    """Shannon entropy -sum_j p_ij ln p_ij of each row (0 ln 0 = 0)."""
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(P > 0, P * np.log(P), 0.0)
    return -t.sum(axis=1)


def entropy_from_scores(s):
    """H_i = ln Z_i - (sum_j e^{s_ij} s_ij) / Z_i, Z_i = sum_j e^{s_ij}; the
    exponentials are taken relative to the row maximum, which leaves H
    unchanged."""
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    Z = e.sum(axis=1)
    return np.log(Z) - (e * (s - m)).sum(axis=1) / Z


def dense_attention_entropy(Q, K, V, scale):
    """Per head: O, H, LSE of full softmax attention, with H from the
    probabilities.  Q, K, V: [heads, N, d] (any float type)."""
    heads = Q.shape[0]
    O = np.empty(Q.shape, np.float64)
    H = np.empty(Q.shape[:2], np.float64)
    L = np.empty(Q.shape[:2], np.float64)
    for h in range(heads):
        O[h], L[h], P = softmax_attention(Q[h], K[h], V[h], scale)
        H[h] = entropy_from_probs(P)
    return O, H, L


def attention_rows(Qh, Kh, Vh, scale, rows, key_mask_rows=None):
    """Attention and entropy of selected query rows of one head (for large
    problems where the full score matrix does not fit)."""
    O, L, P = softmax_attention(np.asarray(Qh)[rows], Kh, Vh, scale, key_mask_rows)
    return O, entropy_from_probs(P), L


# ---------------------------------------------------------------------------
# entropy -> budget -> radius  (§2 Insight I, Insight II; reading R4)
# ---------------------------------------------------------------------------


def budget(H, tau, N):
    """B_i = tau * exp(H_i) / N  (§2 Insight I)."""
    return tau * np.exp(np.asarray(H, np.float64)) / N


def phi(delta, gamma):
    """Temporal decay phi(delta) = exp(-gamma * delta)  (§2 Insight II)."""
    return np.exp(-gamma * np.asarray(delta, np.float64))


def frame_energy(F, gamma):
    """S[t] = sum over existing key frames t' of phi(|t' - t|)^2."""
    S = np.zeros(F)
    for t in range(F):
        for tp in range(F):
            S[t] += phi(abs(tp - t), gamma) ** 2
    return S


def radius(H, frame_of_query, tau, gamma, F, N):
    """Base radius r_i = sqrt(K_i / (pi * S[t_i])) with K_i = B_i * N."""
    K = budget(H, tau, N) * N
    S = frame_energy(F, gamma)
    return np.sqrt(K / (math.pi * S[np.asarray(frame_of_query)]))


# ---------------------------------------------------------------------------
# mask variants: shared budget, 1D distance, Radial's static window
# (§4 ablation study; Radial abstract; readings R12-R14)
# ---------------------------------------------------------------------------


def shared_budget_tokens(H, tau):
    """K_h = mean over the queries of head h of tau * exp(H_i)  (R12).
    H: [heads, N]; returns [heads]."""
    return np.mean(tau * np.exp(np.asarray(H, np.float64)), axis=1)


def frame_length(F, gamma):
    """L[t] = sum over existing key frames t' of phi(|t' - t|)  (R13)."""
    L = np.zeros(F)
    for t in range(F):
        for tp in range(F):
            L[t] += phi(abs(tp - t), gamma)
    return L


def radius_variant(H, frame_of_query, tau, gamma, F, budget="entropy", metric="disk"):
    """Base radii [heads, N] of the budget source ("entropy": K_i = tau *
    exp(H_i); "shared": K_h of R12 for every query of head h) and the distance
    ("disk": r = sqrt(K / (pi S[t])), R4; "line": r = K / (2 L[t]), R13)."""
    H = np.asarray(H, np.float64)
    if budget == "entropy":
        K = tau * np.exp(H)
    elif budget == "shared":
        K = np.repeat(shared_budget_tokens(H, tau)[:, None], H.shape[1], axis=1)
    else:
        raise ValueError(budget)
    t = np.asarray(frame_of_query)
    if metric == "disk":
        return np.sqrt(K / (math.pi * frame_energy(F, gamma)[t]))
    if metric == "line":
        return K / (2.0 * frame_length(F, gamma)[t])
    raise ValueError(metric)


def radial_band(delta):
    """b = floor(log2(delta + 1)) for integers delta >= 0."""
    return np.array([int(dl + 1).bit_length() - 1 for dl in np.ravel(delta)], dtype=np.int64)


def radial_phi(F, metric="disk"):
    """Radial's window factor per temporal distance (R14): 2^(-b/2) for the
    disk, 2^(-b) for the 1D distance, b = floor(log2(delta + 1))."""
    b = radial_band(np.arange(F)).astype(np.float64)
    return 2.0 ** (-b / 2.0) if metric == "disk" else 2.0 ** (-b)


# ---------------------------------------------------------------------------
# token mask, block votes, block mask, CSR  (§2 pipeline, fused mask kernel;
# readings R5, R6, R13)
# ---------------------------------------------------------------------------


def token_mask(r32, phi32, cq, ck, metric="disk", W=None):
    """M[i, j] = 1 when key j lies in query i's support in its frame.

    r32: float32 [Nq] base radii; phi32: float32 [F] decay table indexed by
    |t_j - t_i|; cq, ck: int [Nq, 3] / [Nk, 3] (x, y, t).  The threshold is
    R2 = fl32(fl32(r * phi)^2); +inf or NaN radii keep every key.  metric
    "disk": squared distance dx^2 + dy^2; "line" (R13): (n_j - n_i)^2 with the
    in-frame raster index n = y * W + x."""
    r32 = np.asarray(r32, np.float32)
    phi32 = np.asarray(phi32, np.float32)
    if metric == "disk":
        dx = cq[:, None, 0] - ck[None, :, 0]
        dy = cq[:, None, 1] - ck[None, :, 1]
        d2 = (dx * dx + dy * dy).astype(np.float64)
    elif metric == "line":
        dn = (cq[:, None, 1] * W + cq[:, None, 0]) - (ck[None, :, 1] * W + ck[None, :, 0])
        d2 = (dn * dn).astype(np.float64)
    else:
        raise ValueError(metric)
    dt = np.abs(cq[:, None, 2] - ck[None, :, 2])
    R = (r32[:, None] * phi32[dt]).astype(np.float32)      # fp32 product
    R2 = (R * R).astype(np.float32)                         # fp32 square
    keep_all = ~np.isfinite(r32)
    with np.errstate(invalid="ignore"):
        inside = d2 <= R2.astype(np.float64)
    return inside | keep_all[:, None]


def block_votes(M, Bq, Bk):
    """votes[qb, kb] = number of (query, key) pairs inside the support with
    the query in block qb and the key in block kb; blocks are consecutive runs
    of Bq (Bk) positions, the last one possibly shorter."""
    Nq, Nk = M.shape
    nqb, nkb = -(-Nq // Bq), -(-Nk // Bk)
    votes = np.zeros((nqb, nkb), dtype=np.int64)
    for qb in range(nqb):
        rows = M[qb * Bq:(qb + 1) * Bq]
        for kb in range(nkb):
            votes[qb, kb] = int(rows[:, kb * Bk:(kb + 1) * Bk].sum())
    return votes


def block_mask_from_votes(votes, vote_threshold):
    """A block pair is kept when its votes reach the threshold."""
    return votes >= vote_threshold


def block_mask(r32, phi32, coords_tm, Bq, Bk, vote_threshold, qblocks=None, metric="disk",
               W=None):
    """Kept-block mask of one head, bool [len(qblocks), nkb], brute force over
    every token pair.  coords_tm: (x, y, t) of each tile-major position."""
    N = coords_tm.shape[0]
    nqb = -(-N // Bq)
    if qblocks is None:
        qblocks = range(nqb)
    nkb = -(-N // Bk)
    out = np.zeros((len(qblocks), nkb), dtype=bool)
    for row, qb in enumerate(qblocks):
        q = slice(qb * Bq, min(N, (qb + 1) * Bq))
        M = token_mask(np.asarray(r32)[q], phi32, coords_tm[q], coords_tm, metric, W)
        out[row] = block_mask_from_votes(block_votes(M, Bq, Bk)[0], vote_threshold)
    return out


def to_csr(mask):
    """CSR of a kept-block mask bool [heads, nqb, nkb]: row_ptr int64
    [heads, nqb + 1] holds offsets into one col_idx array shared by all heads
    (row (h, qb) is col_idx[row_ptr[h, qb] : row_ptr[h, qb + 1]]); col_idx lists
    the kept key blocks of each row in ascending order."""
    heads, nqb, nkb = mask.shape
    row_ptr = np.zeros((heads, nqb + 1), dtype=np.int64)
    cols = []
    total = 0
    for h in range(heads):
        for qb in range(nqb):
            row_ptr[h, qb] = total
            kept = [kb for kb in range(nkb) if mask[h, qb, kb]]
            cols.extend(kept)
            total += len(kept)
        row_ptr[h, nqb] = total
    return row_ptr, np.array(cols, dtype=np.int64)


def key_mask_from_blocks(bm_rows, qrows, Bq, Bk, Nk):
    """Token-level key mask implied by a block mask: query i may see key j
    iff block (i // Bq, j // Bk) is kept.  bm_rows is indexed by q-block."""
    qb = np.asarray(qrows) // Bq
    kb = np.arange(Nk) // Bk
    return bm_rows[qb][:, kb]


def sparse_attention(Q, K, V, mask, Bq, Bk, scale):
    """Exact softmax attention over every token of the kept key blocks
    (reading R7).  Q, K, V: [heads, N, d] in tile-major order; mask bool
    [heads, nqb, nkb].  Returns (O, LSE)."""
    heads, N, _ = Q.shape
    O = np.empty(Q.shape, np.float64)
    L = np.empty((heads, N), np.float64)
    for h in range(heads):
        km = key_mask_from_blocks(mask[h], np.arange(N), Bq, Bk, N)
        O[h], L[h], _ = softmax_attention(Q[h], K[h], V[h], scale, km)
    return O, L


def sparse_attention_rows(Qh, Kh, Vh, mask_h, Bq, Bk, scale, rows):
    """Sparse attention of selected query rows of one head."""
    km = key_mask_from_blocks(mask_h, rows, Bq, Bk, Kh.shape[0])
    O, L, _ = softmax_attention(np.asarray(Qh)[rows], Kh, Vh, scale, km)
    return O, L


def kept_fraction(mask):
    return float(np.mean(mask))


# ---------------------------------------------------------------------------
# cross-step reuse  (§2 "TRA pipeline", cross-step reuse; reading R15)
# ---------------------------------------------------------------------------


def reuse_plan(steps, warmup, refresh_every, refresh):
    """Kind of each denoising step: "dense" (dense output, entropy and mask
    from this step), "sparse" (sparse output over the current mask) or
    "sparse+entropy" (sparse output, then entropy and mask from this step)."""
    plan = []
    for k in range(steps):
        if k < warmup:
            plan.append("dense")
        elif refresh_every > 0 and (k - warmup + 1) % refresh_every == 0:
            plan.append("dense" if refresh == "dense" else "sparse+entropy")
        else:
            plan.append("sparse")
    return plan


def mask_from_entropy(H, coords_tm, tau, gamma, F, Bq, Bk, vote):
    """Kept-block mask [heads, nqb, nkb] of entropies H [heads, N]: radius by
    R4 rounded to fp32, phi rounded to fp32, brute-force block votes."""
    N = coords_tm.shape[0]
    phi32 = phi(np.arange(F), gamma).astype(np.float32)
    masks = []
    for h in range(H.shape[0]):
        r32 = radius(H[h], coords_tm[:, 2], tau, gamma, F, N).astype(np.float32)
        masks.append(block_mask(r32, phi32, coords_tm, Bq, Bk, vote))
    return np.stack(masks)


def reuse_run(steps_qkv, coords_tm, F, tau, gamma, Bq, Bk, vote, plan, scale):
    """Outputs of a denoising schedule.  steps_qkv: per step (Q, K, V) [heads,
    N, d] in tile-major order.  Returns (outputs, masks used, entropies of
    the refresh steps)."""
    outputs, used, refreshed = [], [], {}
    mask = None
    for k, ((Q, K, V), kind) in enumerate(zip(steps_qkv, plan)):
        if kind == "dense":
            O, H, _ = dense_attention_entropy(Q, K, V, scale)
            used.append(None)
        else:
            O, _ = sparse_attention(Q, K, V, mask, Bq, Bk, scale)
            used.append(mask)
            if kind == "sparse+entropy":
                _, H, _ = dense_attention_entropy(Q, K, V, scale)
        if kind != "sparse":
            refreshed[k] = H
            mask = mask_from_entropy(H, coords_tm, tau, gamma, F, Bq, Bk, vote)
        outputs.append(O)
    return outputs, used, refreshed


# ---------------------------------------------------------------------------
# FP8 (E4M3) scores  (reading R16)
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0


def round_e4m3(x):
    """Nearest OCP FP8 E4M3 value (1 sign bit, 4 exponent bits with bias 7, 3
    mantissa bits, no infinities, largest finite 448), ties to even; finite
    values beyond +-448 saturate.  The rounding itself is torch's float8_e4m3fn
    conversion (a library primitive, pinned to the format in the tests)."""
    import torch
    x = np.clip(np.asarray(x, np.float32), -E4M3_MAX, E4M3_MAX)
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.float8_e4m3fn).to(
        torch.float32).numpy().astype(np.float64)


def quantize_e4m3_blocks(X, block):
    """Per head and per block of `block` consecutive rows of X [heads, N, d]:
    scale = fl32(amax / 448) (1 when the block is all zero) and codes =
    E4M3(fl32(x / scale)).  Returns (codes [heads, N, d] as float64,
    scales [heads, nblocks] float32)."""
    X32 = np.asarray(X, np.float32)
    heads, N, _ = X32.shape
    nb = -(-N // block)
    codes = np.empty(X32.shape, np.float64)
    scales = np.empty((heads, nb), np.float32)
    for h in range(heads):
        for b in range(nb):
            blk = X32[h, b * block:(b + 1) * block]
            amax = np.float32(np.max(np.abs(blk))) if blk.size else np.float32(0)
            sc = np.float32(amax / np.float32(E4M3_MAX)) if amax > 0 else np.float32(1.0)
            scales[h, b] = sc
            codes[h, b * block:(b + 1) * block] = round_e4m3((blk / sc).astype(np.float32))
    return codes, scales


def sparse_attention_fp8qk(Q8, qs, K8, ks, V, mask, Bq, Bk, scale, rows=None, head=None):
    """Exact softmax over the kept blocks with scores
    s_ij = scale * qs[i // Bq] * ks[j // Bk] * (q8_i . k8_j).  Q8, K8: E4M3
    codes [heads, N, d] (float64), qs / ks: per-block scales; V as for
    sparse_attention.  With `head` and `rows`, only those rows of that head."""
    heads = range(Q8.shape[0]) if head is None else [head]
    outs, lses = [], []
    for h in heads:
        N = K8.shape[1]
        r = np.arange(Q8.shape[1]) if rows is None else np.asarray(rows)
        s = (Q8[h][r] @ K8[h].T) * (np.float64(scale) * qs[h][r // Bq].astype(np.float64)[:, None]
                                      * ks[h][np.arange(N) // Bk].astype(np.float64)[None, :])
        km = key_mask_from_blocks(mask[h], r, Bq, Bk, N)
        s = np.where(km, s, -np.inf)
        m = np.max(s, axis=1, keepdims=True)
        ok = np.isfinite(m)
        e = np.where(km & ok, np.exp(s - np.where(ok, m, 0.0)), 0.0)
        Z = e.sum(axis=1, keepdims=True)
        O = np.where(Z > 0, (e @ np.asarray(V[h], np.float64)) / np.where(Z > 0, Z, 1.0), 0.0)
        L = np.where(Z[:, 0] > 0, np.log(np.where(Z[:, 0] > 0, Z[:, 0], 1.0)) + np.where(ok[:, 0], m[:, 0], 0.0), -np.inf)
        outs.append(O)
        lses.append(L)
    return (np.stack(outs), np.stack(lses)) if head is None else (outs[0], lses[0])
