"""fp64 CPU oracle for Sol block-sparse attention (test infrastructure only).

This module is test infrastructure.  Only the tests, the smoke check and the
bench's CPU-baseline leg may import it; the product path never does, and it
shares no code with the CUDA kernels.

What it computes, step by step, in the order the sources describe it:

  1. pool     -- mean of each block of consecutive rows of Q, K, V ("K/V
                 centroids"; Star7 README "MiniMax H3 Activation Chunk &
                 Attention Acceleration", section 工作原理 > Sol; Spark-H3 news
                 page, "Spark-Attn이 바꾸는 것", Spark-Reweight bullet, which calls
                 them mean-pooled key/value summaries).
  2. scores   -- S[i, j] = s * qbar_i . kbar_j, the block score of every
                 query-block / key-block pair (thakicloud "MiniMax-H3 ComfyUI
                 accel stack", section "이 기술은 무엇인가": tau is measured in
                 standard deviations above the mean of the block scores).
  3. route    -- a key block is exact iff its score is above the row's
                 mean + tau * std (same section; Star7 README, 工作原理 > Sol:
                 Q64/K64 threshold routing with tau = 1.0); key blocks that hold
                 prefix rows are an always-exact KV sink, and query blocks that
                 hold prefix rows attend densely (Star7 README, 工作原理 > Sol,
                 last paragraph; aikraft.ru "ComfyUI Sol-Attn", section
                 "Нововведения версии 2.0", exact_kv / exact_kv_and_rows).
  4. attention -- selected blocks contribute their rows exactly; each
                 unselected block contributes one centroid term (logit
                 s*q.kbar_j + log n_j, value vbar_j) merged into the same
                 softmax (Star7 README, 工作原理 > Sol).
  5. log-mass bias (optional) -- mean pooling gives exp(E[x]) instead of
                 E[exp(x)]; a per-block bias restores the lost mass, scored
                 against one anchor per head, the mean video query (Spark-H3
                 news page, Spark-Reweight bullet and the compressed-branch
                 figure caption).
  6. weighted summaries (optional, implies 5) -- the compressed branch's
                 mean-pooled key/value summaries are replaced by weighted ones
                 (same bullet).  Reading: within key block j the weights are
                 the anchor's own softmax over the block's rows,
                 w_t = exp(s*a.k_t) / sum_u exp(s*a.k_u); the summaries are
                 sum_t w_t k_t and sum_t w_t v_t, and the bias is taken
                 against the weighted key.  A query equal to the anchor then
                 gets the block's exact contribution, mass and value alike.
                 Routing still scores the mean-pooled kbar.
  7. Top-K routing (the SLA variant of the same kernels; Star7 README,
                 section 工作原理 > SLA: Q=128 / K=64 dynamic Top-K block
                 routing keeping about 15% of the key blocks, fp32 online
                 softmax, full attention for the audio query range; Spark-H3
                 news page, workflow paragraph: topk_ratio 0.2 / 0.1).  Each
                 128-row query block keeps the k = round(ratio * n_kb) key
                 blocks with the largest scores s * qbar_i . kbar_j; query
                 blocks holding prefix rows keep every key block; unselected
                 blocks contribute nothing (no centroid term).
  8. Top-K with the compressed branch (the Spark-H3 configuration:
                 topk_mode=topk_ratio, the exact branch on the top-ranked
                 blocks and the compressed branch on the rest; Spark-H3 news
                 page, "Spark-Attn이 바꾸는 것" and the workflow paragraph):
                 steps 1-6 with the threshold test of step 3 replaced by
                 membership in the row's k highest scores; 64-row query
                 blocks, the KV sink and the dense prefix rows as in step 3.
  9. adaptive partition (optional; Spark-H3 news page, Spark-Reblock
                 bullet: fixed tiles replaced by an adaptive partition whose
                 similarity is the cosine under the Mahalanobis metric of the
                 opposite side's second moment, split hierarchically until
                 every leaf has the block size, in O(N log N); workflow
                 paragraph: reblock_layout=q_reuse_k, queries take the keys'
                 partition).  Reading: per (b, h) the keys are whitened by the
                 Cholesky factor of the video queries' second moment
                 M = mean q q^T (plus a ridge of 1e-4 * trace(M) / D), so the
                 plain cosine of the whitened unit vectors is the Mahalanobis
                 cosine; a group splits along its principal axis (REBLOCK_ITERS
                 power-iteration steps on its covariance, started from its
                 first member minus its mean) at the size-balanced median:
                 the left part takes 64 * ceil(ceil(n / 64) / 2) rows, the
                 lowest projections, ties to the lower row index; every group
                 keeps its rows in ascending original order, so the partial
                 leaf is last and each leaf lists its rows ascending.  Blocks
                 holding prefix rows keep their place.  Q, K and V are
                 permuted per head, steps 1-8 run on the permuted rows, and O
                 is permuted back.
 10. INT8 QK with per-block residual keys (optional; thakicloud "MiniMax-H3
                 ComfyUI accel stack", section 실제 실험 결과, closing accuracy
                 paragraph: only each key block's residual from its mean is
                 quantized to INT8, the mean term stays bf16; relative L2 error
                 0.008 against the exact path, 0.030 when the whole key is
                 quantized).  Reading: k_bar16_j = the block mean (an fp32 sum
                 in row order times the fp32 reciprocal of the count, the
                 kernel's precision, since its rounding decides integer codes)
                 rounded to bf16; r_t = k_t - k_bar16_j; one symmetric scale per key block,
                 sigma_j = max |r| / 127, codes rint(r * (1 / sigma_j)) in [-127, 127];
                 each query row quantized the same way with its own scale
                 (the INT8 product needs an INT8 left operand); every exact
                 logit becomes s * (q . k_bar16_j + sigma_q sigma_j (q_code .
                 r_code)), with q . k_bar16_j taken from the unquantized bf16
                 query.  Scales and codes are decided in fp32 (the kernel's
                 precision): x times the fp32 reciprocal of sigma, rounded to
                 the nearest integer, ties to even.  Centroid terms and routing
                 are unchanged.

Readings where the sources are silent (each is listed in the design notes):
blocks are consecutive rows tiling the whole packed sequence from row 0 (the
only partial block is the last); the standard deviation is the population
one over all key blocks; the comparison is strict; a key block is a sink iff
it holds a prefix row and a query block is dense iff it holds a prefix row;
log n_j and the centroid use the block's valid row count; the bias is
bias_j = logsumexp_t(s*a.k_t) - log n_j - s*a.kbar_j and does not change
routing; tau = -inf selects every block.  Top-K: equal scores are ranked by
the lower key-block index; ratio is the float32 the ABI carries and k =
floor(ratio * n_kb + 0.5) (nearest, halves up) is evaluated in double from
it, clamped to [1, n_kb]; no key block
is forced (the SLA passage names full attention for the prefix query rows
only); the dense query blocks are the 128-row ones holding prefix rows.

Layouts: Q, K, V, O are float64 arrays [B, N, H, D] (BTHD); per-head block
quantities are [B, H, n_blocks, ...].
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np


def n_blocks(N: int, bs: int) -> int:
    """Number of blocks of ``bs`` consecutive rows covering N rows."""
    return -(-N // bs)


def block_rows(N: int, bs: int) -> np.ndarray:
    """Valid row count of every block (bs, or the tail count for the last)."""
    nb = n_blocks(N, bs)
    starts = np.arange(nb) * bs
    return np.minimum(starts + bs, N) - starts


def pool(X: np.ndarray, bs: int) -> np.ndarray:
    """Block means: X [B, N, H, D] -> [B, H, n_blocks, D] (step 1)."""
    B, N, H, D = X.shape
    nb = n_blocks(N, bs)
    out = np.zeros((B, H, nb, D))
    for j in range(nb):
        lo, hi = j * bs, min((j + 1) * bs, N)
        out[:, :, j, :] = X[:, lo:hi, :, :].mean(axis=1)
    return out


def scores(qbar: np.ndarray, kbar: np.ndarray, scale: float) -> np.ndarray:
    """Block scores S[b, h, i, j] = scale * qbar_i . kbar_j (step 2)."""
    return scale * np.einsum("bhid,bhjd->bhij", qbar, kbar)


def thresholds(S: np.ndarray, tau: float) -> np.ndarray:
    """Row threshold mean + tau * std over all key blocks (population std)."""
    mu = S.mean(axis=-1)
    sd = np.sqrt(((S - mu[..., None]) ** 2).mean(axis=-1))
    if tau == -math.inf:
        return np.full_like(mu, -math.inf)
    return mu + tau * sd


def route(S: np.ndarray, tau: float, prefix: int, bq: int, bk: int) -> np.ndarray:
    """Exact-block mask sel[b, h, i, j] (step 3)."""
    thr = thresholds(S, tau)
    sel = S > thr[..., None]
    n_sink = n_blocks(prefix, bk)
    n_dense = n_blocks(prefix, bq)
    sel[..., :, :n_sink] = True
    sel[..., :n_dense, :] = True
    return sel


def topk_count(ratio: float, nkb: int) -> int:
    """Key blocks kept per query block by Top-K routing (step 7)."""
    return max(1, min(nkb, math.floor(float(np.float32(ratio)) * nkb + 0.5)))


def route_topk(S: np.ndarray, k: int, prefix: int, bq: int, bk: Optional[int] = None) -> np.ndarray:
    """Top-K mask (steps 7, 8): the k largest scores of each row, ties to the lower index;
    with ``bk`` the key blocks holding prefix rows are kept too (the KV sink of step 8)."""
    order = np.argsort(-S, axis=-1, kind="stable")
    sel = np.zeros(S.shape, bool)
    np.put_along_axis(sel, order[..., :k], True, axis=-1)
    if bk is not None:
        sel[..., :, :n_blocks(prefix, bk)] = True
    sel[..., :n_blocks(prefix, bq), :] = True
    return sel


def to_csr(sel: np.ndarray):
    """CSR of the mask over rows in (b, h, i) order, columns ascending."""
    rows = sel.reshape(-1, sel.shape[-1])
    counts = rows.sum(axis=1).astype(np.int64)
    row_ptr = np.zeros(rows.shape[0] + 1, np.int64)
    np.cumsum(counts, out=row_ptr[1:])
    col_idx = np.nonzero(rows)[1].astype(np.int64)   # row-major order, ascending per row
    return row_ptr, col_idx


def from_csr(row_ptr, col_idx, shape) -> np.ndarray:
    """Inverse of ``to_csr``: rebuild a boolean mask of ``shape`` [B, H, nqb, nkb]."""
    sel = np.zeros(shape, bool)
    flat = sel.reshape(-1, shape[-1])
    for r in range(flat.shape[0]):
        flat[r, col_idx[row_ptr[r]:row_ptr[r + 1]]] = True
    return sel


def anchor(Q: np.ndarray, prefix: int) -> np.ndarray:
    """Per-head anchor: mean of the video (non-prefix) query rows, [B, H, D]."""
    N = Q.shape[1]
    rows = Q[:, prefix:, :, :] if prefix < N else Q
    return rows.mean(axis=1)


def log_mass_bias(Q: np.ndarray, K: np.ndarray, kbar: np.ndarray, prefix: int,
                  scale: float, bk: int) -> np.ndarray:
    """bias[b, h, j] = log mean_t exp(s a.k_t) - s a.kbar_j over block j (step 5)."""
    B, N, H, D = K.shape
    a = anchor(Q, prefix)                                    # [B, H, D]
    logits = scale * np.einsum("bnhd,bhd->bhn", K, a)        # [B, H, N]
    nb = n_blocks(N, bk)
    bias = np.zeros((B, H, nb))
    for j in range(nb):
        lo, hi = j * bk, min((j + 1) * bk, N)
        x = logits[:, :, lo:hi]
        m = x.max(axis=-1, keepdims=True)
        lme = (m[..., 0] + np.log(np.exp(x - m).sum(axis=-1))) - math.log(hi - lo)
        bias[:, :, j] = lme - scale * np.einsum("bhd,bhd->bh", a, kbar[:, :, j, :])
    return bias


def reweighted_summaries(Q: np.ndarray, K: np.ndarray, V: np.ndarray, prefix: int,
                         scale: float, bk: int):
    """Anchor-weighted key/value summaries and their log-mass bias (step 6).

    Per (b, h) and key block j with rows t: w_t = softmax_t(s a.k_t),
    ktil_j = sum_t w_t k_t, vtil_j = sum_t w_t v_t,
    bias_j = logsumexp_t(s a.k_t) - log n_j - s a.ktil_j.
    Returns (ktil [B, H, nb, D], vtil [B, H, nb, D], bias [B, H, nb]).
    """
    B, N, H, D = K.shape
    a = anchor(Q, prefix)                                    # [B, H, D]
    logits = scale * np.einsum("bnhd,bhd->bhn", K, a)        # [B, H, N]
    nb = n_blocks(N, bk)
    ktil = np.zeros((B, H, nb, D))
    vtil = np.zeros((B, H, nb, D))
    bias = np.zeros((B, H, nb))
    for j in range(nb):
        lo, hi = j * bk, min((j + 1) * bk, N)
        x = logits[:, :, lo:hi]
        m = x.max(axis=-1, keepdims=True)
        e = np.exp(x - m)
        z = e.sum(axis=-1)                                   # [B, H]
        w = e / z[..., None]                                 # [B, H, n]
        ktil[:, :, j] = np.einsum("bhn,bnhd->bhd", w, K[:, lo:hi])
        vtil[:, :, j] = np.einsum("bhn,bnhd->bhd", w, V[:, lo:hi])
        lse = m[..., 0] + np.log(z)
        bias[:, :, j] = lse - math.log(hi - lo) - scale * np.einsum("bhd,bhd->bh", a, ktil[:, :, j])
    return ktil, vtil, bias


def int8_codes(X: np.ndarray, axis) -> tuple:
    """Symmetric INT8 codes of X with one scale per slice reduced over ``axis``
    (step 10): sigma = max |x| / 127 and code = rint(x * (1 / sigma)) (ties to
    even), all in fp32 with the reciprocal rounded to fp32 (the kernel's
    precision, which decides the integer); sigma = 0 gives zero codes.
    Returns (codes int64, sigma float64 with the reduced axes kept)."""
    x = np.asarray(X, dtype=np.float32)
    amax = np.max(np.abs(x), axis=axis, keepdims=True)
    sigma = (amax / np.float32(127.0)).astype(np.float32)
    inv = (np.float32(1.0) / np.where(sigma > 0, sigma, np.float32(1.0))).astype(np.float32)
    codes = np.where(sigma > 0, np.rint((x * inv).astype(np.float32)), np.float32(0.0))
    return np.clip(codes, -127, 127).astype(np.int64), sigma.astype(np.float64)


def mean_fp32(K: np.ndarray, bk: int) -> np.ndarray:
    """Block means as the kernels compute them: an fp32 sum over the block's rows
    in row order, times the fp32 reciprocal of the row count ([B, H, nkb, D])."""
    B, N, H, D = K.shape
    out = np.empty((B, H, n_blocks(N, bk), D), dtype=np.float32)
    for j in range(n_blocks(N, bk)):
        lo, hi = j * bk, min((j + 1) * bk, N)
        acc = np.cumsum(K[:, lo:hi].astype(np.float32), axis=1, dtype=np.float32)[:, -1]   # sequential fp32
        out[:, :, j] = acc * (np.float32(1.0) / np.float32(hi - lo))
    return out.astype(np.float64)


def int8_residual_keys(K: np.ndarray, bk: int) -> dict:
    """Per-block residual quantization of the keys (step 10): the block mean
    rounded to bf16 (``kmean16`` [B, H, nkb, D]), the residual codes
    (``kcode`` [B, N, H, D]) and one scale per key block (``ksig`` [B, H, nkb]).
    The mean is summed in fp32 in row order (the kernel's precision): its bf16
    rounding decides the residuals, hence integer codes."""
    B, N, H, D = K.shape
    kmean16 = bf16_round(mean_fp32(K, bk))
    kcode = np.zeros((B, N, H, D), dtype=np.int64)
    ksig = np.zeros((B, H, n_blocks(N, bk)))
    for j in range(n_blocks(N, bk)):
        lo, hi = j * bk, min((j + 1) * bk, N)
        # fp32 difference of two bf16 values (exact), [B, rows, H, D]
        r = K[:, lo:hi].astype(np.float32) - kmean16[:, :, j][:, None, :, :].astype(np.float32)
        c, sg = int8_codes(r, axis=(1, 3))
        kcode[:, lo:hi] = c
        ksig[:, :, j] = sg[:, 0, :, 0]
    return dict(kmean16=kmean16, kcode=kcode, ksig=ksig)


def int8_query_rows(Q: np.ndarray) -> dict:
    """Per-row INT8 codes of the queries (step 10): ``qcode`` [B, N, H, D],
    ``qsig`` [B, N, H]."""
    c, sg = int8_codes(Q, axis=3)
    return dict(qcode=c, qsig=sg[..., 0])


def int8_logits(Q: np.ndarray, z: dict, b: int, h: int, r: np.ndarray, key_rows: np.ndarray, bk: int,
                scale: float) -> np.ndarray:
    """Exact-branch logits of query rows ``r`` against key rows ``key_rows`` of
    (b, h) under step 10: s * (q . kmean16_j + sigma_q sigma_j (q_code . r_code))."""
    blk = key_rows // bk
    codes = (z["qcode"][b, r, h, :] @ z["kcode"][b, key_rows, h, :].T).astype(np.float64)
    return scale * (Q[b, r, h, :] @ z["kmean16"][b, h, blk, :].T
                    + z["qsig"][b, r, h][:, None] * z["ksig"][b, h, blk][None, :] * codes)


def bf16_round(X: np.ndarray) -> np.ndarray:
    """Round to the nearest bf16 value (ties to even), through fp32."""
    u = np.ascontiguousarray(X, dtype=np.float32).view(np.uint32)
    r = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)) << np.uint32(16)
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def attention(Q, K, V, sel, kbar, vbar, bias, scale: float, bq: int, bk: int,
              rows: Optional[dict] = None, centroids: bool = True, qk_int8: Optional[dict] = None):
    """Exact + centroid attention (step 4).

    For every query row r of block i (per b, h): logits are s*q_r.k_t for the
    rows t of selected key blocks, and s*q_r.kbar_j + log n_j + bias_j for each
    unselected key block j, with values v_t and vbar_j; the output is the
    softmax-weighted sum.  Returns (O [B, N, H, D], lse [B, H, N]) where lse is
    the natural-log normaliser.  ``rows`` optionally maps (b, h) to an array
    of query rows to compute; other rows are left NaN.  With ``centroids``
    False unselected blocks contribute nothing (Top-K routing, step 7).
    ``qk_int8`` (the union of int8_residual_keys and int8_query_rows) makes
    every exact logit the step-10 form s * (q . kmean16_j + sigma_q sigma_j
    (q_code . r_code_t)).
    """
    B, N, H, D = Q.shape
    nqb, nkb = sel.shape[-2], sel.shape[-1]
    nk = block_rows(N, bk)
    logn = np.log(nk.astype(np.float64))
    O = np.full((B, N, H, D), np.nan)
    lse = np.full((B, H, N), np.nan)
    for b in range(B):
        for h in range(H):
            want = None if rows is None else rows.get((b, h))
            if rows is not None and want is None:
                continue
            for i in range(nqb):
                lo, hi = i * bq, min((i + 1) * bq, N)
                r = np.arange(lo, hi)
                if want is not None:
                    r = np.intersect1d(r, want)
                    if r.size == 0:
                        continue
                s_j = sel[b, h, i]
                key_rows = np.concatenate([np.arange(j * bk, min((j + 1) * bk, N))
                                           for j in np.nonzero(s_j)[0]] or [np.zeros(0, int)])
                cent = np.nonzero(~s_j)[0] if centroids else np.zeros(0, int)
                q = Q[b, r, h, :]
                if qk_int8 is None:
                    exact = scale * q @ K[b, key_rows, h, :].T
                else:
                    exact = int8_logits(Q, qk_int8, b, h, r, key_rows, bk, scale)
                lg = np.concatenate([exact,
                                     scale * q @ kbar[b, h, cent, :].T
                                     + (logn[cent] + bias[b, h, cent])[None, :]], axis=1)
                vals = np.concatenate([V[b, key_rows, h, :], vbar[b, h, cent, :]], axis=0)
                m = lg.max(axis=1, keepdims=True)
                p = np.exp(lg - m)
                l = p.sum(axis=1, keepdims=True)
                O[b, r, h, :] = (p @ vals) / l
                lse[b, h, r] = (m + np.log(l))[:, 0]
    return O, lse


REBLOCK_ITERS = 4   # power-iteration steps per split (step 9)


def second_moment_whitener(Q: np.ndarray, prefix: int) -> np.ndarray:
    """Lower Cholesky factors L[b, h] of the video queries' second moment
    M = mean q q^T + 1e-4 * trace(M) / D * I (step 9), so that
    (k L) . (k' L) = k^T M k'."""
    B, N, H, D = Q.shape
    rows = Q[:, prefix:, :, :] if prefix < N else Q
    L = np.empty((B, H, D, D))
    for b in range(B):
        for h in range(H):
            X = rows[b, :, h, :]
            M = X.T @ X / X.shape[0]
            tr = np.trace(M)
            M = M + (1e-4 * tr / D if tr > 0 else 1.0) * np.eye(D)
            L[b, h] = np.linalg.cholesky(M)
    return L


def split_projections(Y: np.ndarray, members: np.ndarray, iters: int = REBLOCK_ITERS) -> np.ndarray:
    """Projections of one group's whitened unit vectors on its principal axis
    (step 9): the axis comes from ``iters`` power-iteration steps on the
    group's covariance, started from its first member minus its mean (e_0 if
    that is zero); ``members`` are ascending positions into Y."""
    X = Y[members]
    C = X - X.mean(axis=0)
    w = C[0].copy()
    nw = np.linalg.norm(w)
    if nw > 0:
        w /= nw
    else:
        w = np.zeros(Y.shape[1])
        w[0] = 1.0
    for _ in range(iters):
        z = C.T @ (C @ w)
        nz = np.linalg.norm(z)
        if nz == 0:
            break
        w = z / nz
    return X @ w


def split_left_count(n: int, bs: int = 64) -> int:
    """Rows of the left part of a group of n > bs rows: bs * ceil(ceil(n / bs) / 2)
    (the size-balanced split of step 9)."""
    return bs * (-(-(-(-n // bs)) // 2))


def _split_group(Y: np.ndarray, members: np.ndarray, bs: int, iters: int, leaves: list):
    """Recursive size-balanced principal-axis bisection (step 9); ``members``
    ascending positions into Y (the whitened unit vectors)."""
    n = len(members)
    if n <= bs:
        leaves.append(members)
        return
    left = split_left_count(n, bs)
    p = split_projections(Y, members, iters)
    order = np.lexsort((members, p))       # ascending projection, ties to the lower row
    go_left = np.zeros(n, dtype=bool)
    go_left[order[:left]] = True
    _split_group(Y, members[go_left], bs, iters, leaves)    # boolean selection keeps ascending order
    _split_group(Y, members[~go_left], bs, iters, leaves)


def whitened_unit_keys(K: np.ndarray, L: np.ndarray, n_fix: int) -> np.ndarray:
    """Y[b, h] = normalise(k_t L[b, h]) for the key rows t >= n_fix (step 9; a
    zero row stays zero), so that Y[t] . Y[u] is the Mahalanobis cosine."""
    B, N, H, D = K.shape
    Y = np.zeros((B, H, N - n_fix, D))
    for b in range(B):
        for h in range(H):
            Xw = K[b, n_fix:, h, :] @ L[b, h]
            nrm = np.linalg.norm(Xw, axis=1, keepdims=True)
            Y[b, h] = np.divide(Xw, nrm, out=np.zeros_like(Xw), where=nrm > 0)
    return Y


def reblock_partition(Q: np.ndarray, K: np.ndarray, prefix: int, bs: int = 64,
                      iters: int = REBLOCK_ITERS) -> np.ndarray:
    """perm[b, h, pos] = original row at position ``pos`` of the adaptive
    partition's order (step 9); blocks holding prefix rows stay in place."""
    B, N, H, D = K.shape
    n_fix = min(N, bs * n_blocks(prefix, bs))
    perm = np.tile(np.arange(N, dtype=np.int64), (B, H, 1))
    if N - n_fix == 0:
        return perm
    Y = whitened_unit_keys(K, second_moment_whitener(Q, prefix), n_fix)
    for b in range(B):
        for h in range(H):
            leaves: list = []
            _split_group(Y[b, h], np.arange(N - n_fix), bs, iters, leaves)
            perm[b, h, n_fix:] = n_fix + np.concatenate(leaves)
    return perm


def permute_rows(X: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """Xp[b, pos, h] = X[b, perm[b, h, pos], h] for X [B, N, H, ...]."""
    B, N, H = X.shape[:3]
    out = np.empty_like(X)
    for b in range(B):
        for h in range(H):
            out[b, :, h] = X[b, perm[b, h], h]
    return out


def unpermute_rows(Xp: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """Inverse of ``permute_rows``: X[b, perm[b, h, pos], h] = Xp[b, pos, h]."""
    B, N, H = Xp.shape[:3]
    out = np.empty_like(Xp)
    for b in range(B):
        for h in range(H):
            out[b, perm[b, h], h] = Xp[b, :, h]
    return out


def sol_forward(Q, K, V, tau: float = 1.0, prefix: int = 0, bq: int = 64, bk: int = 64,
                scale: Optional[float] = None, log_mass_bias_on: bool = False,
                mask_override: Optional[np.ndarray] = None, rows: Optional[dict] = None,
                reweight_on: bool = False, topk_ratio: Optional[float] = None, compressed: bool = False,
                reblock: bool = False, perm_override: Optional[np.ndarray] = None, qk_int8: bool = False):
    """The whole forward pass; returns a dict of every intermediate.

    ``qk_int8`` (step 10) computes every exact logit from INT8 query codes
    and INT8 per-block residual key codes plus the bf16 mean term.

    ``reweight_on`` (step 6) gives the centroid terms the anchor-weighted
    summaries ``kc``/``vc`` and their bias; otherwise ``kc``/``vc`` are the
    mean-pooled kbar/vbar.  ``topk_ratio`` selects Top-K routing (step 7)
    with query blocks of ``bq`` rows (128 in the SLA contract) and no
    centroid terms; tau and the bias options are then unused.  With
    ``compressed`` Top-K keeps the compressed branch (step 8): the sink, the
    centroid terms and the bias options work as under threshold routing.
    ``reblock`` (step 9) runs all of it on the rows permuted per head by the
    adaptive partition (``perm_override`` replaces the computed order) and
    returns O and the LSE in the original row order; the block
    intermediates, ``mask_override`` and ``rows`` refer to permuted rows.
    """
    if reblock:
        perm = reblock_partition(Q, K, prefix, bk) if perm_override is None else perm_override
        r = sol_forward(permute_rows(Q, perm), permute_rows(K, perm), permute_rows(V, perm), tau, prefix,
                        bq, bk, scale, log_mass_bias_on, mask_override, rows, reweight_on, topk_ratio,
                        compressed, qk_int8=qk_int8)
        r["O_permuted"], r["perm"] = r["O"], perm
        r["O"] = unpermute_rows(r["O"], perm)
        lse = r["lse"]   # [B, H, N]
        r["lse"] = np.stack([np.stack([lse[b, h][np.argsort(perm[b, h])] for h in range(lse.shape[1])])
                             for b in range(lse.shape[0])])
        return r
    D = Q.shape[-1]
    s = (1.0 / math.sqrt(D)) if not scale else float(scale)
    qbar, kbar, vbar = pool(Q, bq), pool(K, bk), pool(V, bk)
    S = scores(qbar, kbar, s)
    z = {**int8_residual_keys(K, bk), **int8_query_rows(Q)} if qk_int8 else None
    if topk_ratio is not None and not compressed:
        k = topk_count(topk_ratio, kbar.shape[2])
        sel = route_topk(S, k, prefix, bq)
        bias = np.zeros(kbar.shape[:3])
        used = sel if mask_override is None else mask_override
        O, lse = attention(Q, K, V, used, kbar, vbar, bias, s, bq, bk, rows=rows, centroids=False, qk_int8=z)
        return dict(qbar=qbar, kbar=kbar, vbar=vbar, kc=kbar, vc=vbar, S=S, thr=None, sel=sel, k=k,
                    bias=bias, O=O, lse=lse, scale=s)
    k = None
    if topk_ratio is not None:   # step 8
        thr = None
        k = topk_count(topk_ratio, kbar.shape[2])
        sel = route_topk(S, k, prefix, bq, bk)
    else:
        thr = thresholds(S, tau)
        sel = route(S, tau, prefix, bq, bk)
    kc, vc = kbar, vbar
    if reweight_on:
        kc, vc, bias = reweighted_summaries(Q, K, V, prefix, s, bk)
    elif log_mass_bias_on:
        bias = log_mass_bias(Q, K, kbar, prefix, s, bk)
    else:
        bias = np.zeros(kbar.shape[:3])
    used = sel if mask_override is None else mask_override
    O, lse = attention(Q, K, V, used, kc, vc, bias, s, bq, bk, rows=rows, qk_int8=z)
    return dict(qbar=qbar, kbar=kbar, vbar=vbar, kc=kc, vc=vc, S=S, thr=thr, sel=sel, k=k,
                bias=bias, O=O, lse=lse, scale=s)
