"""Scalar brute-force Sol attention for tiny inputs (test infrastructure only).

An independent second statement of the same forward pass as ``sol_ref``,
written with plain Python loops and ``math`` so that it shares no code path
(no NumPy reductions, no einsum) with the oracle it checks.  It is meant for
N <= 256, D <= 16.  Definitions follow the Star7 README ("MiniMax H3
Activation Chunk & Attention Acceleration", section 工作原理 > Sol) for the
exact + centroid split and the KV sink, the thakicloud blog ("이 기술은
무엇인가") for the mean + tau*std threshold, and the Spark-H3 news page
(Spark-Reweight bullet) for the log-mass bias.

Inputs are nested lists or arrays indexed [b][n][h][d].
"""
from __future__ import annotations

import math


def _mean_rows(X, b, h, lo, hi, D):
    acc = [0.0] * D
    for t in range(lo, hi):
        for c in range(D):
            acc[c] += float(X[b][t][h][c])
    return [a / (hi - lo) for a in acc]


def _dot(x, y):
    s = 0.0
    for a, c in zip(x, y):
        s += a * c
    return s


def forward(Q, K, V, B, N, H, D, tau, prefix, bq, bk, scale=None, lmb=False, rw=False, topk=None,
            compressed=False):
    """Return (O[b][n][h][d], sel[b][h][i][j]) computed row by row.

    ``rw`` replaces the centroid key/value of every block by the anchor-softmax
    weighted summaries (and implies the log-mass bias, taken against them).
    ``topk`` (an int k) routes each query block to its k highest-scoring key
    blocks (equal scores: lower index first), keeps every key block for query
    blocks holding prefix rows, and drops unselected blocks; with
    ``compressed`` it also keeps the sink blocks and gives unselected blocks
    their centroid terms (the bias options apply).
    """
    s = scale if scale else 1.0 / math.sqrt(D)
    nqb = (N + bq - 1) // bq
    nkb = (N + bk - 1) // bk
    n_sink = (prefix + bk - 1) // bk
    n_dense = (prefix + bq - 1) // bq
    O = [[[[0.0] * D for _ in range(H)] for _ in range(N)] for _ in range(B)]
    SEL = [[None] * H for _ in range(B)]
    for b in range(B):
        for h in range(H):
            kspan = [(j * bk, min(N, (j + 1) * bk)) for j in range(nkb)]
            qspan = [(i * bq, min(N, (i + 1) * bq)) for i in range(nqb)]
            kbar = [_mean_rows(K, b, h, lo, hi, D) for lo, hi in kspan]
            vbar = [_mean_rows(V, b, h, lo, hi, D) for lo, hi in kspan]
            # anchor = mean of the video queries (all rows when there is no video part)
            alo = prefix if prefix < N else 0
            a = _mean_rows(Q, b, h, alo, N, D)
            bias = []
            kc, vc = list(kbar), list(vbar)        # centroid key/value seen by queries
            for j, (lo, hi) in enumerate(kspan):
                if not (lmb or rw):
                    bias.append(0.0)
                    continue
                total = 0.0
                wk, wv = [0.0] * D, [0.0] * D
                for t in range(lo, hi):
                    kt = [float(x) for x in K[b][t][h]]
                    e = math.exp(s * _dot(a, kt))
                    total += e
                    for c in range(D):
                        wk[c] += e * kt[c]
                        wv[c] += e * float(V[b][t][h][c])
                if rw:
                    kc[j] = [x / total for x in wk]
                    vc[j] = [x / total for x in wv]
                bias.append(math.log(total / (hi - lo)) - s * _dot(a, kc[j]))
            sel_bh = []
            for i, (qlo, qhi) in enumerate(qspan):
                qbar = _mean_rows(Q, b, h, qlo, qhi, D)
                sc = [s * _dot(qbar, kbar[j]) for j in range(nkb)]
                mu = sum(sc) / nkb
                var = sum((x - mu) ** 2 for x in sc) / nkb
                thr = -math.inf if tau == -math.inf else mu + tau * math.sqrt(var)
                row = []
                if topk is None:
                    for j in range(nkb):
                        row.append(i < n_dense or j < n_sink or sc[j] > thr)
                else:   # repeated selection of the best remaining block
                    row = [i < n_dense or (compressed and j < n_sink) for j in range(nkb)]
                    left = list(range(nkb))
                    for _ in range(topk):
                        best = left[0]
                        for jj in left[1:]:
                            if sc[jj] > sc[best]:
                                best = jj
                        row[best] = True
                        left.remove(best)
                sel_bh.append(row)
                for r in range(qlo, qhi):
                    q = [float(x) for x in Q[b][r][h]]
                    logits, vals = [], []
                    for j, (lo, hi) in enumerate(kspan):
                        if row[j]:
                            for t in range(lo, hi):
                                logits.append(s * _dot(q, [float(x) for x in K[b][t][h]]))
                                vals.append([float(x) for x in V[b][t][h]])
                        elif topk is None or compressed:
                            logits.append(s * _dot(q, kc[j]) + math.log(hi - lo) + bias[j])
                            vals.append(vc[j])
                    m = max(logits)
                    w = [math.exp(x - m) for x in logits]
                    z = sum(w)
                    for c in range(D):
                        O[b][r][h][c] = sum(wi * vi[c] for wi, vi in zip(w, vals)) / z
            SEL[b][h] = sel_bh
    return O, SEL


# ---- adaptive partition (Spark-H3 news page, Spark-Reblock bullet), scalar form ----------------
def _cholesky(M, D):
    """Textbook Cholesky-Banachiewicz: lower L with L L^T = M."""
    L = [[0.0] * D for _ in range(D)]
    for i in range(D):
        for j in range(i + 1):
            s = M[i][j]
            for c in range(j):
                s -= L[i][c] * L[j][c]
            L[i][j] = math.sqrt(s) if i == j else s / L[j][j]
    return L


def reblock_perm(Q, K, B, N, H, D, prefix, bs=64, iters=4):
    """perm[b][h][pos] of the size-balanced principal-axis bisection of the keys
    whitened by the video queries' second moment (ridge 1e-4 * trace / D).

    Level by level over explicit group lists (the oracle recurses); the same
    reading: split along the covariance's principal axis by ``iters`` power
    steps from the group's first member minus its mean, the left part takes
    bs * ceil(ceil(n / bs) / 2) lowest projections (ties to the lower row),
    groups keep ascending row order, prefix blocks stay in place.
    """
    n_fix = min(N, bs * (-(-prefix // bs)))
    perm = [[list(range(N)) for _ in range(H)] for _ in range(B)]
    if n_fix == N:
        return perm
    lo = prefix if prefix < N else 0
    for b in range(B):
        for h in range(H):
            M = [[0.0] * D for _ in range(D)]
            for t in range(lo, N):
                q = [float(Q[b][t][h][c]) for c in range(D)]
                for i in range(D):
                    for j in range(D):
                        M[i][j] += q[i] * q[j]
            n = N - lo
            tr = 0.0
            for i in range(D):
                for j in range(D):
                    M[i][j] /= n
                tr += M[i][i]
            ridge = 1e-4 * tr / D if tr > 0 else 1.0
            for i in range(D):
                M[i][i] += ridge
            L = _cholesky(M, D)
            Y = []
            for t in range(n_fix, N):
                k = [float(K[b][t][h][c]) for c in range(D)]
                x = [sum(k[r] * L[r][c] for r in range(D)) for c in range(D)]   # row k times L
                nx = math.sqrt(_dot(x, x))
                Y.append([v / nx for v in x] if nx > 0 else [0.0] * D)
            groups = [list(range(N - n_fix))]
            while any(len(g) > bs for g in groups):
                nxt = []
                for g in groups:
                    if len(g) <= bs:
                        nxt.append(g)
                        continue
                    m = len(g)
                    left = bs * (-(-(-(-m // bs)) // 2))
                    mean = [sum(Y[t][c] for t in g) / m for c in range(D)]
                    C = [[Y[t][c] - mean[c] for c in range(D)] for t in g]
                    w = list(C[0])
                    nw = math.sqrt(_dot(w, w))
                    w = [v / nw for v in w] if nw > 0 else [1.0] + [0.0] * (D - 1)
                    for _ in range(iters):
                        proj = [_dot(c, w) for c in C]
                        z = [sum(C[r][c] * proj[r] for r in range(m)) for c in range(D)]
                        nz = math.sqrt(_dot(z, z))
                        if nz == 0:
                            break
                        w = [v / nz for v in z]
                    ranked = sorted(range(m), key=lambda r: (_dot(Y[g[r]], w), g[r]))
                    in_left = set(ranked[:left])
                    nxt.append([g[r] for r in range(m) if r in in_left])
                    nxt.append([g[r] for r in range(m) if r not in in_left])
                groups = nxt
            perm[b][h] = list(range(n_fix)) + [n_fix + t for g in groups for t in g]
    return perm
