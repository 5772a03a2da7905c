"""Pins of the oracle's adaptive partition (step 9 of oracle/sol_ref.py).

Spark-H3 news page, Spark-Reblock bullet: the fixed tiles are replaced by an
adaptive partition; similarity is the cosine under the Mahalanobis metric of
the opposite side's second moment; a hierarchical splitter divides groups
until every leaf has the block size.  The pins: an independent scalar
implementation (oracle/brute.py) on small inputs; the structure of the
permutation; a planted hierarchy that the splitter must recover leaf by leaf
and level by level; invariance of the partition under k -> k A, q -> q A^-T
(which keeps every score q.k, and only the Mahalanobis metric sees it so);
the split direction converging to the covariance's principal eigenvector
(numpy.linalg.eigh); and permutation equivariance of the whole forward pass
(all blocks exact => dense softmax attention).  The planted-mistake test at
the end shows that plausible bugs fail them.
"""
import math

import numpy as np
import pytest

from oracle import brute, sol_ref


def _planted(seed=0, D=16, levels=3, scales=(8.0, 4.0, 2.0), prefix=0, noise=0.01, H=1):
    """Keys of 2^levels clusters of 64 rows at random positions; cluster c's
    center is 10 e_D-1 + sum_l scales[l] * (+-1) e_l, bit l of c choosing the
    sign; queries isotropic.  Returns Q, K and the cluster id of every row."""
    rng = np.random.default_rng(seed)
    n_v = 64 * 2 ** levels
    n_fix = 64 * (-(-prefix // 64))
    N = n_fix + n_v
    cid = rng.permutation(np.repeat(np.arange(2 ** levels), 64))
    K = np.zeros((1, N, H, D))
    for h in range(H):
        K[0, :, h, :] = rng.standard_normal((N, D))
        for t in range(n_v):
            c = cid[t]
            center = np.zeros(D)
            center[D - 1] = 10.0
            for lvl in range(levels):
                center[lvl] = scales[lvl] * (1.0 if (c >> (levels - 1 - lvl)) & 1 else -1.0)
            K[0, n_fix + t, h, :] = center + noise * rng.standard_normal(D)
    Q = rng.standard_normal((1, N, H, D))
    return Q, K, cid, n_fix


def _structure_failures(perm, N, prefix, bs=64):
    """Count violations of: a permutation per head, prefix blocks in place,
    leaves of bs rows listed ascending, the partial leaf last."""
    bad = 0
    n_fix = min(N, bs * (-(-prefix // bs)))
    for row in perm.reshape(-1, N):
        bad += int(sorted(row.tolist()) != list(range(N)))
        bad += int(not np.array_equal(row[:n_fix], np.arange(n_fix)))
        for s in range(n_fix, N, bs):
            leaf = row[s:s + bs]
            bad += int(not np.all(np.diff(leaf) > 0))
    return bad


def _hierarchy_failures(seed=0, levels=3, prefix=0):
    """The planted clusters come out as leaves, in the order of their bits."""
    Q, K, cid, n_fix = _planted(seed, levels=levels, prefix=prefix)
    perm = sol_ref.reblock_partition(Q, K, prefix)[0, 0]
    leaves = [cid[perm[s:s + 64] - n_fix] for s in range(n_fix, len(perm), 64)]
    bad = sum(int(len(set(leaf.tolist())) != 1) for leaf in leaves)
    if bad:
        return bad
    order = [int(leaf[0]) for leaf in leaves]
    # each split separates by the largest remaining scale: the first half of the
    # leaves share the top bit, and so on down; which side comes first follows
    # the sign of the power iteration's start, so compare up to that
    for lvl in range(levels):
        span = len(order) >> lvl
        for g in range(0, len(order), span):
            bits = [(c >> (levels - 1 - lvl)) & 1 for c in order[g:g + span]]
            half = span // 2
            bad += int(len(set(bits[:half])) != 1 or len(set(bits[half:])) != 1 or bits[0] == bits[half])
    return bad


def _invariance_failures(seed=3):
    """k -> k A and q -> q A^-T keep every score; the partition must not change.
    A scales the planted axes so that a plain (Euclidean) cosine would rank them
    in the opposite order."""
    Q, K, _, _ = _planted(seed)
    D = K.shape[-1]
    rng = np.random.default_rng(seed + 1)
    d = np.ones(D)
    d[0], d[2] = 0.25, 4.0
    R, _ = np.linalg.qr(rng.standard_normal((D, D)))
    R[:, :3] = np.eye(D)[:, :3]            # keep the planted axes, mix the rest
    R, _ = np.linalg.qr(R)
    A = np.diag(d) @ R
    K2 = np.einsum("bnhd,de->bnhe", K, A)
    Q2 = np.einsum("bnhd,de->bnhe", Q, np.linalg.inv(A).T)
    assert np.allclose(np.einsum("bnhd,bmhd->bhnm", Q, K), np.einsum("bnhd,bmhd->bhnm", Q2, K2))
    return int(not np.array_equal(sol_ref.reblock_partition(Q, K, 0), sol_ref.reblock_partition(Q2, K2, 0)))


def _principal_axis_failures(seed=5):
    """With many power steps the first split is the principal-axis split."""
    rng = np.random.default_rng(seed)
    N, D = 256, 8
    Q = rng.standard_normal((1, N, 1, D))
    K = rng.standard_normal((1, N, 1, D)) * np.linspace(0.5, 2.0, D) + 1.0
    perm = sol_ref.reblock_partition(Q, K, 0, iters=300)[0, 0]
    L = sol_ref.second_moment_whitener(Q, 0)[0, 0]
    Y = K[0, :, 0, :] @ L
    Y /= np.linalg.norm(Y, axis=1, keepdims=True)
    C = Y - Y.mean(axis=0)
    _, vecs = np.linalg.eigh(C.T @ C)
    v = vecs[:, -1]
    if C[0] @ v < 0:
        v = -v
    left = set(np.lexsort((np.arange(N), Y @ v))[:128].tolist())
    return int(set(perm[:128].tolist()) != left)


def _brute_failures(seed=7):
    rng = np.random.default_rng(seed)
    bad = 0
    for N, D, P in [(300, 8, 0), (257, 8, 70), (200, 4, 0), (130, 8, 128), (64, 4, 0), (65, 4, 0)]:
        Q = rng.standard_normal((1, N, 2, D))
        K = rng.standard_normal((1, N, 2, D)) + 0.5
        a = sol_ref.reblock_partition(Q, K, P)
        b = np.array(brute.reblock_perm(Q.tolist(), K.tolist(), 1, N, 2, D, P))
        bad += int(not np.array_equal(a, b))
    return bad


def test_scalar_brute_force_agrees():
    assert _brute_failures() == 0


@pytest.mark.parametrize("N,P", [(64, 0), (65, 0), (300, 0), (300, 70), (300, 300), (1000, 1)])
def test_structure(N, P):
    rng = np.random.default_rng(N + P)
    Q = rng.standard_normal((2, N, 3, 8))
    K = rng.standard_normal((2, N, 3, 8))
    perm = sol_ref.reblock_partition(Q, K, P)
    assert _structure_failures(perm, N, P) == 0


@pytest.mark.parametrize("levels,prefix", [(2, 0), (3, 0), (3, 100)])
def test_planted_hierarchy_is_recovered(levels, prefix):
    assert _hierarchy_failures(levels=levels, prefix=prefix) == 0


def test_partition_is_invariant_under_reparametrisation():
    assert _invariance_failures() == 0


def test_split_follows_the_principal_axis():
    assert _principal_axis_failures() == 0


@pytest.mark.parametrize("P", [0, 70])
def test_all_exact_reblocked_pass_is_dense_attention(P):
    rng = np.random.default_rng(11)
    N, H, D = 300, 2, 8
    Q, K, V = (rng.standard_normal((1, N, H, D)) for _ in range(3))
    r = sol_ref.sol_forward(Q, K, V, tau=-math.inf, prefix=P, reblock=True)
    assert not np.array_equal(r["perm"][0, 0], np.arange(N))
    for h in range(H):
        S = Q[0, :, h] @ K[0, :, h].T / math.sqrt(D)
        Pm = np.exp(S - S.max(axis=1, keepdims=True))
        O = (Pm / Pm.sum(axis=1, keepdims=True)) @ V[0, :, h]
        assert np.allclose(r["O"][0, :, h], O, atol=1e-12)
        lse = np.log(np.exp(S - S.max(axis=1, keepdims=True)).sum(axis=1)) + S.max(axis=1)
        assert np.allclose(r["lse"][0, h], lse, atol=1e-12)


def test_reblocked_pass_is_the_plain_pass_on_permuted_rows():
    rng = np.random.default_rng(12)
    N, H, D = 300, 2, 8
    Q, K, V = (rng.standard_normal((1, N, H, D)) for _ in range(3))
    r = sol_ref.sol_forward(Q, K, V, tau=1.0, prefix=0, reblock=True, log_mass_bias_on=True)
    perm = r["perm"]
    p = sol_ref.sol_forward(sol_ref.permute_rows(Q, perm), sol_ref.permute_rows(K, perm),
                            sol_ref.permute_rows(V, perm), tau=1.0, prefix=0, log_mass_bias_on=True)
    assert np.array_equal(r["O_permuted"], p["O"])
    assert np.array_equal(sol_ref.permute_rows(r["O"], perm), p["O"])


def test_planted_reblock_mistakes_are_caught(monkeypatch):
    def plain_cosine(Q, prefix):
        B, N, H, D = Q.shape
        return np.tile(np.eye(D), (B, H, 1, 1))

    def uncentred_split(Y, members, bs, iters, leaves):
        n = len(members)
        if n <= bs:
            leaves.append(members)
            return
        left = bs * (-(-(-(-n // bs)) // 2))
        X = Y[members]
        w = X[0] / np.linalg.norm(X[0])
        for _ in range(iters):
            w = X.T @ (X @ w)
            w /= np.linalg.norm(w)
        go = np.zeros(n, dtype=bool)
        go[np.lexsort((members, X @ w))[:left]] = True
        uncentred_split(Y, members[go], bs, iters, leaves)
        uncentred_split(Y, members[~go], bs, iters, leaves)

    def halving_split(Y, members, bs, iters, leaves):
        n = len(members)
        if n <= bs:
            leaves.append(members)
            return
        X = Y[members]
        C = X - X.mean(axis=0)
        w = C[0] / np.linalg.norm(C[0])
        for _ in range(iters):
            w = C.T @ (C @ w)
            w /= np.linalg.norm(w)
        go = np.zeros(n, dtype=bool)
        go[np.lexsort((members, X @ w))[:n // 2]] = True
        halving_split(Y, members[go], bs, iters, leaves)
        halving_split(Y, members[~go], bs, iters, leaves)

    def all_pins():
        rng = np.random.default_rng(2)
        Q = rng.standard_normal((1, 300, 1, 8))
        K = rng.standard_normal((1, 300, 1, 8))
        return (_brute_failures() + _structure_failures(sol_ref.reblock_partition(Q, K, 0), 300, 0)
                + _hierarchy_failures() + _invariance_failures() + _principal_axis_failures())

    assert all_pins() == 0
    for name, fn in [("second_moment_whitener", plain_cosine), ("_split_group", uncentred_split),
                     ("_split_group", halving_split)]:
        monkeypatch.setattr(sol_ref, name, fn)
        assert all_pins() > 0, (name, fn.__name__)
        monkeypatch.undo()


# ---- the split-by-split checker the GPU tests apply to the GPU's order --------------------------

def _topic_inputs(N=1000, H=2, D=32, prefix=70, seed=11):
    """Keys with a mild cluster structure (16 topics) and isotropic queries."""
    rng = np.random.default_rng(seed)
    topics = rng.standard_normal((16, D))
    K = topics[rng.integers(0, 16, size=(1, N, H))] + rng.standard_normal((1, N, H, D))
    Q = rng.standard_normal((1, N, H, D))
    return Q, K, prefix


@pytest.mark.parametrize("N,H,D,prefix", [(1000, 2, 32, 70), (777, 1, 16, 13), (4096, 1, 16, 0), (300, 2, 8, 300)])
def test_split_checker_accepts_the_oracles_partition(N, H, D, prefix):
    from tests.reblock_check import check_splits
    Q, K, P = _topic_inputs(N, H, D, prefix)
    perm = sol_ref.reblock_partition(Q, K, P)
    rep = check_splits(Q, K, perm, P, band=0.0)
    assert rep.exact == rep.groups   # the oracle's own splits, recomputed on their own members
    n_v = N - min(N, 64 * (-(-P // 64)))
    assert rep.levels == (math.ceil(math.log2(n_v / 64)) if n_v > 64 else 0)


def _swap_across(perm, n_fix, start, n, which):
    """Move the left part's highest-projecting row and the right part's
    lowest-projecting row of one group across its split (each leaf re-sorted, so
    only the split itself is wrong)."""
    out = perm.copy()
    left = sol_ref.split_left_count(n)
    a, b = n_fix + start + which[0], n_fix + start + left + which[1]
    out[0, 0, a], out[0, 0, b] = perm[0, 0, b], perm[0, 0, a]
    for s in range(n_fix, out.shape[-1], 64):
        out[0, 0, s:s + 64] = np.sort(out[0, 0, s:s + 64])
    return out


def test_split_checker_catches_planted_mistakes():
    from tests.reblock_check import check_splits
    Q, K, P = _topic_inputs(N=1000, H=1, D=32, prefix=70)
    perm = sol_ref.reblock_partition(Q, K, P)
    n_fix = 128
    Y = sol_ref.whitened_unit_keys(K, sol_ref.second_moment_whitener(Q, P), n_fix)[0, 0]

    def extremes(start, n):
        part = perm[0, 0, n_fix + start:n_fix + start + n] - n_fix
        members = np.sort(part)
        p = sol_ref.split_projections(Y, members)[np.searchsorted(members, part)]
        left = sol_ref.split_left_count(n)
        return int(np.argmax(p[:left])), int(np.argmin(p[left:]))

    n_v = 1000 - n_fix
    first = _swap_across(perm, n_fix, 0, n_v, extremes(0, n_v))
    # 872 video rows: groups [0, 448), [0, 256), [0, 128); the last splits the first two leaves
    deep = _swap_across(perm, n_fix, 0, 128, extremes(0, 128))
    moved = perm.copy()
    moved[0, 0, [0, 500]] = moved[0, 0, [500, 0]]
    unsorted = perm.copy()
    unsorted[0, 0, [n_fix, n_fix + 1]] = unsorted[0, 0, [n_fix + 1, n_fix]]
    for bad in (first, deep, moved, unsorted):
        with pytest.raises(AssertionError):
            check_splits(Q, K, bad, P, band=1e-3)


@pytest.mark.parametrize("levels,prefix", [(8, 100), (9, 0)])
def test_planted_hierarchy_is_recovered_at_full_depth(levels, prefix):
    """The depth of the 16,384- and 32,768-row workloads: every leaf is one planted
    cluster and every split is the oracle's own, far from a tie (the inputs the GPU
    tests compare bit for bit)."""
    from block_sparse_video_sol_b200 import synth
    from tests.reblock_check import check_splits
    q, k, _, cid, n_fix = synth.planted_clusters(levels, 128, H=1, prefix=prefix, seed=10 * levels + 128, noise=0.004)
    Q, K = synth.bf16_bits_to_f64(q), synth.bf16_bits_to_f64(k)
    perm = sol_ref.reblock_partition(Q, K, prefix)
    for s in range(n_fix, perm.shape[-1], 64):
        assert len(set(cid[0, 0][perm[0, 0, s:s + 64] - n_fix].tolist())) == 1
    rep = check_splits(Q, K, perm, prefix, band=0.0)
    assert rep.levels == levels and rep.exact == rep.groups == 2 ** levels - 1
    assert rep.worst < -0.1   # every left part ends well below its right part
