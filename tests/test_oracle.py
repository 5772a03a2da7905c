"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test checks the oracle against a hand-derived case, an independent
brute-force restatement, a textbook special case (dense softmax attention,
also via torch's SDPA in fp64), or an invariant the method guarantees.  The
planted-mistake tests at the end show that plausible bugs in the oracle are
caught by at least one of these pins.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import brute, sol_ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
_MATH = {k: getattr(math, k) for k in ("exp", "log", "sqrt", "cosh")}


def _ev(expr):
    return float(eval(expr, {"__builtins__": {}}, _MATH))


def _hand():
    with open(os.path.join(GOLDEN, "hand_case.json")) as f:
        g = json.load(f)
    to4 = lambda a: np.array(a, float)[None, :, None, :]       # [B=1, N, H=1, D]
    return g, to4(g["Q"]), to4(g["K"]), to4(g["V"])


def dense_attention(Q, K, V, scale):
    """Textbook softmax(s Q K^T) V per (b, h)."""
    lg = scale * np.einsum("bnhd,bmhd->bhnm", Q, K)
    lg -= lg.max(axis=-1, keepdims=True)
    p = np.exp(lg)
    p /= p.sum(axis=-1, keepdims=True)
    return np.einsum("bhnm,bmhd->bnhd", p, V)


def rand_qkv(B, N, H, D, seed, structured=True):
    rng = np.random.default_rng(seed)
    if structured:
        # blockwise-correlated keys so routing has something to find
        topics = rng.standard_normal((4, D))
        t = rng.integers(0, 4, size=(B, N // 4 + 1, H))
        base = topics[np.repeat(t, 4, axis=1)[:, :N]]
        Q = 1.5 * base + rng.standard_normal((B, N, H, D))
        K = 1.5 * base + rng.standard_normal((B, N, H, D))
    else:
        Q = rng.standard_normal((B, N, H, D))
        K = rng.standard_normal((B, N, H, D))
    V = rng.standard_normal((B, N, H, D))
    return Q, K, V


# ---------------------------------------------------------------- hand case
def test_hand_case_scores_thresholds_masks():
    g, Q, K, V = _hand()
    bs = g["block"]
    out = sol_ref.sol_forward(Q, K, V, tau=0.5, bq=bs, bk=bs)
    np.testing.assert_allclose(out["S"][0, 0], np.array(g["S"], float), rtol=0, atol=1e-15)
    for tau, thr in g["thr"].items():
        got = sol_ref.thresholds(out["S"], float(tau))[0, 0]
        np.testing.assert_allclose(got, [_ev(e) for e in thr], rtol=0, atol=1e-14)
    for m in g["masks"]:
        tau = -math.inf if m["tau"] == "-inf" else float(m["tau"])
        o = sol_ref.sol_forward(Q, K, V, tau=tau, prefix=m["prefix"], bq=bs, bk=bs)
        assert o["sel"][0, 0].astype(int).tolist() == m["sel"], m
        _, bsel = brute.forward(Q, K, V, 1, g["N"], 1, g["D"], tau, m["prefix"], bs, bs)
        assert np.array(bsel[0][0]).astype(int).tolist() == m["sel"], m


def test_hand_case_bias_and_outputs():
    g, Q, K, V = _hand()
    bs = g["block"]
    o = sol_ref.sol_forward(Q, K, V, tau=1.0, bq=bs, bk=bs, log_mass_bias_on=True)
    np.testing.assert_allclose(o["bias"][0, 0], [_ev(e) for e in g["bias_prefix0"]], atol=1e-13)
    for case in g["outputs"]:
        want = [_ev(e) for e in case["o"]]
        o = sol_ref.sol_forward(Q, K, V, tau=case["tau"], prefix=case["prefix"], bq=bs, bk=bs,
                                log_mass_bias_on=case["log_mass_bias"])
        np.testing.assert_allclose(o["O"][0, case["row"], 0], want, rtol=1e-13, atol=1e-15)
        bo, _ = brute.forward(Q, K, V, 1, g["N"], 1, g["D"], case["tau"], case["prefix"], bs, bs,
                              lmb=case["log_mass_bias"])
        np.testing.assert_allclose(bo[0][case["row"]][0], want, rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------- pooling
def test_pool_ragged_matches_loops():
    Q, _, _ = rand_qkv(2, 77, 3, 5, seed=1)
    for bs in (1, 4, 16, 64, 100):
        got = sol_ref.pool(Q, bs)
        nb = -(-77 // bs)
        assert got.shape == (2, 3, nb, 5)
        for b in range(2):
            for h in range(3):
                for j in range(nb):
                    rows = range(j * bs, min(77, (j + 1) * bs))
                    ref = [sum(Q[b, r, h, c] for r in rows) / len(rows) for c in range(5)]
                    np.testing.assert_allclose(got[b, h, j], ref, rtol=1e-14, atol=1e-14)


def test_block_rows_tail():
    assert sol_ref.block_rows(38247, 64)[-1] == 38247 - 597 * 64 == 39
    assert sol_ref.n_blocks(38247, 64) == 598
    assert sol_ref.block_rows(4096, 64).tolist() == [64] * 64
    assert sol_ref.n_blocks(0, 64) == 0


def test_pool_block1_is_identity():
    Q, _, _ = rand_qkv(1, 9, 2, 3, seed=2)
    np.testing.assert_array_equal(sol_ref.pool(Q, 1), Q.transpose(0, 2, 1, 3))


# ---------------------------------------------------------------- routing
def test_route_matches_brute_random():
    rng = np.random.default_rng(3)
    for trial in range(6):
        N = int(rng.integers(20, 120))
        bq, bk = int(rng.choice([4, 8, 16])), int(rng.choice([4, 8, 16]))
        P = int(rng.integers(0, N // 3))
        tau = float(rng.choice([-1.0, 0.0, 0.5, 1.0, 2.0]))
        Q, K, V = rand_qkv(1, N, 2, 6, seed=10 + trial)
        o = sol_ref.sol_forward(Q, K, V, tau=tau, prefix=P, bq=bq, bk=bk)
        _, bsel = brute.forward(Q, K, V, 1, N, 2, 6, tau, P, bq, bk)
        # compare away from the threshold (ties are measure-zero with random data)
        assert (o["sel"][0] == np.array(bsel[0])).all(), (N, bq, bk, P, tau)


def test_route_nesting_and_density_monotone():
    Q, K, V = rand_qkv(1, 256, 3, 8, seed=4)
    qbar, kbar = sol_ref.pool(Q, 8), sol_ref.pool(K, 8)
    S = sol_ref.scores(qbar, kbar, 1 / math.sqrt(8))
    taus = [-math.inf, -1.0, 0.0, 0.5, 1.0, 1.5, 2.0, 3.0]
    sels = [sol_ref.route(S, t, 0, 8, 8) for t in taus]
    assert sels[0].all()
    dens = [s.mean() for s in sels]
    for a, b in zip(sels, sels[1:]):
        assert not (b & ~a).any(), "selection must shrink as tau grows"
    assert all(x >= y for x, y in zip(dens, dens[1:]))
    assert dens[-1] < dens[1]


def test_route_sinks_and_dense_rows():
    Q, K, V = rand_qkv(1, 130, 2, 4, seed=5)
    qbar, kbar = sol_ref.pool(Q, 16), sol_ref.pool(K, 16)
    S = sol_ref.scores(qbar, kbar, 0.5)
    for P in (0, 1, 16, 17, 130):
        sel = sol_ref.route(S, 5.0, P, 16, 16)
        ns = -(-P // 16)
        assert sel[..., :, :ns].all()
        assert sel[..., :ns, :].all()
        if P == 0:
            assert not sel.all()


def test_route_zero_std_selects_nothing():
    S = np.zeros((1, 1, 3, 5))
    assert not sol_ref.route(S, 0.0, 0, 64, 64).any()
    assert sol_ref.route(S, -math.inf, 0, 64, 64).all()


def test_csr_roundtrip_and_order():
    rng = np.random.default_rng(6)
    sel = rng.random((2, 3, 5, 7)) < 0.3
    row_ptr, col = sol_ref.to_csr(sel)
    assert row_ptr[0] == 0 and row_ptr[-1] == sel.sum() == col.size
    flat = sel.reshape(-1, 7)
    for r in range(flat.shape[0]):
        seg = col[row_ptr[r]:row_ptr[r + 1]]
        assert (np.diff(seg) > 0).all()
        assert seg.tolist() == [j for j in range(7) if flat[r, j]]
    assert (sol_ref.from_csr(row_ptr, col, sel.shape) == sel).all()


# ---------------------------------------------------------------- attention
@pytest.mark.parametrize("N,bq,bk", [(64, 8, 8), (77, 16, 8), (50, 8, 16)])
def test_all_exact_equals_dense(N, bq, bk):
    Q, K, V = rand_qkv(2, N, 2, 8, seed=7)
    s = 1 / math.sqrt(8)
    ref = dense_attention(Q, K, V, s)
    o1 = sol_ref.sol_forward(Q, K, V, tau=-math.inf, bq=bq, bk=bk)
    np.testing.assert_allclose(o1["O"], ref, rtol=1e-12, atol=1e-12)
    o2 = sol_ref.sol_forward(Q, K, V, tau=1.0, prefix=N, bq=bq, bk=bk, log_mass_bias_on=True)
    np.testing.assert_allclose(o2["O"], ref, rtol=1e-12, atol=1e-12)
    # library cross-check of the textbook reference itself
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)
    sd = torch.nn.functional.scaled_dot_product_attention(t(Q), t(K), t(V), scale=s)
    np.testing.assert_allclose(sd.permute(0, 2, 1, 3).numpy(), ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("tau", [-1.0, 0.0, 1.0, 2.5])
@pytest.mark.parametrize("lmb", [False, True])
def test_block_size_one_is_dense(tau, lmb):
    """With one-row blocks a centroid term is its row, so any routing gives dense attention."""
    Q, K, V = rand_qkv(1, 40, 2, 4, seed=8)
    o = sol_ref.sol_forward(Q, K, V, tau=tau, prefix=3, bq=1, bk=1, log_mass_bias_on=lmb)
    np.testing.assert_allclose(o["bias"], 0.0, atol=1e-12)
    np.testing.assert_allclose(o["O"], dense_attention(Q, K, V, 0.5), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("tau", [0.0, 1.0, 2.0])
@pytest.mark.parametrize("lmb", [False, True])
def test_blockwise_constant_kv_is_dense(tau, lmb):
    """If K and V rows are constant inside each key block, n identical exact terms
    equal one centroid term with logit + log n, for any routing (ragged tail too)."""
    rng = np.random.default_rng(9)
    N, bk, D = 100, 16, 8
    Q = rng.standard_normal((1, N, 2, D))
    kb = rng.standard_normal((1, -(-N // bk), 2, D))
    vb = rng.standard_normal((1, -(-N // bk), 2, D))
    K = np.repeat(kb, bk, axis=1)[:, :N]
    V = np.repeat(vb, bk, axis=1)[:, :N]
    o = sol_ref.sol_forward(Q, K, V, tau=tau, prefix=5, bq=16, bk=bk, log_mass_bias_on=lmb)
    assert not o["sel"].all()
    np.testing.assert_allclose(o["O"], dense_attention(Q, K, V, 1 / math.sqrt(D)),
                               rtol=1e-11, atol=1e-12)


def test_constant_v_gives_constant_output():
    Q, K, _ = rand_qkv(1, 90, 2, 6, seed=10)
    V = np.full_like(Q, 0.375)
    o = sol_ref.sol_forward(Q, K, V, tau=1.0, prefix=7, bq=16, bk=16, log_mass_bias_on=True)
    np.testing.assert_allclose(o["O"], 0.375, rtol=1e-13)


def test_bias_properties():
    Q, K, _ = rand_qkv(2, 70, 2, 6, seed=11)
    s = 1 / math.sqrt(6)
    for P in (0, 9, 70):
        kbar = sol_ref.pool(K, 16)
        bias = sol_ref.log_mass_bias(Q, K, kbar, P, s, 16)
        assert (bias >= -1e-13).all(), "Jensen: log-mean-exp >= mean"
        # the defining property: for a query equal to the anchor the centroid
        # term carries exactly the block's exact mass
        a = sol_ref.anchor(Q, P)
        nk = sol_ref.block_rows(70, 16)
        for j in range(kbar.shape[2]):
            lo, hi = 16 * j, min(70, 16 * (j + 1))
            exact = np.exp(s * np.einsum("bnhd,bhd->bhn", K[:, lo:hi], a)).sum(-1)
            cent = nk[j] * np.exp(s * np.einsum("bhd,bhd->bh", a, kbar[:, :, j]) + bias[:, :, j])
            np.testing.assert_allclose(cent, exact, rtol=1e-12)
    Kc = np.repeat(K[:, :1], 70, axis=1)
    np.testing.assert_allclose(sol_ref.log_mass_bias(Q, Kc, sol_ref.pool(Kc, 16), 0, s, 16), 0,
                               atol=1e-12)


def test_anchor_is_video_mean():
    Q, _, _ = rand_qkv(1, 30, 1, 3, seed=12)
    np.testing.assert_allclose(sol_ref.anchor(Q, 10)[0, 0], Q[0, 10:, 0].mean(0))
    np.testing.assert_allclose(sol_ref.anchor(Q, 30)[0, 0], Q[0, :, 0].mean(0))


@pytest.mark.parametrize("seed", range(5))
def test_matches_brute_random(seed):
    rng = np.random.default_rng(100 + seed)
    N = int(rng.integers(17, 90))
    bq, bk = int(rng.choice([4, 8, 16])), int(rng.choice([4, 8, 16]))
    P = int(rng.integers(0, N // 2))
    tau = float(rng.choice([-0.5, 0.5, 1.0, 1.5]))
    lmb = bool(seed % 2)
    Q, K, V = rand_qkv(1, N, 2, 4, seed=200 + seed)
    o = sol_ref.sol_forward(Q, K, V, tau=tau, prefix=P, bq=bq, bk=bk, log_mass_bias_on=lmb)
    bo, bsel = brute.forward(Q, K, V, 1, N, 2, 4, tau, P, bq, bk, lmb=lmb)
    assert (o["sel"][0] == np.array(bsel[0])).all()
    np.testing.assert_allclose(o["O"], np.array(bo), rtol=1e-11, atol=1e-12)


def test_row_subset_and_mask_override():
    Q, K, V = rand_qkv(1, 96, 2, 4, seed=13)
    full = sol_ref.sol_forward(Q, K, V, tau=0.5, bq=16, bk=16)
    part = sol_ref.sol_forward(Q, K, V, tau=0.5, bq=16, bk=16,
                               rows={(0, 1): np.array([3, 50, 95])})
    np.testing.assert_allclose(part["O"][0, [3, 50, 95], 1], full["O"][0, [3, 50, 95], 1],
                               rtol=1e-13, atol=1e-15)
    assert np.isnan(part["O"][0, :, 0]).all()
    allsel = np.ones_like(full["sel"])
    ov = sol_ref.sol_forward(Q, K, V, tau=0.5, bq=16, bk=16, mask_override=allsel)
    np.testing.assert_allclose(ov["O"], dense_attention(Q, K, V, 0.5), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- planted mistakes
def _pins_fail(monkeypatch, name, fn):
    """Replace one oracle step with a mistaken version and report whether the pins notice."""
    monkeypatch.setattr(sol_ref, name, fn)
    failures = 0
    for test in (test_hand_case_scores_thresholds_masks, test_hand_case_bias_and_outputs,
                 lambda: test_blockwise_constant_kv_is_dense(1.0, True),
                 lambda: test_all_exact_equals_dense(77, 16, 8),
                 lambda: test_matches_brute_random(1)):
        try:
            test()
        except AssertionError:
            failures += 1
    return failures


def test_planted_mistakes_are_caught(monkeypatch):
    good_attention, good_thr, good_bias, good_pool = (sol_ref.attention, sol_ref.thresholds,
                                                      sol_ref.log_mass_bias, sol_ref.pool)

    def no_log_n(Q, K, V, sel, kbar, vbar, bias, scale, bq, bk, rows=None, **kw):
        return good_attention(Q, K, V, sel, kbar, vbar, bias - np.log(
            sol_ref.block_rows(Q.shape[1], bk))[None, None, :], scale, bq, bk, rows, **kw)

    def sample_std(S, tau):
        mu = S.mean(-1)
        return mu + tau * S.std(-1, ddof=1)

    def bias_sign(Q, K, kbar, prefix, scale, bk):
        return -good_bias(Q, K, kbar, prefix, scale, bk)

    def pool_sum(X, bs):
        return good_pool(X, bs) * bs

    for name, fn in [("attention", no_log_n), ("thresholds", sample_std),
                     ("log_mass_bias", bias_sign), ("pool", pool_sum)]:
        assert _pins_fail(monkeypatch, name, fn) > 0, name
        monkeypatch.undo()


# ---------------------------------------------------------------- weighted summaries
def _uniform_q(N, H, D, seed):
    """Every query row of a head equal to one vector: the anchor itself."""
    c = np.random.default_rng(seed).standard_normal((1, 1, H, D))
    return np.repeat(c, N, axis=1)


@pytest.mark.parametrize("N,bk,P", [(77, 16, 0), (77, 16, 9), (64, 8, 64), (50, 50, 3)])
def test_reweight_anchor_query_is_exact(N, bk, P):
    """A query equal to the anchor gets each centroid block's exact contribution
    (mass and value), so any routing reproduces dense attention for it; the
    mean-pooled summary with the bias gets the mass but not the value."""
    _, K, V = rand_qkv(1, N, 2, 6, seed=14)
    Q = _uniform_q(N, 2, 6, seed=15)
    s = 1 / math.sqrt(6)
    dense = dense_attention(Q, K, V, s)
    none = np.zeros((1, 2, -(-N // 16), -(-N // bk)), bool)
    for ov in (none, None):
        o = sol_ref.sol_forward(Q, K, V, tau=0.3, prefix=P, bq=16, bk=bk, reweight_on=True,
                                mask_override=ov)
        np.testing.assert_allclose(o["O"], dense, rtol=1e-11, atol=1e-12)
    lmb = sol_ref.sol_forward(Q, K, V, tau=0.3, prefix=P, bq=16, bk=bk, log_mass_bias_on=True,
                              mask_override=none)
    assert np.abs(lmb["O"] - dense).max() > 1e-3


def test_reweight_bias_is_entropy_gap():
    """log mean exp(x) - E_w[x] with w = softmax(x) equals H(w) - log n, so the
    bias is the weights' entropy deficit: <= 0, and 0 exactly for uniform weights."""
    Q, K, V = rand_qkv(2, 70, 2, 6, seed=16)
    s = 1 / math.sqrt(6)
    for P in (0, 11):
        kc, vc, bias = sol_ref.reweighted_summaries(Q, K, V, P, s, 16)
        a = sol_ref.anchor(Q, P)
        for j in range(kc.shape[2]):
            lo, hi = 16 * j, min(70, 16 * (j + 1))
            x = s * np.einsum("bnhd,bhd->bhn", K[:, lo:hi], a)
            w = np.exp(x - x.max(-1, keepdims=True))
            w /= w.sum(-1, keepdims=True)
            H = -(w * np.log(w)).sum(-1)
            np.testing.assert_allclose(bias[:, :, j], H - math.log(hi - lo), rtol=1e-10,
                                       atol=1e-12)
            # summaries are convex combinations: inside each coordinate's range
            for X, C in ((K, kc), (V, vc)):
                blk = X[:, lo:hi].transpose(0, 2, 1, 3)
                assert (C[:, :, j] <= blk.max(2) + 1e-12).all()
                assert (C[:, :, j] >= blk.min(2) - 1e-12).all()
        assert (bias <= 1e-13).all()


def test_reweight_zero_anchor_is_mean_pooling():
    """With a zero anchor the weights are uniform: the summaries are the block
    means, the bias vanishes and the pass equals the plain one."""
    Q, K, V = rand_qkv(1, 96, 2, 4, seed=17)
    P = 8
    Q[0, P + 44:] = -Q[0, P:P + 44]                       # video rows cancel in pairs
    o = sol_ref.sol_forward(Q, K, V, tau=0.5, prefix=P, bq=16, bk=16, reweight_on=True)
    p = sol_ref.sol_forward(Q, K, V, tau=0.5, prefix=P, bq=16, bk=16)
    np.testing.assert_allclose(sol_ref.anchor(Q, P), 0, atol=1e-14)
    np.testing.assert_allclose(o["kc"], p["kbar"], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(o["vc"], p["vbar"], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(o["bias"], 0, atol=1e-13)
    np.testing.assert_allclose(o["O"], p["O"], rtol=1e-12, atol=1e-13)
    assert (o["sel"] == p["sel"]).all()


@pytest.mark.parametrize("tau", [-1.0, 1.0])
def test_reweight_block_size_one_is_dense(tau):
    Q, K, V = rand_qkv(1, 40, 2, 4, seed=18)
    o = sol_ref.sol_forward(Q, K, V, tau=tau, prefix=3, bq=1, bk=1, reweight_on=True)
    np.testing.assert_allclose(o["kc"], K.transpose(0, 2, 1, 3), rtol=1e-14)
    np.testing.assert_allclose(o["vc"], V.transpose(0, 2, 1, 3), rtol=1e-14)
    np.testing.assert_allclose(o["bias"], 0.0, atol=1e-12)
    np.testing.assert_allclose(o["O"], dense_attention(Q, K, V, 0.5), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("seed", range(4))
def test_reweight_matches_brute_random(seed):
    rng = np.random.default_rng(300 + seed)
    N = int(rng.integers(17, 90))
    bq, bk = int(rng.choice([4, 8, 16])), int(rng.choice([4, 8, 16]))
    P = int(rng.integers(0, N // 2))
    tau = float(rng.choice([-0.5, 0.5, 1.0, 1.5]))
    Q, K, V = rand_qkv(1, N, 2, 4, seed=400 + seed)
    o = sol_ref.sol_forward(Q, K, V, tau=tau, prefix=P, bq=bq, bk=bk, reweight_on=True)
    bo, bsel = brute.forward(Q, K, V, 1, N, 2, 4, tau, P, bq, bk, rw=True)
    assert (o["sel"][0] == np.array(bsel[0])).all()
    np.testing.assert_allclose(o["O"], np.array(bo), rtol=1e-11, atol=1e-12)


def test_planted_reweight_mistakes_are_caught(monkeypatch):
    good = sol_ref.reweighted_summaries

    def unscaled_weights(Q, K, V, prefix, scale, bk):   # softmax of a.k without s
        kc, vc, _ = good(Q, K, V, prefix, 1.0, bk)
        _, _, bias = good(Q, K, V, prefix, scale, bk)
        return kc, vc, bias

    def bias_vs_mean(Q, K, V, prefix, scale, bk):       # bias taken against kbar
        kc, vc, _ = good(Q, K, V, prefix, scale, bk)
        return kc, vc, sol_ref.log_mass_bias(Q, K, sol_ref.pool(K, bk), prefix, scale, bk)

    def mean_values(Q, K, V, prefix, scale, bk):        # values left mean-pooled
        kc, _, bias = good(Q, K, V, prefix, scale, bk)
        return kc, sol_ref.pool(V, bk), bias

    for fn in (unscaled_weights, bias_vs_mean, mean_values):
        monkeypatch.setattr(sol_ref, "reweighted_summaries", fn)
        failures = 0
        for test in (lambda: test_reweight_anchor_query_is_exact(77, 16, 9),
                     lambda: test_reweight_matches_brute_random(0)):
            try:
                test()
            except AssertionError:
                failures += 1
        assert failures > 0, fn.__name__
        monkeypatch.undo()


# ---------------------------------------------------------------- Top-K routing
def test_topk_count_reading():
    # k = nearest integer to ratio * n_kb (halves up), from the float32 ratio the ABI carries
    assert sol_ref.topk_count(0.15, 512) == 77       # 76.8
    assert sol_ref.topk_count(0.1, 10) == 1          # float32(0.1) * 10 is just above 1
    assert sol_ref.topk_count(0.3, 10) == 3          # float32(0.3) * 10 is just above 3
    assert sol_ref.topk_count(0.25, 10) == 3         # exactly 2.5: halves up
    assert sol_ref.topk_count(0.25, 512) == 128      # exact in float32
    assert sol_ref.topk_count(1e-9, 100) == 1
    assert sol_ref.topk_count(1.0, 100) == 100


def test_topk_selection_invariants():
    rng = np.random.default_rng(19)
    S = rng.standard_normal((2, 3, 9, 40))
    prev = None
    for k in (1, 5, 12, 40):
        sel = sol_ref.route_topk(S, k, prefix=0, bq=128)
        assert (sel.sum(-1) == k).all()
        # the selected scores dominate the unselected ones row by row
        lo = np.where(sel, S, np.inf).min(-1)
        hi = np.where(sel, -np.inf, S).max(-1)
        assert (lo >= hi).all()
        if prev is not None:
            assert (sel | ~prev).all(), "top-k sets nest"
        prev = sel
    # ties rank the lower index first; prefix query blocks keep everything
    T = np.zeros((1, 1, 3, 10))
    T[..., 7] = 1.0
    sel = sol_ref.route_topk(T, 3, prefix=130, bq=128)
    assert sel[0, 0, :2].all()
    assert np.nonzero(sel[0, 0, 2])[0].tolist() == [0, 1, 7]


def _masked_dense(Q, K, V, sel, scale, bq, bk):
    """Softmax attention of each query row over only the keys of its selected blocks."""
    B, N, H, D = Q.shape
    keep = np.repeat(np.repeat(sel, bq, axis=2)[:, :, :N], bk, axis=3)[..., :N]   # [B, H, N, N]
    lg = scale * np.einsum("bnhd,bmhd->bhnm", Q, K)
    lg = np.where(keep, lg, -np.inf)
    lg -= lg.max(-1, keepdims=True)
    p = np.exp(lg)
    p /= p.sum(-1, keepdims=True)
    return np.einsum("bhnm,bmhd->bnhd", p, V)


@pytest.mark.parametrize("N,bq,bk,P,ratio", [(300, 128, 64, 0, 0.2), (257, 128, 64, 70, 0.1),
                                             (90, 16, 8, 5, 0.3)])
def test_topk_attention_is_masked_softmax(N, bq, bk, P, ratio):
    """Unselected blocks are dropped: the output is softmax attention restricted to
    the selected keys (no centroid term); ratio 1 gives dense attention."""
    Q, K, V = rand_qkv(1, N, 2, 8, seed=20)
    s = 1 / math.sqrt(8)
    o = sol_ref.sol_forward(Q, K, V, prefix=P, bq=bq, bk=bk, topk_ratio=ratio)
    nkb = -(-N // bk)
    assert o["k"] == sol_ref.topk_count(ratio, nkb)
    np.testing.assert_allclose(o["O"], _masked_dense(Q, K, V, o["sel"], s, bq, bk), rtol=1e-11, atol=1e-12)
    full = sol_ref.sol_forward(Q, K, V, prefix=P, bq=bq, bk=bk, topk_ratio=1.0)
    np.testing.assert_allclose(full["O"], dense_attention(Q, K, V, s), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("seed", range(4))
def test_topk_matches_brute_random(seed):
    rng = np.random.default_rng(500 + seed)
    N = int(rng.integers(17, 90))
    bq, bk = int(rng.choice([8, 16, 32])), int(rng.choice([4, 8, 16]))
    P = int(rng.integers(0, N // 2))
    ratio = float(rng.choice([0.1, 0.25, 0.5]))
    Q, K, V = rand_qkv(1, N, 2, 4, seed=600 + seed)
    o = sol_ref.sol_forward(Q, K, V, prefix=P, bq=bq, bk=bk, topk_ratio=ratio)
    bo, bsel = brute.forward(Q, K, V, 1, N, 2, 4, 0.0, P, bq, bk, topk=o["k"])
    assert (o["sel"][0] == np.array(bsel[0])).all()
    np.testing.assert_allclose(o["O"], np.array(bo), rtol=1e-11, atol=1e-12)


def test_planted_topk_mistakes_are_caught(monkeypatch):
    good_route, good_count, good_att = sol_ref.route_topk, sol_ref.topk_count, sol_ref.attention

    def ties_high(S, k, prefix, bq):              # equal scores ranked by the higher index
        return good_route(S[..., ::-1], k, prefix, bq)[..., ::-1]

    def one_short(ratio, nkb):                    # floor instead of the nearest integer
        return max(1, int(float(np.float32(ratio)) * nkb))

    def keeps_centroids(*args, centroids=True, **kw):
        return good_att(*args, centroids=True, **kw)

    for name, fn in [("route_topk", ties_high), ("topk_count", one_short), ("attention", keeps_centroids)]:
        monkeypatch.setattr(sol_ref, name, fn)
        failures = 0
        for test in (test_topk_count_reading, test_topk_selection_invariants,
                     lambda: test_topk_attention_is_masked_softmax(257, 128, 64, 70, 0.1),
                     lambda: test_topk_matches_brute_random(0)):
            try:
                test()
            except AssertionError:
                failures += 1
        assert failures > 0, name
        monkeypatch.undo()


# ---------------------------------------------------------------- Top-K with the compressed branch
@pytest.mark.parametrize("seed", range(4))
def test_topk_compressed_matches_brute_random(seed):
    rng = np.random.default_rng(700 + seed)
    N = int(rng.integers(17, 90))
    bq, bk = int(rng.choice([4, 8, 16])), int(rng.choice([4, 8, 16]))
    P = int(rng.integers(0, N // 2))
    ratio = float(rng.choice([0.1, 0.25, 0.5]))
    lmb, rw = [(False, False), (True, False), (False, True), (False, False)][seed]
    Q, K, V = rand_qkv(1, N, 2, 4, seed=800 + seed)
    o = sol_ref.sol_forward(Q, K, V, prefix=P, bq=bq, bk=bk, topk_ratio=ratio, compressed=True,
                            log_mass_bias_on=lmb, reweight_on=rw)
    bo, bsel = brute.forward(Q, K, V, 1, N, 2, 4, 0.0, P, bq, bk, topk=o["k"], compressed=True, lmb=lmb, rw=rw)
    assert (o["sel"][0] == np.array(bsel[0])).all()
    np.testing.assert_allclose(o["O"], np.array(bo), rtol=1e-11, atol=1e-12)


def test_topk_compressed_selection_and_reductions():
    Q, K, V = rand_qkv(1, 200, 2, 8, seed=28)
    P, bk = 40, 16
    nkb = -(-200 // bk)
    o = sol_ref.sol_forward(Q, K, V, prefix=P, bq=16, bk=bk, topk_ratio=0.3, compressed=True)
    k, n_sink, n_dense = o["k"], sol_ref.n_blocks(P, bk), sol_ref.n_blocks(P, 16)
    cnt = o["sel"].sum(-1)[:, :, n_dense:]
    assert (cnt >= k).all() and (cnt <= k + n_sink).all()
    assert o["sel"][..., :n_sink].all() and o["sel"][:, :, :n_dense].all()
    plain = sol_ref.route_topk(o["S"], k, P, 16)
    assert (o["sel"] == (plain | (np.arange(nkb) < n_sink))).all()
    # every block kept: dense attention; blockwise-constant K/V: dense for any k
    full = sol_ref.sol_forward(Q, K, V, prefix=P, bq=16, bk=bk, topk_ratio=1.0, compressed=True, reweight_on=True)
    np.testing.assert_allclose(full["O"], dense_attention(Q, K, V, 1 / math.sqrt(8)), rtol=1e-11, atol=1e-12)
    kb = np.random.default_rng(29).standard_normal((1, nkb, 2, 8))
    vb = np.random.default_rng(30).standard_normal((1, nkb, 2, 8))
    Kc, Vc = np.repeat(kb, bk, axis=1)[:, :200], np.repeat(vb, bk, axis=1)[:, :200]
    oc = sol_ref.sol_forward(Q, Kc, Vc, prefix=P, bq=16, bk=bk, topk_ratio=0.2, compressed=True)
    np.testing.assert_allclose(oc["O"], dense_attention(Q, Kc, Vc, 1 / math.sqrt(8)), rtol=1e-11, atol=1e-12)


def test_planted_topk_compressed_mistakes_are_caught(monkeypatch):
    good_route, good_att = sol_ref.route_topk, sol_ref.attention

    def no_sink(S, k, prefix, bq, bk=None):
        return good_route(S, k, prefix, bq)

    def drops_centroids(*args, centroids=True, **kw):
        return good_att(*args, centroids=False, **kw)

    for name, fn in [("route_topk", no_sink), ("attention", drops_centroids)]:
        monkeypatch.setattr(sol_ref, name, fn)
        failures = 0
        for test in (test_topk_compressed_selection_and_reductions,
                     lambda: test_topk_compressed_matches_brute_random(1)):
            try:
                test()
            except AssertionError:
                failures += 1
        assert failures > 0, name
        monkeypatch.undo()
