"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and compare each stage with the fp64 oracle.

Criteria (bf16 I/O, fp32 accumulate):
  * pooled centroids: fp32 means within 1e-5 relative (+1e-6 absolute) of the
    oracle; bf16 copies within one bf16 rounding of the oracle's mean (of the
    anchor-weighted summary in mode 2, +1e-5 absolute for the fp32 weighted
    sums with expf weights);
  * routing: the GPU mask equals the oracle's on every block whose score is
    more than 1e-4 from its row threshold (Top-K: from the row's k-th
    largest score, with exactly k blocks per row and both 64-row halves of a
    128-row block carrying the same list), and the GPU CSR equals the
    oracle's CSR of the GPU mask bit for bit;
  * attention: with the oracle run on the GPU's mask, max |O_gpu - O_ref| <=
    2e-2 and mean |O_gpu - O_ref| <= 2e-3.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from block_sparse_video_sol_b200 import synth
from oracle import sol_ref

MAX_ABS, MEAN_ABS, BAND = 2e-2, 2e-3, 1e-4


def to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def run_gpu(q, k, v, tau, prefix, lmb, with_lse=True, in_strides=None, topk_ratio=None, compressed=False,
            qk_int8=False):
    from block_sparse_video_sol_b200 import sol
    B, N, H, D = q.shape
    strides = in_strides or (q.stride(0), q.stride(1), q.stride(2))
    p = sol.make_params(B, N, H, D, tau=tau, prefix_len=prefix, log_mass_bias=lmb, in_strides=strides,
                        topk_ratio=topk_ratio, compressed=compressed, qk_int8=qk_int8)
    buf = sol.alloc_buffers(p, q.device, with_lse=with_lse)
    sol.forward(p, q, k, v, buf)
    sol.sol_last_device_status()
    torch.cuda.synchronize()
    return p, buf


def gpu_mask(p, buf):
    nb = -(-p.N // 64)
    rp = buf.row_ptr.cpu().numpy().astype(np.int64)
    ci = buf.col_idx[:int(rp[-1])].cpu().numpy().astype(np.int64)
    return rp, ci, sol_ref.from_csr(rp, ci, (p.B, p.H, nb, nb))


def oracle_modes(lmb):
    """sol_forward flags for the centroid mode 0 / 1 (bias) / 2 (weighted summaries)."""
    return dict(log_mass_bias_on=int(lmb) == 1, reweight_on=int(lmb) == 2)


def check_pool(p, buf, Qd, Kd, Vd, heads, lmb, prefix, topk=False):
    """Pooled quantities of the given head indices vs the oracle (Top-K routing pools no V)."""
    from block_sparse_video_sol_b200 import sol
    w = sol.workspace_views(p, buf.ws)
    s = 1.0 / math.sqrt(p.D)
    qbar, kbar, vbar = sol_ref.pool(Qd, 64), sol_ref.pool(Kd, 64), sol_ref.pool(Vd, 64)
    names = ("qbar", "kbar", "kbar16", "cbias") + (() if topk else ("vbar16",))   # Top-K pools no V
    g = {k: w[k][:, heads].float().cpu().numpy().astype(np.float64) for k in names}
    np.testing.assert_allclose(g["qbar"], qbar, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(g["kbar"], kbar, rtol=1e-5, atol=1e-6)
    logn = np.log(sol_ref.block_rows(p.N, 64).astype(np.float64))
    if int(lmb) == 2:
        kc, vc, bias = sol_ref.reweighted_summaries(Qd, Kd, Vd, prefix, s, 64)
        np.testing.assert_allclose(g["kbar16"], kc, rtol=2 ** -8, atol=1e-5)
        np.testing.assert_allclose(g["vbar16"], vc, rtol=2 ** -8, atol=1e-5)
    else:
        np.testing.assert_allclose(g["kbar16"], kbar, rtol=2 ** -8, atol=1e-6)
        if not topk:
            np.testing.assert_allclose(g["vbar16"], vbar, rtol=2 ** -8, atol=1e-6)
        bias = sol_ref.log_mass_bias(Qd, Kd, kbar, prefix, s, 64) if lmb else 0.0
    want = logn[None, None, :] + bias
    want = np.broadcast_to(want, g["cbias"].shape)
    np.testing.assert_allclose(g["cbias"], want, rtol=0, atol=2e-4)
    return qbar, kbar, vbar


def check_route(p, buf, qbar, kbar, heads, tau, prefix):
    """Mask parity outside the threshold band, and CSR bit-exactness."""
    s = 1.0 / math.sqrt(p.D)
    S = sol_ref.scores(qbar, kbar, s)
    thr = sol_ref.thresholds(S, tau)
    sel = sol_ref.route(S, tau, prefix, 64, 64)
    rp, ci, gm = gpu_mask(p, buf)
    # CSR bit-exact for the GPU's own mask (every head)
    rp_ref, ci_ref = sol_ref.to_csr(gm)
    assert np.array_equal(rp, rp_ref)
    assert np.array_equal(ci, ci_ref)
    g = gm[:, heads]
    far = np.abs(S - thr[..., None]) > BAND if tau != -math.inf else np.ones_like(sel)
    bad = (g != sel) & far
    assert not bad.any(), f"{int(bad.sum())} mask mismatches outside the {BAND} band"
    return gm, int(((g != sel) & ~far).sum())


def check_route_topk(p, buf, Qd, Kd, heads, ratio, prefix, compressed=False):
    """Top-K mask parity outside the tie band, k per row (plus sinks with the
    compressed branch), equal halves of a 128-row block (SLA), CSR bit-exactness.

    Returns the GPU mask of the given heads at the routing's query-block granularity."""
    s = 1.0 / math.sqrt(p.D)
    bq = 64 if compressed else 128
    S = sol_ref.scores(sol_ref.pool(Qd, bq), sol_ref.pool(Kd, 64), s)
    nkb = S.shape[-1]
    k = sol_ref.topk_count(ratio, nkb)
    sel = sol_ref.route_topk(S, k, prefix, bq, 64 if compressed else None)
    rp, ci, gm = gpu_mask(p, buf)
    rp_ref, ci_ref = sol_ref.to_csr(gm)
    assert np.array_equal(rp, rp_ref) and np.array_equal(ci, ci_ref)
    nqb = gm.shape[2]
    if compressed:
        g = gm[:, heads]
    else:
        assert (gm[:, :, 1::2] == gm[:, :, 0:nqb - nqb % 2:2]).all(), "both halves of a 128-row block share a list"
        g = gm[:, :, ::2][:, heads]
    n_dense = sol_ref.n_blocks(prefix, bq)
    n_sink = sol_ref.n_blocks(prefix, 64) if compressed else 0
    cnt = g.sum(-1)
    assert (cnt[:, :, n_dense:] >= k).all() and (cnt[:, :, n_dense:] <= k + n_sink).all()
    assert (cnt[:, :, :n_dense] == nkb).all() and g[..., :n_sink].all()
    kth = -np.sort(-S, axis=-1)[..., k - 1]
    far = np.abs(S - kth[..., None]) > BAND
    far[:, :, :n_dense] = True
    bad = (g != sel) & far
    assert not bad.any(), f"{int(bad.sum())} top-k mismatches outside the {BAND} band"
    return gm, g, int(((g != sel) & ~far).sum())


def oracle_on_gpu_mask(Qd, Kd, Vd, gm_heads, tau, prefix, lmb, rows=None, topk_ratio=None, compressed=False,
                       qk_int8=False):
    """The oracle's forward pass of the given heads on the GPU's routing mask."""
    if topk_ratio is not None and compressed:
        return sol_ref.sol_forward(Qd, Kd, Vd, prefix=prefix, mask_override=gm_heads, rows=rows,
                                   topk_ratio=topk_ratio, compressed=True, qk_int8=qk_int8, **oracle_modes(lmb))
    if topk_ratio is not None:
        return sol_ref.sol_forward(Qd, Kd, Vd, prefix=prefix, bq=128, mask_override=gm_heads, rows=rows,
                                   topk_ratio=topk_ratio, qk_int8=qk_int8)
    return sol_ref.sol_forward(Qd, Kd, Vd, tau=tau, prefix=prefix, mask_override=gm_heads, rows=rows,
                               qk_int8=qk_int8, **oracle_modes(lmb))


def check_attention(p, buf, Qd, Kd, Vd, gm_heads, heads, tau, prefix, lmb, rows=None, topk_ratio=None,
                    compressed=False, qk_int8=False):
    """O (and lse) of the given heads vs the oracle run on the GPU mask."""
    ref = oracle_on_gpu_mask(Qd, Kd, Vd, gm_heads, tau, prefix, lmb, rows, topk_ratio, compressed, qk_int8)
    O = buf.o[:, :, heads].float().cpu().numpy().astype(np.float64)
    Oref = ref["O"]
    keep = ~np.isnan(Oref)
    err = np.abs(O[keep] - Oref[keep])
    assert keep.any()
    assert err.max() <= MAX_ABS, f"max abs err {err.max()}"
    assert err.mean() <= MEAN_ABS, f"mean abs err {err.mean()}"
    if buf.lse is not None:
        L = buf.lse[:, heads].cpu().numpy().astype(np.float64)
        k2 = ~np.isnan(ref["lse"])
        np.testing.assert_allclose(L[k2], ref["lse"][k2], rtol=0, atol=2e-3)
    return float(err.max()), float(err.mean())


def full_check(w: synth.Workload, heads=None, rows_per_head=None, seed_rows=0):
    """Generate a workload, run it on the GPU, check pool/route/attention on `heads`."""
    q, k, v = synth.generate(w)
    Q, K, V = to_dev(q), to_dev(k), to_dev(v)
    p, buf = run_gpu(Q, K, V, w.tau, w.prefix, w.log_mass_bias, topk_ratio=w.topk_ratio, compressed=w.compressed,
                     qk_int8=w.qk_int8)
    heads = list(range(w.H)) if heads is None else list(heads)
    Qd, Kd, Vd = (synth.bf16_bits_to_f64(x[:, :, heads]) for x in (q, k, v))
    sla = w.topk_ratio is not None and not w.compressed
    qbar, kbar, _ = check_pool(p, buf, Qd, Kd, Vd, heads, w.log_mass_bias, w.prefix, topk=sla)
    if w.topk_ratio is not None:
        _, g128, flips = check_route_topk(p, buf, Qd, Kd, heads, w.topk_ratio, w.prefix, w.compressed)
    else:
        gm, flips = check_route(p, buf, qbar, kbar, heads, w.tau, w.prefix)
    rows = None
    if rows_per_head:
        rng = np.random.default_rng(seed_rows)
        rows = {(b, hh): np.sort(rng.choice(w.N, size=min(rows_per_head, w.N), replace=False))
                for b in range(w.B) for hh in range(len(heads))}
    mask = g128 if w.topk_ratio is not None else gm[:, heads]
    errs = check_attention(p, buf, Qd, Kd, Vd, mask, heads, w.tau, w.prefix, w.log_mass_bias, rows,
                           topk_ratio=w.topk_ratio, compressed=w.compressed, qk_int8=w.qk_int8)
    return dict(flips=flips, errs=errs, nnz=int(buf.row_ptr[-1].item()), p=p, buf=buf, mask=mask, heads=heads,
                Qd=Qd, Kd=Kd, Vd=Vd, rows=rows)
