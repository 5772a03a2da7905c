"""GPU parity of the adaptive partition (sol_reblock), the row gathers and the
reblocked forward pass, against the oracle's step 9.

* planted hierarchies (synth.planted_clusters) of 2 to 9 levels, up to 32,768
  partitioned rows: every split is far from a tie, so the GPU order must
  equal the oracle's bit for bit;
* topic and random inputs, up to the full 32,768-row and 38,247-row
  workloads: the GPU order is cut back into its hierarchy and every split,
  at every level, is checked on its own members against the oracle's
  projections (tests/reblock_check.py): every left row projects at or below
  every right row, outside a band of 1e-4 of the group's projection range
  (fp32 against fp64 whitening and power steps); and the reblocked forward
  pass must match the oracle run on the GPU's order and mask (the usual
  2e-2 max / 2e-3 mean bound);
* gathers and scatters are exact copies, and an all-exact reblocked pass is
  dense attention (checked against torch SDPA in fp32).
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_video_sol_b200 import synth
from oracle import sol_ref
from tests.parity import MAX_ABS, MEAN_ABS, to_dev
from tests.reblock_check import check_splits

SPLIT_BAND = 1e-4   # of a group's projection range: fp32 power steps against fp64

pytestmark = pytest.mark.gpu


def _gpu_perm(q, k, prefix, D):
    from block_sparse_video_sol_b200 import sol
    B, N, H, _ = q.shape
    p = sol.make_params(B, N, H, D, prefix_len=prefix)
    ws = torch.empty(max(1, sol.sol_reblock_workspace_bytes(p)), dtype=torch.uint8, device="cuda")
    perm = torch.empty(B * H * N, dtype=torch.int32, device="cuda")
    sol.sol_reblock(p, q, k, ws, perm)
    sol.sol_last_device_status()
    return perm.cpu().numpy().astype(np.int64).reshape(B, H, N)


@pytest.mark.parametrize("levels,D,H,prefix,noise", [(2, 64, 2, 0, 0.05), (4, 64, 3, 0, 0.05), (5, 128, 2, 100, 0.05),
                                                     (6, 128, 1, 64, 0.05), (3, 64, 2, 1, 0.05),
                                                     (8, 128, 2, 100, 0.004), (9, 128, 1, 0, 0.004),
                                                     (9, 128, 2, 100, 0.004)])
def test_planted_partition_is_the_oracles(levels, D, H, prefix, noise):
    """8 and 9 levels are the depth of the 16,384- and 32,768-row workloads (groups of up to
    32,768 rows); their finest split separates centers 2 * 16 / 2^8 apart, so the noise is
    smaller there."""
    q, k, v, cid, n_fix = synth.planted_clusters(levels, D, H=H, prefix=prefix, seed=10 * levels + D, noise=noise)
    perm = _gpu_perm(to_dev(q), to_dev(k), prefix, D)
    ref = sol_ref.reblock_partition(synth.bf16_bits_to_f64(q), synth.bf16_bits_to_f64(k), prefix)
    assert np.array_equal(perm, ref)
    for h in range(H):   # and the clusters are the leaves
        for s in range(n_fix, perm.shape[-1], 64):
            assert len(set(cid[0, h][perm[0, h, s:s + 64] - n_fix].tolist())) == 1


def _valid(perm, N, prefix):
    n_fix = min(N, 64 * (-(-prefix // 64)))
    for row in perm.reshape(-1, N):
        assert np.array_equal(np.sort(row), np.arange(N))
        assert np.array_equal(row[:n_fix], np.arange(n_fix))
        for s in range(n_fix, N, 64):
            assert np.all(np.diff(row[s:s + 64]) > 0)


def _check_every_split(Qd, Kd, perm, prefix, min_exact):
    """Every split of the GPU's hierarchy against the oracle's projections of its own
    members; at least ``min_exact`` of the splits pick the oracle's left part exactly
    (the others differ only inside the band, where fp32 and fp64 may order rows apart)."""
    rep = check_splits(Qd, Kd, perm, prefix, band=SPLIT_BAND)
    print(f"splits checked {rep.groups}, exact {rep.exact}, levels {rep.levels}, worst gap/range {rep.worst:.2e}")
    assert rep.groups == 0 or rep.exact >= min_exact * rep.groups, rep
    return rep


@pytest.mark.parametrize("prefix", [0, 100])
def test_topic_partition_splits_like_the_oracle(prefix):
    w = synth.tiny()
    q, k, _ = synth.generate(w)
    perm = _gpu_perm(to_dev(q), to_dev(k), prefix, w.D)
    _valid(perm, w.N, prefix)
    _check_every_split(synth.bf16_bits_to_f64(q), synth.bf16_bits_to_f64(k), perm, prefix, 0.95)


@pytest.mark.slow
@pytest.mark.parametrize("which", ["h56_n32768", "h56_joint"])
def test_full_size_partition_splits_like_the_oracle(which):
    """The workloads the bench times (9 and 10 levels, groups of up to 32,768 and 35,815 rows;
    the joint sequence also has a ragged last leaf and 2,432 rows of prefix blocks), two heads."""
    w = synth.h56_sweep(32768) if which == "h56_n32768" else synth.h56_joint()
    q, k, _ = synth.generate(w, heads=[0, 1])
    perm = _gpu_perm(to_dev(q), to_dev(k), w.prefix, w.D)
    _valid(perm, w.N, w.prefix)
    rep = _check_every_split(synth.bf16_bits_to_f64(q), synth.bf16_bits_to_f64(k), perm, w.prefix, 0.95)
    n_v = w.N - 64 * (-(-w.prefix // 64))
    assert rep.levels == math.ceil(math.log2(-(-n_v // 64))) == (9 if w.prefix == 0 else 10)


def test_gather_scatter_are_exact_copies():
    from block_sparse_video_sol_b200 import sol
    B, N, H, D = 2, 300, 3, 128
    x = torch.randn(B, N, H, D, device="cuda").to(torch.bfloat16)
    perm = torch.stack([torch.randperm(N) for _ in range(B * H)]).to(torch.int32).cuda()
    p = sol.make_params(B, N, H, D)
    xp = torch.empty(B, H, N, D, dtype=torch.bfloat16, device="cuda")
    sol.sol_gather_rows(p, perm, x, xp)
    pr = perm.view(B, H, N).long()
    want = torch.stack([torch.stack([x[b, pr[b, h], h] for h in range(H)]) for b in range(B)])
    assert torch.equal(xp, want)
    y = torch.zeros_like(x)
    sol.sol_scatter_rows(p, perm, xp, y)
    sol.sol_last_device_status()
    assert torch.equal(y, x)


@pytest.mark.parametrize("kw", [dict(), dict(log_mass_bias=1, prefix=100), dict(topk_ratio=0.2, compressed=True,
                                                                                  log_mass_bias=2)])
def test_reblocked_forward_matches_the_oracle(kw):
    from block_sparse_video_sol_b200 import sol
    w = synth.tiny()
    q, k, v = synth.generate(w)
    Q, K, V = to_dev(q), to_dev(k), to_dev(v)
    prefix = kw.get("prefix", 0)
    p = sol.make_params(w.B, w.N, w.H, w.D, tau=w.tau, prefix_len=prefix, log_mass_bias=kw.get("log_mass_bias", 0),
                        topk_ratio=kw.get("topk_ratio"), compressed=kw.get("compressed", False))
    rb = sol.alloc_reblock(p, Q.device)
    o = torch.empty_like(Q)
    sol.forward_reblocked(p, Q, K, V, o, rb)
    sol.sol_last_device_status()
    perm = rb.perm.cpu().numpy().astype(np.int64).reshape(w.B, w.H, w.N)
    _valid(perm, w.N, prefix)
    nb = -(-w.N // 64)
    rp = rb.buf.row_ptr.cpu().numpy().astype(np.int64)
    ci = rb.buf.col_idx[:int(rp[-1])].cpu().numpy().astype(np.int64)
    gm = sol_ref.from_csr(rp, ci, (w.B, w.H, nb, nb))
    Qd, Kd, Vd = (synth.bf16_bits_to_f64(x) for x in (q, k, v))
    lmb = kw.get("log_mass_bias", 0)
    ref = sol_ref.sol_forward(Qd, Kd, Vd, tau=w.tau, prefix=prefix, reblock=True, perm_override=perm,
                              mask_override=gm, log_mass_bias_on=lmb == 1, reweight_on=lmb == 2,
                              topk_ratio=kw.get("topk_ratio"), compressed=kw.get("compressed", False))
    err = np.abs(o.float().cpu().numpy() - ref["O"])
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    # the head-major output holds the same values in the partition's order
    pt = torch.from_numpy(perm).cuda()
    for b in range(w.B):
        for h in range(w.H):
            assert torch.equal(rb.buf.o[b, h], o[b, pt[b, h], h])


def test_all_exact_reblocked_pass_is_dense_attention():
    from block_sparse_video_sol_b200 import sol
    w = synth.tiny()
    q, k, v = synth.generate(w)
    Q, K, V = to_dev(q), to_dev(k), to_dev(v)
    o, rb = sol.attention(Q, K, V, tau=-math.inf, reblock=True)
    sol.sol_last_device_status()
    ref = torch.nn.functional.scaled_dot_product_attention(*(x.float().transpose(1, 2) for x in (Q, K, V)))
    err = (o.float() - ref.transpose(1, 2)).abs()
    assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS
    assert not torch.equal(rb.perm[:w.N].cpu(), torch.arange(w.N, dtype=torch.int32))


@pytest.mark.parametrize("N,D,prefix", [(1000, 64, 70), (777, 128, 13)])
def test_ragged_reblocked_forward(N, D, prefix):
    """Ragged lengths: a partial last leaf, a prefix that is not block aligned."""
    from block_sparse_video_sol_b200 import sol
    B, H = 1, 2
    q, k, v = (synth.random_bf16((B, N, H, D), seed=s) for s in (21, 22, 23))
    Q, K, V = to_dev(q), to_dev(k), to_dev(v)
    p = sol.make_params(B, N, H, D, tau=1.0, prefix_len=prefix)
    rb = sol.alloc_reblock(p, Q.device)
    o = torch.empty_like(Q)
    sol.forward_reblocked(p, Q, K, V, o, rb)
    sol.sol_last_device_status()
    perm = rb.perm.cpu().numpy().astype(np.int64).reshape(B, H, N)
    _valid(perm, N, prefix)
    Qd, Kd, Vd = (synth.bf16_bits_to_f64(x) for x in (q, k, v))
    _check_every_split(Qd, Kd, perm, prefix, 0.95)
    nb = -(-N // 64)
    rp = rb.buf.row_ptr.cpu().numpy().astype(np.int64)
    ci = rb.buf.col_idx[:int(rp[-1])].cpu().numpy().astype(np.int64)
    gm = sol_ref.from_csr(rp, ci, (B, H, nb, nb))
    ref = sol_ref.sol_forward(Qd, Kd, Vd, tau=1.0, prefix=prefix, reblock=True, perm_override=perm, mask_override=gm)
    err = np.abs(o.float().cpu().numpy() - ref["O"])
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())


def test_batch2_gram_levels_split_like_the_oracle():
    """B = 2 through the Gram-axis levels (groups of 512 rows or more, D = 128): 2,036 video
    rows per head (three Gram levels, then the streamed levels), a prefix that is not block
    aligned, and two heads per batch entry; every split is checked on its own members."""
    B, N, H, D, prefix = 2, 2100, 2, 128, 40
    q, k = (synth.random_bf16((B, N, H, D), seed=s) for s in (41, 42))
    perm = _gpu_perm(to_dev(q), to_dev(k), prefix, D)
    _valid(perm, N, prefix)
    rep = _check_every_split(synth.bf16_bits_to_f64(q), synth.bf16_bits_to_f64(k), perm, prefix, 0.95)
    assert rep.levels == 5 and rep.groups == B * H * 31


def test_all_prefix_and_empty_partitions():
    """P = N: nothing to partition, the order is the identity; N = 0: nothing runs."""
    from block_sparse_video_sol_b200 import sol
    N, H, D = 300, 2, 64
    q, k = (to_dev(synth.random_bf16((1, N, H, D), seed=s)) for s in (31, 32))
    perm = _gpu_perm(q, k, N, D)
    assert np.array_equal(perm, np.tile(np.arange(N), (1, H, 1)))
    p0 = sol.make_params(1, 0, H, D)
    assert sol.sol_reblock_workspace_bytes(p0) == 0
    e = torch.empty(16, dtype=torch.int32, device="cuda")
    sol.sol_reblock(p0, q, k, torch.empty(1, dtype=torch.uint8, device="cuda"), e)
    sol.sol_last_device_status()
