"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle."""
import dataclasses
import math

import numpy as np
import pytest
import torch

from block_sparse_video_sol_b200 import synth
from oracle import sol_ref
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from block_sparse_video_sol_b200 import build
    build.build()


def test_tiny_workload_full():
    r = parity.full_check(synth.tiny())
    assert r["flips"] <= 2


@pytest.mark.parametrize("lmb", [0, 1, 2])
def test_ragged_prefix_batch2_d64(lmb):
    # N = 1000 (tail block of 40 rows), prefix 100 (mixed block 1), B = 2
    w = synth.Workload("ragged", B=2, H=3, N=1000, D=64, grid=(9, 10, 10), n_topics=8, prefix=100,
                       tau=0.5, seed=7, log_mass_bias=lmb)
    parity.full_check(w)


@pytest.mark.parametrize("lmb", [0, 1, 2])
def test_ragged_prefix_d128(lmb):
    w = synth.Workload("ragged128", B=1, H=4, N=777, D=128, grid=(4, 1, 191), n_topics=8, prefix=13,
                       tau=1.0, seed=8, log_mass_bias=lmb)
    parity.full_check(w)


def test_h56_n4096_full():
    r = parity.full_check(synth.h56_n4096())
    nb = 64
    dens = r["nnz"] / (56 * nb * nb)
    assert 0.05 < dens < 0.3


@pytest.mark.parametrize("tau", [0.5, 2.0])
@pytest.mark.parametrize("lmb", [0, 1, 2])
def test_tau_sweep_n8192(tau, lmb):
    # the density sweep of the length-sweep workload: tau sets how many blocks
    # each query block takes exactly, hence the mix of blocks one or both of a
    # tile's two query blocks need (the order the kernel walks them in)
    w = synth.h56_sweep(8192, tau=tau, log_mass_bias=lmb)
    r = parity.full_check(w, heads=[0, 23, 55])
    nb = 8192 // 64
    dens = r["nnz"] / (56 * nb * nb)
    assert (0.2 < dens < 0.5) if tau == 0.5 else (0.005 < dens < 0.1)


@pytest.mark.parametrize("B,N,H,prefix,tau,grid", [(1, 30001, 2, 200, 1.0, (1, 17, 1753)),
                                                   (2, 5000, 3, 0, 0.5, (5, 20, 50)),
                                                   (1, 32768, 1, 64, 2.0, (8, 8, 511)),
                                                   (2, 40000, 1, 300, 1.0, (4, 25, 397)),
                                                   (1, 40000, 2, 0, -math.inf, (16, 25, 100))])
def test_tensor_core_routing_ragged(B, N, H, prefix, tau, grid):
    """Threshold routing takes its scores from the tensor cores for D = 128 and up to 1024 key
    blocks.  Cases: a partial last 128-block chunk of k-bar and a partial last mask word (469
    key blocks), a partial last 128-row query tile, two batch entries, sinks and dense rows, the
    full 512 key blocks, and 625 key blocks (two halves of the row, the second one a single
    partial chunk), also with tau = -inf (every block exact).  The mask must match the oracle
    outside the 1e-4 band."""
    w = synth.Workload("rt", B=B, H=H, N=N, D=128, grid=grid, n_topics=8, prefix=prefix, tau=tau, seed=31)
    q, k, v = synth.generate(w)
    p, buf = parity.run_gpu(parity.to_dev(q), parity.to_dev(k), parity.to_dev(v), tau, prefix, 0)
    heads = list(range(H))
    Qd, Kd, Vd = (synth.bf16_bits_to_f64(x) for x in (q, k, v))
    qbar, kbar, _ = parity.check_pool(p, buf, Qd, Kd, Vd, heads, 0, prefix)
    _, flips = parity.check_route(p, buf, qbar, kbar, heads, tau, prefix)
    print(f"decisions that differ inside the band: {flips}")


def test_all_exact_matches_dense_sdpa():
    w = synth.Workload("dense", B=1, H=2, N=700, D=128, grid=(7, 10, 10), n_topics=4, tau=-math.inf, seed=9)
    q, k, v = synth.generate(w)
    Q, K, V = parity.to_dev(q), parity.to_dev(k), parity.to_dev(v)
    p, buf = parity.run_gpu(Q, K, V, -math.inf, 0, False)
    assert int(buf.row_ptr[-1]) == 2 * 11 * 11
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q.float().transpose(1, 2), K.float().transpose(1, 2), V.float().transpose(1, 2)).transpose(1, 2)
    err = (buf.o.float() - ref).abs()
    assert err.max().item() <= parity.MAX_ABS and err.mean().item() <= parity.MEAN_ABS


def test_prefix_equals_n_is_dense():
    w = synth.Workload("alldense", B=1, H=2, N=300, D=64, grid=(3, 10, 10), n_topics=4, seed=10)
    q, k, v = synth.generate(w)
    Q, K, V = parity.to_dev(q), parity.to_dev(k), parity.to_dev(v)
    p, buf = parity.run_gpu(Q, K, V, 1.0, 300, True)
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q.float().transpose(1, 2), K.float().transpose(1, 2), V.float().transpose(1, 2)).transpose(1, 2)
    assert (buf.o.float() - ref).abs().max().item() <= parity.MAX_ABS


def test_fused_qkv_strided_views():
    w = synth.Workload("fused", B=2, H=4, N=640, D=128, grid=(4, 10, 16), n_topics=8, tau=1.0, seed=11)
    q, k, v = synth.generate(w)
    qkv = torch.empty((2, 640, 3, 4, 128), dtype=torch.bfloat16, device="cuda")
    qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2] = parity.to_dev(q), parity.to_dev(k), parity.to_dev(v)
    Qv, Kv, Vv = qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2]
    assert Qv.stride(1) == 3 * 4 * 128
    p, buf = parity.run_gpu(Qv, Kv, Vv, 1.0, 0, False)
    p2, buf2 = parity.run_gpu(parity.to_dev(q), parity.to_dev(k), parity.to_dev(v), 1.0, 0, False)
    assert torch.equal(buf.row_ptr, buf2.row_ptr)
    assert torch.equal(buf.o, buf2.o)


@pytest.mark.parametrize("N", [1, 5, 63, 64, 65])
@pytest.mark.parametrize("lmb", [0, 2])
def test_small_and_single_block(N, lmb):
    w = synth.Workload(f"small{N}", B=1, H=2, N=N, D=64, grid=(1, 1, N), n_topics=2, tau=0.0, seed=12 + N,
                       log_mass_bias=lmb)
    parity.full_check(w)


@pytest.mark.parametrize("N,D,prefix", [(8192, 128, 0), (5000, 64, 321)])
def test_reweight_anchor_queries_match_dense(N, D, prefix):
    """With every query row equal to the anchor, the weighted summaries give each
    centroid block its exact contribution, so the sparse output equals dense
    attention whatever the routing (fp32 SDPA on the same bf16 inputs)."""
    w = synth.Workload("anchorq", B=1, H=4, N=N, D=D, grid=(1, 1, N - prefix), n_topics=16, prefix=prefix,
                       tau=1.0, seed=14)
    q, k, v = synth.generate(w)
    Q, K, V = parity.to_dev(q), parity.to_dev(k), parity.to_dev(v)
    Q = Q[:, :1].expand_as(Q).contiguous()
    p, buf = parity.run_gpu(Q, K, V, 1.0, prefix, 2)
    nb = -(-N // 64)
    assert int(buf.row_ptr[-1]) < 0.5 * 4 * nb * nb          # most blocks are centroid terms
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q.float().transpose(1, 2), K.float().transpose(1, 2), V.float().transpose(1, 2)).transpose(1, 2)
    err = (buf.o.float() - ref).abs()
    assert err.max().item() <= parity.MAX_ABS and err.mean().item() <= parity.MEAN_ABS
    # the mean-pooled summaries with the bias do not have this property
    p1, buf1 = parity.run_gpu(Q, K, V, 1.0, prefix, 1)
    assert (buf1.o.float() - ref).abs().mean().item() > 2 * err.mean().item()


def test_empty_problem_is_noop():
    from block_sparse_video_sol_b200 import sol
    p = sol.make_params(1, 0, 4, 128)
    sol.sol_pool(p, None, None, None, torch.empty(1, dtype=torch.uint8, device="cuda"))
    sol.sol_last_device_status()


def test_max_key_blocks():
    # N = 65536 is the longest sequence the routing kernel takes (1024 key blocks)
    w = synth.Workload("maxN", B=1, H=2, N=65536, D=128, grid=(64, 32, 32), n_topics=128, seed=13)
    parity.full_check(w, rows_per_head=300)


@pytest.mark.parametrize("kw", [dict(topk_ratio=0.1), dict(topk_ratio=0.1, compressed=True, log_mass_bias=2)])
def test_max_key_blocks_topk(kw):
    # 1024 key blocks: the Top-K selection's widest register layout (32 keys per lane)
    w = synth.Workload("maxN_topk", B=1, H=2, N=65536, D=128, grid=(64, 32, 32), n_topics=128, seed=13, **kw)
    parity.full_check(w, rows_per_head=300)


def test_bad_csr_entry_is_reported_not_read():
    from block_sparse_video_sol_b200 import sol
    w = synth.tiny()
    q, k, v = synth.generate(w)
    Q, K, V = parity.to_dev(q), parity.to_dev(k), parity.to_dev(v)
    p, buf = parity.run_gpu(Q, K, V, 1.0, 0, False)
    bad = buf.col_idx.clone()
    bad[0] = 10 ** 6
    sol.sol_attn_fwd(p, Q, K, V, buf.ws, buf.row_ptr, bad, buf.o)
    with pytest.raises(sol.SolError) as e:
        sol.sol_last_device_status()
    assert e.value.status == sol.SOL_ERR_INVALID_ARG
    sol.sol_last_device_status()   # cleared


@pytest.mark.slow
def test_h56_n32768_sampled():
    # full problem on the GPU; oracle on two heads, sampled rows
    w = synth.h56_sweep(32768)
    r = parity.full_check(w, heads=[0, 41], rows_per_head=256)
    assert r["flips"] <= 20


@pytest.mark.slow
@pytest.mark.parametrize("lmb", [0, 1, 2])
def test_joint_sequence_sampled(lmb):
    w = synth.h56_joint()
    if lmb:
        w = synth.Workload(w.name + synth.mode_suffix(lmb), w.B, w.H, w.N, w.D, w.grid, w.n_topics, w.prefix,
                           w.tau, w.seed, lmb)
    r = parity.full_check(w, heads=[3, 55], rows_per_head=256, seed_rows=1)
    assert r["flips"] <= 20


# ---------------------------------------------------------------- Top-K routing (SLA variant)
@pytest.mark.parametrize("ratio", [0.2, 0.5])
def test_topk_ragged_prefix_batch2_d64(ratio):
    w = synth.Workload("topk_ragged", B=2, H=3, N=1000, D=64, grid=(9, 10, 10), n_topics=8, prefix=100,
                       seed=21, topk_ratio=ratio)
    parity.full_check(w)


def test_topk_odd_blocks_d128():
    # 13 query blocks of 64 rows: the last 128-row block has one half
    w = synth.Workload("topk_odd", B=1, H=4, N=777, D=128, grid=(4, 1, 191), n_topics=8, prefix=13,
                       seed=22, topk_ratio=0.15)
    parity.full_check(w)


@pytest.mark.parametrize("N", [1, 5, 63, 64, 65, 129])
def test_topk_small(N):
    w = synth.Workload(f"topk_small{N}", B=1, H=2, N=N, D=64, grid=(1, 1, N), n_topics=2, seed=23 + N,
                       topk_ratio=0.3)
    parity.full_check(w)


def test_topk_h56_n8192():
    w = dataclasses.replace(synth.h56_sweep(8192), name="h56_n8192_sla15", topk_ratio=0.15)
    r = parity.full_check(w, heads=[0, 23, 55])
    nb = 8192 // 64
    assert r["nnz"] == 56 * nb * sol_ref.topk_count(0.15, nb)


def test_topk_ties_take_lower_index():
    # identical key rows give every key block the same score: the first k blocks are kept
    from block_sparse_video_sol_b200 import sol
    w = synth.Workload("ties", B=1, H=2, N=640, D=64, grid=(1, 1, 640), n_topics=4, seed=24)
    q, k, v = synth.generate(w)
    k[:] = k[:, :1]
    Q, K, V = parity.to_dev(q), parity.to_dev(k), parity.to_dev(v)
    p, buf = parity.run_gpu(Q, K, V, 1.0, 0, 0, topk_ratio=0.3)
    rp, ci, gm = parity.gpu_mask(p, buf)
    kk = sol_ref.topk_count(0.3, 10)
    assert kk == 3 and gm[..., :kk].all() and not gm[..., kk:].any()


def test_topk_ratio_one_is_dense_sdpa():
    w = synth.Workload("topk_dense", B=1, H=2, N=700, D=128, grid=(67, 10, 1), n_topics=4, prefix=30, seed=25)
    q, k, v = synth.generate(w)
    Q, K, V = parity.to_dev(q), parity.to_dev(k), parity.to_dev(v)
    p, buf = parity.run_gpu(Q, K, V, 1.0, 30, 0, topk_ratio=1.0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q.float().transpose(1, 2), K.float().transpose(1, 2), V.float().transpose(1, 2)).transpose(1, 2)
    err = (buf.o.float() - ref).abs()
    assert err.max().item() <= parity.MAX_ABS and err.mean().item() <= parity.MEAN_ABS


@pytest.mark.slow
def test_topk_h56_n32768_sampled():
    w = dataclasses.replace(synth.h56_sweep(32768), name="h56_n32768_sla15", topk_ratio=0.15)
    r = parity.full_check(w, heads=[0, 41], rows_per_head=256)
    assert r["flips"] <= 20


@pytest.mark.slow
def test_topk_joint_sequence_sampled():
    w = dataclasses.replace(synth.h56_joint(), name="h56_joint_sla15", topk_ratio=0.15)
    r = parity.full_check(w, heads=[3, 55], rows_per_head=256, seed_rows=2)
    assert r["flips"] <= 20


# ---------------------------------------------------------------- host-buffer entry point
def _host_vs_device(w, heads_per_chunk, pin=True, host_view=None):
    from block_sparse_video_sol_b200 import sol
    q, k, v = synth.generate(w)
    to_host = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
    Qh, Kh, Vh = (to_host(x) for x in (q, k, v))
    if host_view is not None:
        Qh, Kh, Vh = host_view(Qh), host_view(Kh), host_view(Vh)
    if pin:
        Qh, Kh, Vh = (x.pin_memory() for x in (Qh, Kh, Vh))
    B, N, H, D = Qh.shape
    p = sol.make_params(B, N, H, D, tau=w.tau, prefix_len=w.prefix, log_mass_bias=w.log_mass_bias,
                        topk_ratio=w.topk_ratio, in_strides=(Qh.stride(0), Qh.stride(1), Qh.stride(2)))
    Oh = torch.full((B, N, H, D), float("nan"), dtype=torch.bfloat16)
    Oh = Oh.pin_memory() if pin else Oh
    staging = torch.empty(sol.sol_host_staging_bytes(p, heads_per_chunk), dtype=torch.uint8, device="cuda")
    sol.sol_forward_host(p, Qh, Kh, Vh, Oh, staging, heads_per_chunk)
    torch.cuda.synchronize()
    sol.sol_last_device_status()
    pd = sol.make_params(B, N, H, D, tau=w.tau, prefix_len=w.prefix, log_mass_bias=w.log_mass_bias,
                         topk_ratio=w.topk_ratio)
    buf = sol.alloc_buffers(pd, "cuda")
    sol.forward(pd, Qh.contiguous().cuda(), Kh.contiguous().cuda(), Vh.contiguous().cuda(), buf)
    torch.cuda.synchronize()
    assert torch.equal(Oh, buf.o.cpu()), "host pipeline differs from the device path"


@pytest.mark.parametrize("hc", [0, 3, 56])
def test_host_entry_matches_device_h56(hc):
    _host_vs_device(synth.h56_n4096(), hc)


@pytest.mark.parametrize("mode", ["lmb", "rw", "topk"])
def test_host_entry_modes(mode):
    kw = dict(lmb=dict(log_mass_bias=1), rw=dict(log_mass_bias=2), topk=dict(topk_ratio=0.2))[mode]
    w = synth.Workload("host_" + mode, B=2, H=5, N=1000, D=64, grid=(9, 10, 10), n_topics=8, prefix=100, seed=26, **kw)
    _host_vs_device(w, 2)


def test_host_entry_strided_and_pageable():
    w = synth.Workload("host_strided", B=1, H=6, N=640, D=128, grid=(4, 10, 16), n_topics=8, seed=27)
    # every other head of a 12-head host tensor: heads are not adjacent (per-head copies)
    wide = lambda x: torch.stack([x, torch.zeros_like(x)], dim=3).reshape(1, 640, 12, 128)[:, :, 0::2]
    _host_vs_device(w, 4, pin=False, host_view=wide)


# ---------------------------------------------------------------- Top-K with the compressed branch (routing 2)
@pytest.mark.parametrize("lmb", [0, 1, 2])
def test_spark_ragged_prefix_batch2_d64(lmb):
    w = synth.Workload("spark_ragged", B=2, H=3, N=1000, D=64, grid=(9, 10, 10), n_topics=8, prefix=100,
                       seed=31, log_mass_bias=lmb, topk_ratio=0.2, compressed=True)
    parity.full_check(w)


def test_spark_d128_small_and_ties():
    w = synth.Workload("spark_d128", B=1, H=4, N=777, D=128, grid=(4, 1, 191), n_topics=8, prefix=13,
                       seed=32, log_mass_bias=2, topk_ratio=0.1, compressed=True)
    parity.full_check(w)
    for N in (1, 65):
        parity.full_check(synth.Workload(f"spark_small{N}", B=1, H=2, N=N, D=64, grid=(1, 1, N), n_topics=2,
                                         seed=33 + N, topk_ratio=0.5, compressed=True))


def test_spark_h56_n8192():
    w = dataclasses.replace(synth.h56_sweep(8192), name="h56_n8192_spark20", log_mass_bias=2, topk_ratio=0.2,
                            compressed=True)
    parity.full_check(w, heads=[0, 23, 55])


@pytest.mark.slow
def test_spark_joint_sequence_sampled():
    w = dataclasses.replace(synth.h56_joint(), name="h56_joint_spark20", log_mass_bias=2, topk_ratio=0.2,
                            compressed=True)
    r = parity.full_check(w, heads=[3, 55], rows_per_head=256, seed_rows=3)
    assert r["flips"] <= 20


# ---------------------------------------------------------------- CUDA graphs
@pytest.mark.parametrize("kw", [dict(), dict(log_mass_bias=2), dict(topk_ratio=0.2, compressed=True),
                                dict(topk_ratio=0.15)])
def test_forward_captures_into_a_cuda_graph(kw):
    """The entry points allocate nothing and never synchronise, so one forward pass
    captures into a CUDA graph; replays on new inputs equal eager calls bit for bit."""
    from block_sparse_video_sol_b200 import sol
    w = synth.Workload("graph", B=1, H=4, N=2048, D=128, grid=(2, 974, 1), n_topics=16, prefix=100, seed=34)
    q, k, v = (parity.to_dev(x) for x in synth.generate(w))
    p = sol.make_params(1, 2048, 4, 128, tau=1.0, prefix_len=100, **kw)
    buf = sol.alloc_buffers(p, "cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        sol.forward(p, q, k, v, buf, stream=s)   # first call per device before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        sol.forward(p, q, k, v, buf, stream=s)
    ref_buf = sol.alloc_buffers(p, "cuda")
    for seed in (35, 36):
        w2 = dataclasses.replace(w, seed=seed)
        q2, k2, v2 = (parity.to_dev(x) for x in synth.generate(w2))
        q.copy_(q2), k.copy_(k2), v.copy_(v2)
        g.replay()
        sol.forward(p, q2, k2, v2, ref_buf)
        torch.cuda.synchronize()
        assert torch.equal(buf.o, ref_buf.o)
        assert torch.equal(buf.row_ptr, ref_buf.row_ptr)
    sol.sol_last_device_status()


# ---------------------------------------------------------------- head split (one call over several GPUs)
@pytest.mark.parametrize("kw", [dict(), dict(prefix_len=100, log_mass_bias=2, topk_ratio=0.2, compressed=True),
                                dict(topk_ratio=0.15)])
def test_head_runs_equal_the_whole_call(kw):
    """Heads are independent in every stage: calls on the head runs [0, 21) and [21, 56)
    of the same tensors (H = the run's length, base pointers offset by h0 heads, strides
    kept) give the whole call's O and LSE bit for bit, and their CSR lists, concatenated,
    are the whole call's.  This is how one call is split over GPUs."""
    from block_sparse_video_sol_b200 import sol
    w = synth.h56_n4096()
    q, k, v = (parity.to_dev(x) for x in synth.generate(w))
    B, N, H, D = q.shape
    whole_p = sol.make_params(B, N, H, D, **kw)
    whole = sol.alloc_buffers(whole_p, "cuda", with_lse=True)
    sol.forward(whole_p, q, k, v, whole)
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, N), float("nan"), device="cuda")
    rp_all, ci_all, base = [], [], 0
    for h0, h1 in ((0, 21), (21, 56)):
        p = sol.make_params(B, N, h1 - h0, D, in_strides=q.stride()[:3], out_strides=o.stride()[:3], **kw)
        buf = sol.alloc_buffers(p, "cuda")
        qs, ks, vs, os_ = (x[:, :, h0:h1] for x in (q, k, v, o))
        sol.sol_pool(p, qs, ks, vs, buf.ws)
        sol.sol_route(p, buf.ws, buf.row_ptr, buf.col_idx)
        part_lse = torch.empty((B, h1 - h0, N), device="cuda")
        sol.sol_attn_fwd(p, qs, ks, vs, buf.ws, buf.row_ptr, buf.col_idx, os_, part_lse)
        lse[:, h0:h1] = part_lse
        nnz = int(buf.row_ptr[-1])
        rp_all.append(buf.row_ptr[:-1] + base)
        ci_all.append(buf.col_idx[:nnz])
        base += nnz
    sol.sol_last_device_status()
    assert torch.equal(o, whole.o)
    assert torch.equal(lse, whole.lse)
    rp = torch.cat(rp_all + [torch.tensor([base], dtype=torch.int32, device="cuda")])
    assert torch.equal(rp, whole.row_ptr)
    assert torch.equal(torch.cat(ci_all), whole.col_idx[:base])
