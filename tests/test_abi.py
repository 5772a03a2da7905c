"""The C-ABI library without a GPU: it loads, exports every declared entry
point, and validates arguments synchronously (no compute is launched)."""
import ctypes
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def sol():
    from block_sparse_video_sol_b200 import build
    build.build()
    from block_sparse_video_sol_b200 import sol as mod
    return mod


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(sol_[a-z_0-9]+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported(sol):
    declared = _declared()
    assert {"sol_pool", "sol_route", "sol_attn_fwd"} <= declared
    for name in declared:
        assert hasattr(sol.lib, name), name
    assert declared == set(sol.EXPORTS)


def test_fault_hook_is_inert_in_the_product_library(sol):
    assert sol.lib.sol_debug_drop_arrive(0) == sol.SOL_ERR_UNSUPPORTED
    assert "SOL_FAULT_TEST" in sol.lib.sol_last_error_text().decode()


def test_fault_test_library_builds_and_exports_the_same_entry_points(sol):
    from block_sparse_video_sol_b200 import build
    fault = ctypes.CDLL(build.build(fault_test=True))
    for name in sol.EXPORTS:
        assert hasattr(fault, name), name


def test_status_strings(sol):
    for code, name in enumerate(["SOL_OK", "SOL_ERR_INVALID_ARG", "SOL_ERR_UNSUPPORTED", "SOL_ERR_WORKSPACE",
                                 "SOL_ERR_CUDA", "SOL_ERR_TIMEOUT"]):
        assert sol.lib.sol_status_string(code).decode() == name


def test_workspace_sizes(sol):
    p = sol.make_params(1, 32768, 56, 128)
    nb = 512
    ws = sol.sol_workspace_bytes(p)
    # two fp32 and two bf16 centroid arrays and the attention plans (a 16-int header, two
    # bitmaps of 16 words and a union list of up to 512 entries per 128-row query tile) dominate
    plans = 56 * (nb // 2) * ((16 + 2 * 16 + nb + 3) // 4 * 4) * 4
    assert ws >= 56 * nb * 128 * (4 + 4 + 2 + 2) + plans
    assert ws < (56 * nb * 128 * 12 + plans) * 1.05
    assert sol.sol_col_capacity(p) == 56 * nb * nb
    off = sol.sol_workspace_offsets(p)
    assert off == sorted(off) and all(o % 256 == 0 for o in off) and off[-1] < ws
    assert sol.sol_workspace_bytes(sol.make_params(1, 0, 56, 128)) == 0
    assert sol.sol_workspace_bytes(sol.make_params(1, 100, 56, 96)) == 0   # bad head dim


def _call_pool(sol, p, ws_bytes=1 << 30, ptr=4096):
    return sol.lib.sol_pool(ctypes.byref(p), ptr, ptr, ptr, ptr, ws_bytes, None)


def test_argument_validation_is_synchronous(sol):
    ok = sol.make_params(1, 1000, 4, 128)
    assert _call_pool(sol, sol.make_params(1, 1000, 4, 96)) == sol.SOL_ERR_UNSUPPORTED
    assert _call_pool(sol, sol.make_params(1, 1000, 4, 128, q_block=32, k_block=32)) == sol.SOL_ERR_UNSUPPORTED
    assert _call_pool(sol, sol.make_params(1, 1000, 4, 128, tau=math.nan)) == sol.SOL_ERR_INVALID_ARG
    assert _call_pool(sol, sol.make_params(1, 1000, 4, 128, tau=math.inf)) == sol.SOL_ERR_INVALID_ARG
    assert _call_pool(sol, sol.make_params(1, 1000, 4, 128, prefix_len=1001)) == sol.SOL_ERR_INVALID_ARG
    assert _call_pool(sol, sol.make_params(1, 1000, 4, 128, in_strides=(512000, 516, 128))) == sol.SOL_ERR_INVALID_ARG
    assert _call_pool(sol, sol.make_params(1, 70000, 4, 128)) == sol.SOL_ERR_UNSUPPORTED
    for mode in (-1, 3):
        assert _call_pool(sol, sol.make_params(1, 1000, 4, 128, log_mass_bias=mode)) == sol.SOL_ERR_INVALID_ARG
        assert "log_mass_bias" in sol.lib.sol_last_error_text().decode()
    bad = sol.make_params(1, 1000, 4, 128, topk_ratio=0.2)
    bad.routing = 3
    assert _call_pool(sol, bad) == sol.SOL_ERR_INVALID_ARG
    # top-k with the compressed branch: 64-row query blocks, every centroid mode
    spark = lambda **kw: sol.make_params(1, 1000, 4, 128, topk_ratio=0.2, compressed=True, **kw)
    assert spark().routing == 2 and spark().q_block == 64
    assert _call_pool(sol, spark(q_block=128)) == sol.SOL_ERR_UNSUPPORTED
    assert _call_pool(sol, spark(log_mass_bias=2), ws_bytes=10) == sol.SOL_ERR_WORKSPACE
    for r in (0.0, 1.5, float("nan")):
        assert _call_pool(sol, sol.make_params(1, 1000, 4, 128, topk_ratio=r)) == sol.SOL_ERR_INVALID_ARG
    assert _call_pool(sol, sol.make_params(1, 1000, 4, 128, topk_ratio=0.2, q_block=64)) == sol.SOL_ERR_UNSUPPORTED
    assert _call_pool(sol, sol.make_params(1, 1000, 4, 128, topk_ratio=0.2, log_mass_bias=1)) == sol.SOL_ERR_INVALID_ARG
    assert _call_pool(sol, sol.make_params(1, 1000, 4, 128, topk_ratio=0.2), ws_bytes=10) == sol.SOL_ERR_WORKSPACE
    for mode in (1, 2):   # valid modes pass validation and reach the size check
        assert _call_pool(sol, sol.make_params(1, 1000, 4, 128, log_mass_bias=mode), ws_bytes=10) \
            == sol.SOL_ERR_WORKSPACE
    assert _call_pool(sol, ok, ptr=4100) == sol.SOL_ERR_INVALID_ARG          # misaligned
    assert _call_pool(sol, ok, ws_bytes=10) == sol.SOL_ERR_WORKSPACE
    assert sol.lib.sol_pool(ctypes.byref(ok), None, 4096, 4096, 4096, 1 << 30, None) == sol.SOL_ERR_INVALID_ARG
    assert "NULL" in sol.lib.sol_last_error_text().decode()
    assert sol.lib.sol_pool(None, None, None, None, None, 0, None) == sol.SOL_ERR_INVALID_ARG
    # an empty problem is valid and enqueues nothing
    assert _call_pool(sol, sol.make_params(0, 1000, 4, 128), ptr=0) == sol.SOL_OK
    assert sol.lib.sol_route(ctypes.byref(sol.make_params(1, 0, 4, 128)), None, 0, None, None, None) == sol.SOL_OK
    assert sol.lib.sol_attn_fwd(ctypes.byref(sol.make_params(1, 0, 4, 64)), None, None, None, None, 0,
                                None, None, None, None, None) == sol.SOL_OK


def test_no_gpu_reports_cuda_error(sol):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st = _call_pool(sol, sol.make_params(1, 1000, 4, 128))
    assert st in (sol.SOL_ERR_CUDA, sol.SOL_ERR_UNSUPPORTED)


def test_host_entry_validation(sol):
    p = sol.make_params(1, 1000, 4, 128)
    one = sol.lib.sol_host_staging_bytes(ctypes.byref(p), 1)
    four = sol.lib.sol_host_staging_bytes(ctypes.byref(p), 4)
    assert 0 < one < four
    # a full 4-head chunk holds Q, K, V, O of the whole problem in each of two slots
    assert four >= 2 * 4 * 1000 * 4 * 128 * 2
    assert sol.lib.sol_host_staging_bytes(ctypes.byref(p), 0) == sol.lib.sol_host_staging_bytes(ctypes.byref(p), 4)
    assert sol.lib.sol_host_staging_bytes(ctypes.byref(p), -1) == 0
    h = 4096
    assert sol.lib.sol_forward_host(ctypes.byref(p), h, h, h, h, -1, h, 1 << 40, None) == sol.SOL_ERR_INVALID_ARG
    assert sol.lib.sol_forward_host(ctypes.byref(p), None, h, h, h, 0, h, 1 << 40, None) == sol.SOL_ERR_INVALID_ARG
    assert sol.lib.sol_forward_host(ctypes.byref(p), h, h, h, h, 0, h + 16, 1 << 40, None) == sol.SOL_ERR_INVALID_ARG
    assert sol.lib.sol_forward_host(ctypes.byref(p), h, h, h, h, 2, h, one, None) == sol.SOL_ERR_WORKSPACE
    assert sol.lib.sol_forward_host(ctypes.byref(sol.make_params(0, 1000, 4, 128)), None, None, None, None, 0,
                                    None, 0, None) == sol.SOL_OK


def test_reblock_sizes_and_argument_checks(sol):
    p = sol.make_params(1, 32768, 56, 128)
    ws = sol.sol_reblock_workspace_bytes(p)
    # fp32 whitened keys dominate: B*H*N*D*4, plus the partial moments (reused for the
    # Gram partials of the levels down to 512-row groups: 3,732 slots of 64.5 KB),
    # factor, orders, keys, axes and means
    assert 56 * 32768 * 128 * 4 < ws < 56 * 32768 * 128 * 4 * 1.35
    assert sol.sol_reblock_workspace_bytes(sol.make_params(1, 300, 2, 64, prefix_len=300)) == 0   # all prefix
    assert sol.sol_reblock_workspace_bytes(sol.make_params(1, 0, 2, 64)) == 0
    assert sol.reblock_levels(32768) == 9 and sol.reblock_levels(64) == 0 and sol.reblock_levels(65) == 1
    P = ctypes.byref(p)
    assert sol.lib.sol_reblock(P, None, None, None, 0, None, None) == sol.SOL_ERR_INVALID_ARG
    assert sol.lib.sol_gather_rows(P, None, None, None, None) == sol.SOL_ERR_INVALID_ARG
    assert sol.lib.sol_scatter_rows(P, None, None, None, None) == sol.SOL_ERR_INVALID_ARG
    bad = sol.make_params(1, 100, 2, 96)
    assert sol.lib.sol_reblock(ctypes.byref(bad), None, None, None, 0, None, None) == sol.SOL_ERR_UNSUPPORTED


def test_reblock_buffers_layout(sol):
    p = sol.make_params(2, 300, 3, 64, prefix_len=70)
    rb = sol.alloc_reblock(p, "cpu")   # allocation only: no kernel runs
    assert rb.ws.numel() == sol.sol_reblock_workspace_bytes(p) > 0
    assert rb.perm.numel() == 2 * 3 * 300 and rb.perm.dtype.is_floating_point is False
    for t in (rb.qp, rb.kp, rb.vp, rb.buf.o):
        assert tuple(t.shape) == (2, 3, 300, 64)
    hm = rb.hm
    assert (hm.in_stride_b, hm.in_stride_n, hm.in_stride_h) == (3 * 300 * 64, 64, 300 * 64)
    assert (hm.out_stride_b, hm.out_stride_n, hm.out_stride_h) == (3 * 300 * 64, 64, 300 * 64)
    assert (hm.B, hm.N, hm.H, hm.D, hm.prefix_len, hm.routing) == (2, 300, 3, 64, 70, p.routing)
    assert rb.buf.ws.numel() == sol.sol_workspace_bytes(hm)
