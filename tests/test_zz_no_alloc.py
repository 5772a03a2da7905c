"""sol_route_static: routing for callers that cannot allocate device memory.

Such callers (a host framework that owns every device allocation through a
fixed-budget pool, or a path that must not allocate) cannot hand the library
routing scratch; sol_route_static keeps that scratch in a fixed array inside
the library.  Its CSR output must equal sol_route's bit for bit -- the same
criterion the routing parity tests use -- on calls in a row: the problem,
then a different problem of the same shape (another tau or Top-K ratio, so
other bitmap words and counts land in the same bytes of the array), then the
first problem again.  The array keeps the previous call's contents; a word
or count the next call failed to write would show there.
This file is collected last so that a run stopping at the first failure has
run every other test first.
"""
import ctypes

import pytest
import torch

from block_sparse_video_sol_b200 import synth
from tests import parity


def _lib():
    from block_sparse_video_sol_b200 import build
    build.build()
    from block_sparse_video_sol_b200 import sol
    return sol


def test_rejects_problems_beyond_the_fixed_array():
    sol = _lib()
    p = sol.make_params(2, 65536, 56, 128)          # ~15 MB of routing scratch > 8 MiB
    st = sol.lib.sol_route_static(ctypes.byref(p), 4096 * 64, 1 << 40, 4096, 4096, None)
    assert st == sol.SOL_ERR_UNSUPPORTED
    assert "8388608" in sol.lib.sol_last_error_text().decode()


@pytest.mark.gpu
@pytest.mark.parametrize("make", [synth.tiny, synth.h56_n4096,
                                  lambda: synth.Workload("ragged", B=2, H=3, N=1000, D=64, grid=(9, 10, 10),
                                                         n_topics=8, prefix=100, tau=0.5, seed=7),
                                  lambda: synth.Workload("ragged_topk", B=2, H=3, N=1000, D=64, grid=(9, 10, 10),
                                                         n_topics=8, prefix=100, seed=7, topk_ratio=0.2),
                                  lambda: synth.Workload("ragged_spark", B=2, H=3, N=1000, D=64, grid=(9, 10, 10),
                                                         n_topics=8, prefix=100, seed=7, log_mass_bias=2,
                                                         topk_ratio=0.2, compressed=True)])
def test_static_route_matches_sol_route_twice(make):
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    sol = _lib()
    w = make()
    q, k, v = synth.generate(w)
    Q, K, V = parity.to_dev(q), parity.to_dev(k), parity.to_dev(v)
    p = sol.make_params(w.B, w.N, w.H, w.D, tau=w.tau, prefix_len=w.prefix, log_mass_bias=w.log_mass_bias,
                        topk_ratio=w.topk_ratio, compressed=w.compressed)
    buf = sol.alloc_buffers(p, Q.device)
    sol.sol_pool(p, Q, K, V, buf.ws)
    sol.sol_route(p, buf.ws, buf.row_ptr, buf.col_idx)
    nnz = int(buf.row_ptr[-1].item())
    off6 = sol.sol_workspace_offsets(p)[6]
    pooled = buf.ws[:off6]                                   # only the pooled part of the workspace
    # the same pooled problem routed differently (same shapes, other mask contents)
    if w.topk_ratio is None:
        p2 = sol.make_params(w.B, w.N, w.H, w.D, tau=w.tau - 0.7, prefix_len=w.prefix, log_mass_bias=w.log_mass_bias)
    else:
        p2 = sol.make_params(w.B, w.N, w.H, w.D, prefix_len=w.prefix, log_mass_bias=w.log_mass_bias,
                             topk_ratio=min(1.0, w.topk_ratio + 0.3), compressed=w.compressed)
    buf2 = sol.alloc_buffers(p2, Q.device)
    buf2.ws[:off6].copy_(pooled)
    sol.sol_route(p2, buf2.ws, buf2.row_ptr, buf2.col_idx)
    nnz2 = int(buf2.row_ptr[-1].item())
    assert nnz2 != nnz
    for prm, ref, n in ((p, buf, nnz), (p2, buf2, nnz2), (p, buf, nnz)):
        rp = torch.full_like(ref.row_ptr, -7)
        ci = torch.full_like(ref.col_idx, -7)
        sol.sol_route_static(prm, pooled, rp, ci)
        sol.sol_last_device_status()
        assert torch.equal(rp, ref.row_ptr)
        assert torch.equal(ci[:n], ref.col_idx[:n])
    # the static CSR drives attention to the same output
    o2 = torch.empty_like(buf.o)
    sol.sol_attn_fwd(p, Q, K, V, buf.ws, rp, ci, o2)
    sol.sol_attn_fwd(p, Q, K, V, buf.ws, buf.row_ptr, buf.col_idx, buf.o)
    torch.cuda.synchronize()
    assert torch.equal(o2, buf.o)
