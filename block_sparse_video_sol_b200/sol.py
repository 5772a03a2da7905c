"""Thin ctypes binding of libsol.so (the C ABI declared in include/sol.h).

Argument marshalling only: every step of the forward pass runs in the CUDA
kernels of libsol.so.  Torch tensors supply device memory and the current
stream; nothing here computes.  Importing this module loads the library and
raises if it is missing -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional

import torch

_LIB_PATH = os.environ.get("SOL_LIB_PATH") or os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsol.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libsol.so not built ({_LIB_PATH}); run `python -m block_sparse_video_sol_b200.build`")
lib = ctypes.CDLL(_LIB_PATH)

SOL_OK, SOL_ERR_INVALID_ARG, SOL_ERR_UNSUPPORTED, SOL_ERR_WORKSPACE, SOL_ERR_CUDA, SOL_ERR_TIMEOUT = range(6)

# Every entry point declared in include/sol.h.
EXPORTS = ("sol_workspace_bytes", "sol_workspace_offsets", "sol_workspace_int8_offsets", "sol_col_capacity", "sol_pool", "sol_route", "sol_route_static",
           "sol_attn_fwd", "sol_forward_host", "sol_host_staging_bytes", "sol_last_device_status",
           "sol_status_string", "sol_last_error_text", "sol_debug_drop_arrive",
           "sol_reblock_workspace_bytes", "sol_reblock", "sol_gather_rows", "sol_scatter_rows")


class sol_params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("N", ctypes.c_int32), ("H", ctypes.c_int32), ("D", ctypes.c_int32),
                ("q_block", ctypes.c_int32), ("k_block", ctypes.c_int32),
                ("tau", ctypes.c_float), ("scale", ctypes.c_float),
                ("prefix_len", ctypes.c_int32), ("log_mass_bias", ctypes.c_int32),
                ("in_stride_b", ctypes.c_int64), ("in_stride_n", ctypes.c_int64), ("in_stride_h", ctypes.c_int64),
                ("out_stride_b", ctypes.c_int64), ("out_stride_n", ctypes.c_int64), ("out_stride_h", ctypes.c_int64),
                ("routing", ctypes.c_int32), ("topk_ratio", ctypes.c_float), ("qk_int8", ctypes.c_int32)]


_P = ctypes.POINTER(sol_params)
_vp = ctypes.c_void_p
lib.sol_workspace_bytes.argtypes = [_P]
lib.sol_workspace_bytes.restype = ctypes.c_size_t
lib.sol_workspace_offsets.argtypes = [_P, ctypes.POINTER(ctypes.c_int64)]
lib.sol_workspace_offsets.restype = ctypes.c_int
lib.sol_workspace_int8_offsets.argtypes = [_P, ctypes.POINTER(ctypes.c_int64)]
lib.sol_workspace_int8_offsets.restype = ctypes.c_int
lib.sol_col_capacity.argtypes = [_P]
lib.sol_col_capacity.restype = ctypes.c_int64
lib.sol_pool.argtypes = [_P, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
lib.sol_pool.restype = ctypes.c_int
lib.sol_route.argtypes = [_P, _vp, ctypes.c_size_t, _vp, _vp, _vp]
lib.sol_route.restype = ctypes.c_int
lib.sol_route_static.argtypes = [_P, _vp, ctypes.c_size_t, _vp, _vp, _vp]
lib.sol_route_static.restype = ctypes.c_int
lib.sol_attn_fwd.argtypes = [_P, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp, _vp, _vp, _vp, _vp]
lib.sol_attn_fwd.restype = ctypes.c_int
lib.sol_forward_host.argtypes = [_P, _vp, _vp, _vp, _vp, ctypes.c_int32, _vp, ctypes.c_size_t, _vp]
lib.sol_forward_host.restype = ctypes.c_int
lib.sol_host_staging_bytes.argtypes = [_P, ctypes.c_int32]
lib.sol_host_staging_bytes.restype = ctypes.c_size_t
lib.sol_last_device_status.argtypes = [_vp]
lib.sol_last_device_status.restype = ctypes.c_int
lib.sol_status_string.argtypes = [ctypes.c_int]
lib.sol_status_string.restype = ctypes.c_char_p
lib.sol_last_error_text.argtypes = []
lib.sol_last_error_text.restype = ctypes.c_char_p
lib.sol_debug_drop_arrive.argtypes = [ctypes.c_int32]
lib.sol_debug_drop_arrive.restype = ctypes.c_int
lib.sol_reblock_workspace_bytes.argtypes = [_P]
lib.sol_reblock_workspace_bytes.restype = ctypes.c_size_t
lib.sol_reblock.argtypes = [_P, _vp, _vp, _vp, ctypes.c_size_t, _vp, _vp]
lib.sol_reblock.restype = ctypes.c_int
lib.sol_gather_rows.argtypes = [_P, _vp, _vp, _vp, _vp]
lib.sol_gather_rows.restype = ctypes.c_int
lib.sol_scatter_rows.argtypes = [_P, _vp, _vp, _vp, _vp]
lib.sol_scatter_rows.restype = ctypes.c_int


class SolError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        text = lib.sol_last_error_text().decode()
        super().__init__(f"{where}: {lib.sol_status_string(status).decode()} ({text})")


def _check(status: int, where: str):
    if status != SOL_OK:
        raise SolError(status, where)


def make_params(B: int, N: int, H: int, D: int, tau: float = 1.0, prefix_len: int = 0,
                log_mass_bias: int = 0, scale: float = 0.0, in_strides=None, out_strides=None,
                q_block: Optional[int] = None, k_block: int = 64, topk_ratio: Optional[float] = None,
                compressed: bool = False, qk_int8: bool = False) -> sol_params:
    """Fill a sol_params; strides default to contiguous BTHD [B, N, H, D].

    ``log_mass_bias``: 0 (or False) mean-pooled centroids, 1 (or True) plus the
    log-mass bias, 2 anchor-weighted key/value summaries with the bias.
    ``topk_ratio`` selects Top-K routing: the SLA variant (128-row query
    blocks, unselected blocks dropped), or with ``compressed`` the Spark-H3
    configuration (64-row blocks, sink and centroid terms as under threshold
    routing); otherwise threshold routing with ``tau``.
    """
    routing = 0 if topk_ratio is None else (2 if compressed else 1)
    if q_block is None:
        q_block = 128 if routing == 1 else 64
    in_strides = in_strides or (N * H * D, H * D, D)
    out_strides = out_strides or (N * H * D, H * D, D)
    return sol_params(B, N, H, D, q_block, k_block, float(tau), float(scale), prefix_len, int(log_mass_bias),
                      *[int(s) for s in in_strides], *[int(s) for s in out_strides], routing,
                      float(topk_ratio or 0.0), int(bool(qk_int8)))


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def sol_workspace_bytes(p: sol_params) -> int:
    return lib.sol_workspace_bytes(ctypes.byref(p))


def sol_workspace_offsets(p: sol_params) -> list:
    out = (ctypes.c_int64 * 8)()
    _check(lib.sol_workspace_offsets(ctypes.byref(p), out), "sol_workspace_offsets")
    return list(out)


def workspace_views(p: sol_params, ws: torch.Tensor) -> dict:
    """Typed views of the pooled quantities inside a workspace (see sol_workspace_offsets)."""
    off = sol_workspace_offsets(p)
    nb = -(-p.N // 64)   # the workspace holds 64-row blocks for Q and K whatever the routing
    mw = -(-nb // 32)
    B, H, D = p.B, p.H, p.D

    def view(i, dtype, shape):
        n = math.prod(shape)
        esz = torch.tensor([], dtype=dtype).element_size()
        return ws[off[i]:off[i] + n * esz].view(dtype).view(*shape)

    return dict(qbar=view(0, torch.float32, (B, H, nb, D)), kbar=view(1, torch.float32, (B, H, nb, D)),
                kbar16=view(2, torch.bfloat16, (B, H, nb, D)), vbar16=view(3, torch.bfloat16, (B, H, nb, D)),
                cbias=view(4, torch.float32, (B, H, nb)), anchor=view(5, torch.float32, (B, H, D)),
                mask=view(6, torch.int32, (B * H * nb, mw)), counts=view(7, torch.int32, (B * H * nb,)))


def int8_views(p: sol_params, ws: torch.Tensor) -> dict:
    """Typed views of the INT8 QK quantities sol_pool leaves in a workspace (qk_int8 = 1)."""
    off = (ctypes.c_int64 * 3)()
    _check(lib.sol_workspace_int8_offsets(ctypes.byref(p), off), "sol_workspace_int8_offsets")
    nb = -(-p.N // 64)
    B, H, N, D = p.B, p.H, p.N, p.D
    return dict(kcode=ws[off[0]:off[0] + B * H * N * D].view(torch.int8).view(B, H, N, D),
                ksig=ws[off[1]:off[1] + B * H * nb * 4].view(torch.float32).view(B, H, nb),
                kmean16=ws[off[2]:off[2] + B * H * nb * D * 2].view(torch.bfloat16).view(B, H, nb, D))


def sol_col_capacity(p: sol_params) -> int:
    return lib.sol_col_capacity(ctypes.byref(p))


def sol_pool(p: sol_params, q, k, v, ws: torch.Tensor, stream=None):
    _check(lib.sol_pool(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(ws), ws.numel() * ws.element_size(),
                        _stream(stream)), "sol_pool")


def sol_route(p: sol_params, ws: torch.Tensor, row_ptr: torch.Tensor, col_idx: torch.Tensor, stream=None):
    _check(lib.sol_route(ctypes.byref(p), _ptr(ws), ws.numel() * ws.element_size(), _ptr(row_ptr), _ptr(col_idx),
                         _stream(stream)), "sol_route")


def sol_route_static(p: sol_params, ws: torch.Tensor, row_ptr: torch.Tensor, col_idx: torch.Tensor,
                     stream=None):
    """Routing without caller scratch (see include/sol.h); ws may hold only the pooled part."""
    _check(lib.sol_route_static(ctypes.byref(p), _ptr(ws), ws.numel() * ws.element_size(), _ptr(row_ptr),
                                _ptr(col_idx), _stream(stream)), "sol_route_static")


def sol_host_staging_bytes(p: sol_params, heads_per_chunk: int = 0) -> int:
    return lib.sol_host_staging_bytes(ctypes.byref(p), heads_per_chunk)


def sol_forward_host(p: sol_params, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                     staging: torch.Tensor, heads_per_chunk: int = 0, stream=None):
    """Whole forward pass on host (CPU) tensors, pipelined over head chunks (see include/sol.h).

    q, k, v, o are CPU bf16 tensors (pinned for copy/compute overlap); staging is a
    CUDA uint8 tensor of at least sol_host_staging_bytes(p, heads_per_chunk) bytes.
    Asynchronous: synchronise the stream before reading o."""
    for t in (q, k, v, o):
        if t.is_cuda:
            raise ValueError("sol_forward_host takes host tensors")
    _check(lib.sol_forward_host(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o), heads_per_chunk, _ptr(staging),
                                staging.numel() * staging.element_size(), _stream(stream)), "sol_forward_host")


def sol_attn_fwd(p: sol_params, q, k, v, ws: torch.Tensor, row_ptr: torch.Tensor, col_idx: torch.Tensor,
                 o: torch.Tensor, lse: Optional[torch.Tensor] = None, stream=None):
    _check(lib.sol_attn_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(ws), ws.numel() * ws.element_size(),
                            _ptr(row_ptr), _ptr(col_idx), _ptr(o), _ptr(lse), _stream(stream)), "sol_attn_fwd")


def sol_last_device_status(stream=None):
    _check(lib.sol_last_device_status(_stream(stream)), "device status")


def sol_debug_drop_arrive(step: int):
    """Fault-test library only: withhold the attention's "P ready" arrive of S
    tile `step` in every CTA (-1: none), so that its bounded wait expires."""
    _check(lib.sol_debug_drop_arrive(step), "sol_debug_drop_arrive")


def sol_reblock_workspace_bytes(p: sol_params) -> int:
    return lib.sol_reblock_workspace_bytes(ctypes.byref(p))


def sol_reblock(p: sol_params, q, k, ws: torch.Tensor, perm: torch.Tensor, stream=None):
    _check(lib.sol_reblock(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(ws), ws.numel(), _ptr(perm), _stream(stream)),
           "sol_reblock")


def sol_gather_rows(p: sol_params, perm: torch.Tensor, x, xp: torch.Tensor, stream=None):
    _check(lib.sol_gather_rows(ctypes.byref(p), _ptr(perm), _ptr(x), _ptr(xp), _stream(stream)), "sol_gather_rows")


def sol_scatter_rows(p: sol_params, perm: torch.Tensor, xp: torch.Tensor, x, stream=None):
    _check(lib.sol_scatter_rows(ctypes.byref(p), _ptr(perm), _ptr(xp), _ptr(x), _stream(stream)), "sol_scatter_rows")


def reblock_levels(n_v: int) -> int:
    """Split levels (sol_reblock launches one kernel per level) for n_v partitioned rows."""
    lv, leaves = 0, -(-n_v // 64)
    while leaves > 1:
        leaves, lv = -(-leaves // 2), lv + 1
    return lv


def head_major_params(p: sol_params) -> sol_params:
    """The same problem on head-major [B, H, N, D] copies (inputs and output)."""
    hm = (p.H * p.N * p.D, p.D, p.N * p.D)
    return sol_params(p.B, p.N, p.H, p.D, p.q_block, p.k_block, p.tau, p.scale, p.prefix_len, p.log_mass_bias,
                      *hm, *hm, p.routing, p.topk_ratio, p.qk_int8)


@dataclass
class Buffers:
    """Caller-owned device buffers of one problem shape (allocated by torch)."""
    ws: torch.Tensor
    row_ptr: torch.Tensor
    col_idx: torch.Tensor
    o: torch.Tensor
    lse: Optional[torch.Tensor]


def alloc_buffers(p: sol_params, device, with_lse: bool = False, head_major_out: bool = False) -> Buffers:
    """Workspace, CSR and output of one problem; the output is [B, N, H, D], or
    [B, H, N, D] with ``head_major_out`` (the layout of the reblocked copies)."""
    nqb = -(-p.N // 64)   # CSR rows are 64-row query blocks whatever the routing
    ws = torch.empty(max(1, sol_workspace_bytes(p)), dtype=torch.uint8, device=device)
    row_ptr = torch.empty(p.B * p.H * nqb + 1, dtype=torch.int32, device=device)
    col_idx = torch.empty(max(1, sol_col_capacity(p)), dtype=torch.int32, device=device)
    shape = (p.B, p.H, p.N, p.D) if head_major_out else (p.B, p.N, p.H, p.D)
    o = torch.empty(shape, dtype=torch.bfloat16, device=device)
    lse = torch.empty((p.B, p.H, p.N), dtype=torch.float32, device=device) if with_lse else None
    return Buffers(ws, row_ptr, col_idx, o, lse)


@dataclass
class ReblockBuffers:
    """Caller-owned buffers of a reblocked pass: the partition's workspace and
    order, the head-major row copies and the Sol buffers of the copies (whose
    ``o`` is the head-major output, in the partition's order)."""
    ws: torch.Tensor
    perm: torch.Tensor
    qp: torch.Tensor
    kp: torch.Tensor
    vp: torch.Tensor
    hm: sol_params
    buf: Buffers


def alloc_reblock(p: sol_params, device) -> ReblockBuffers:
    hm = head_major_params(p)
    ws = torch.empty(max(1, sol_reblock_workspace_bytes(p)), dtype=torch.uint8, device=device)
    perm = torch.empty(max(1, p.B * p.H * p.N), dtype=torch.int32, device=device)
    qp, kp, vp = (torch.empty((p.B, p.H, p.N, p.D), dtype=torch.bfloat16, device=device) for _ in range(3))
    return ReblockBuffers(ws, perm, qp, kp, vp, hm, alloc_buffers(hm, device, head_major_out=True))


def forward_reblocked(p: sol_params, q, k, v, o: torch.Tensor, rb: ReblockBuffers, stream=None):
    """Partition, gather q/k/v, pool -> route -> attention on the copies, scatter into ``o``."""
    sol_reblock(p, q, k, rb.ws, rb.perm, stream)
    for x, xp in ((q, rb.qp), (k, rb.kp), (v, rb.vp)):
        sol_gather_rows(p, rb.perm, x, xp, stream)
    forward(rb.hm, rb.qp, rb.kp, rb.vp, rb.buf, stream)
    sol_scatter_rows(p, rb.perm, rb.buf.o, o, stream)
    return o


def forward(p: sol_params, q, k, v, buf: Buffers, stream=None) -> Buffers:
    """Enqueue pool -> route -> attention on one stream; returns ``buf``."""
    sol_pool(p, q, k, v, buf.ws, stream)
    sol_route(p, buf.ws, buf.row_ptr, buf.col_idx, stream)
    sol_attn_fwd(p, q, k, v, buf.ws, buf.row_ptr, buf.col_idx, buf.o, buf.lse, stream)
    return buf


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, tau: float = 1.0, prefix_len: int = 0,
              log_mass_bias: int = 0, scale: float = 0.0, with_lse: bool = False,
              topk_ratio: Optional[float] = None, compressed: bool = False, reblock: bool = False,
              qk_int8: bool = False):
    """Convenience call on BTHD bf16 CUDA tensors (views with unit head-dim stride allowed).

    Returns (o, buffers); the buffers hold row_ptr / col_idx / lse for inspection.  With
    ``reblock`` the rows are first ordered by the adaptive partition (sol_reblock) and the
    buffers are a ReblockBuffers (its ``perm``, and the Sol buffers of the permuted rows;
    ``with_lse`` is not offered there: the LSE would be in the permuted order).
    """
    B, N, H, D = q.shape
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_cuda or t.stride(3) != 1 or t.stride() != q.stride():
            raise ValueError("q, k, v must be bf16 CUDA tensors with identical strides and contiguous head dim")
    p = make_params(B, N, H, D, tau, prefix_len, log_mass_bias, scale,
                    in_strides=(q.stride(0), q.stride(1), q.stride(2)), topk_ratio=topk_ratio,
                    compressed=compressed, qk_int8=qk_int8)
    if reblock:
        if with_lse:
            raise ValueError("with_lse is not offered with reblock")
        rb = alloc_reblock(p, q.device)
        o = torch.empty((B, N, H, D), dtype=torch.bfloat16, device=q.device)
        forward_reblocked(p, q, k, v, o, rb)
        return o, rb
    buf = alloc_buffers(p, q.device, with_lse)
    forward(p, q, k, v, buf)
    return buf.o, buf
