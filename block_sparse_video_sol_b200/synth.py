"""Seeded synthetic inputs for Sol block-sparse attention.

This module is the only code shared by the CUDA path's callers (tests, bench,
smoke) and by the oracle's tests.  It draws random numbers and rounds them to
bf16; it holds none of the method's arithmetic (no pooling, scoring, routing
or attention).

Inputs stand in for MiniMax-H3 attention activations (the pages measure on
H3 renders; no model, weights or prompts are available here).  They follow
the shapes the pages benchmark -- B=1, H=56, d=128, bf16, BTHD layout ("ComfyUI
Sol-Attn: ускорение MiniMax H3 на RTX 5090 до 9x", table "Производительность
на RTX 5090") -- and the packed joint text/audio/video sequence of 38,247 rows
("SM121-optimized MiniMax-H3 / Sol-Engine port" README, introduction).

Recipe (topic-structured video tokens):
  * video tokens are laid out in raster (t, h, w) order;
  * a 4x4x4 spatio-temporal tile (t//4, h//4, w//4) -- partial tiles allowed --
    is assigned one topic, drawn uniformly from ``n_topics`` per-head unit
    vectors u = normalise(N(0, I_d));
  * q = 2.0*u + N(0,1)^d and k = 2.0*u + N(0,1)^d with independent noise;
    v ~ N(0,1)^d;
  * prefix rows (text/audio conditioning) have i.i.d. N(0,1) q, k, v.
Values are drawn in fp32 and rounded to bf16 with round-to-nearest-even.

Every (batch, head) pair draws from its own PCG64 stream keyed by
(seed, b, h), so heads can be generated in parallel and any subset of heads
can be regenerated alone, bit-identically.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import os
from typing import Optional, Sequence

import numpy as np

TOPIC_GAIN = 2.0
TILE = 4


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic problem: shapes, grid and routing knobs."""

    name: str
    B: int
    H: int
    N: int
    D: int
    grid: tuple            # (T, Hs, Ws) of the video part; T*Hs*Ws == N - prefix
    n_topics: int
    prefix: int = 0
    tau: float = 1.0
    seed: int = 1000
    log_mass_bias: int = 0     # centroid mode: 0 means, 1 + log-mass bias, 2 weighted summaries
    topk_ratio: Optional[float] = None   # Top-K routing instead of tau
    compressed: bool = False             # Top-K keeps the compressed branch (64-row blocks, centroids)
    reblock: bool = False                # rows ordered by the adaptive partition first
    qk_int8: bool = False                # exact logits from INT8 query and residual key codes
    q_block: int = 64
    k_block: int = 64

    def __post_init__(self):
        t, hs, ws = self.grid
        if t * hs * ws != self.N - self.prefix:
            raise ValueError(f"grid {self.grid} does not cover {self.N - self.prefix} video rows")


# The pages' workloads (shapes of the H3 attention call).
def tiny() -> Workload:
    """CPU-seconds case: 8x8x16 grid, 16 topics per head."""
    return Workload("tiny_h2_n1024_d64", B=1, H=2, N=1024, D=64, grid=(8, 8, 16),
                    n_topics=16, seed=1000)


def h56_n4096() -> Workload:
    return Workload("h56_n4096_d128", B=1, H=56, N=4096, D=128, grid=(16, 16, 16),
                    n_topics=64, seed=1001)


def mode_suffix(log_mass_bias: int) -> str:
    """Workload-name suffix of a centroid mode."""
    return ("", "_lmb", "_rw")[int(log_mass_bias)]


def h56_sweep(N: int, tau: float = 1.0, log_mass_bias: int = 0) -> Workload:
    if N % 1024:
        raise ValueError("length sweep uses N = T*1024")
    return Workload(f"h56_n{N}_d128_tau{tau:g}" + mode_suffix(log_mass_bias),
                    B=1, H=56, N=N, D=128, grid=(N // 1024, 32, 32), n_topics=128,
                    tau=tau, log_mass_bias=log_mass_bias, seed=1002)


def h56_joint() -> Workload:
    """Joint text/audio/video sequence: 2,407 prefix rows + 10x56x64 video grid."""
    return Workload("h56_joint_n38247_p2407_d128", B=1, H=56, N=38247, D=128,
                    grid=(10, 56, 64), n_topics=128, prefix=2407, seed=1003)


def _stream(seed: int, b: int, h: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, b, h])))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round-to-nearest-even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _tile_index(w: Workload) -> np.ndarray:
    """Tile id of every video row (raster t, h, w order)."""
    t, hs, ws = w.grid
    tt, hh, ww = np.meshgrid(np.arange(t) // TILE, np.arange(hs) // TILE,
                             np.arange(ws) // TILE, indexing="ij")
    nth, ntw = -(-hs // TILE), -(-ws // TILE)
    return ((tt * nth + hh) * ntw + ww).reshape(-1)


def _n_tiles(w: Workload) -> int:
    t, hs, ws = w.grid
    return (-(-t // TILE)) * (-(-hs // TILE)) * (-(-ws // TILE))


def _one_head(w: Workload, b: int, h: int, tile_idx: np.ndarray):
    """Draw q, k, v (fp32, [N, D]) for one (b, h) in a fixed draw order."""
    rng = _stream(w.seed, b, h)
    d, n_vid = w.D, w.N - w.prefix
    topics = rng.standard_normal((w.n_topics, d), dtype=np.float32)
    topics /= np.linalg.norm(topics, axis=1, keepdims=True)
    tile_topic = rng.integers(0, w.n_topics, size=_n_tiles(w))
    mean = TOPIC_GAIN * topics[tile_topic[tile_idx]]                 # [n_vid, d]
    q = np.empty((w.N, d), np.float32)
    k = np.empty((w.N, d), np.float32)
    q[w.prefix:] = mean + rng.standard_normal((n_vid, d), dtype=np.float32)
    k[w.prefix:] = mean + rng.standard_normal((n_vid, d), dtype=np.float32)
    if w.prefix:
        q[:w.prefix] = rng.standard_normal((w.prefix, d), dtype=np.float32)
        k[:w.prefix] = rng.standard_normal((w.prefix, d), dtype=np.float32)
    v = rng.standard_normal((w.N, d), dtype=np.float32)
    return f32_to_bf16_bits(q), f32_to_bf16_bits(k), f32_to_bf16_bits(v)


def generate(w: Workload, heads: Optional[Sequence[int]] = None, threads: Optional[int] = None,
             out: Optional[tuple] = None, b_offset: int = 0):
    """Return (q, k, v) as uint16 bf16 bit arrays in BTHD layout [B, N, len(heads), D].

    ``heads`` selects a subset of head indices (default: all); the values of a
    head do not depend on which other heads are generated.  ``out`` may hold
    three preallocated uint16 arrays of that shape (e.g. views of pinned host
    memory) to be filled in place.  ``b_offset`` shifts the batch index of the
    random streams, so that shard r of a larger batch draws sequence b_offset + b.
    """
    heads = list(range(w.H)) if heads is None else list(heads)
    shape = (w.B, w.N, len(heads), w.D)
    if out is None:
        out = tuple(np.empty(shape, np.uint16) for _ in range(3))
    tile_idx = _tile_index(w)

    def work(job):
        b, slot = job
        q, k, v = _one_head(w, b_offset + b, heads[slot], tile_idx)
        out[0][b, :, slot, :] = q
        out[1][b, :, slot, :] = k
        out[2][b, :, slot, :] = v

    jobs = [(b, s) for b in range(w.B) for s in range(len(heads))]
    threads = threads or min(len(jobs), os.cpu_count() or 1)
    if threads <= 1:
        for j in jobs:
            work(j)
    else:
        with _cf.ThreadPoolExecutor(threads) as ex:
            list(ex.map(work, jobs))
    return out


def random_bf16(shape, seed: int, scale: float = 1.0) -> np.ndarray:
    """Plain i.i.d. N(0, scale^2) tensor as bf16 bits (for edge-case tests)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return f32_to_bf16_bits(scale * rng.standard_normal(shape, dtype=np.float32))


def planted_clusters(levels: int, D: int, H: int = 1, B: int = 1, prefix: int = 0, seed: int = 0,
                     scale0: float = 16.0, offset: float = 10.0, noise: float = 0.05):
    """Inputs with a planted hierarchy of key clusters (bf16 bit patterns, BTHD).

    The rows past the prefix blocks form 2**levels clusters of 64 rows at random
    positions; cluster c's keys are offset * e_(D-1) + sum_l scale0 / 2**l * s_l(c) e_l
    plus Gaussian noise, s_l(c) = +1 or -1 from bit l of c (most significant
    first).  Queries, values and the prefix rows are standard normal.  Returns
    (q, k, v, cluster id of every partitioned row, number of prefix-block rows).
    """
    assert levels + 1 <= D
    rng = np.random.default_rng(seed)
    n_fix = 64 * (-(-prefix // 64))
    n_v = 64 * 2 ** levels
    N = n_fix + n_v
    q = rng.standard_normal((B, N, H, D)).astype(np.float32)
    k = rng.standard_normal((B, N, H, D)).astype(np.float32)
    v = rng.standard_normal((B, N, H, D)).astype(np.float32)
    cid = np.empty((B, H, n_v), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            c = rng.permutation(np.repeat(np.arange(2 ** levels), 64))
            cid[b, h] = c
            centers = np.zeros((2 ** levels, D), dtype=np.float32)
            centers[:, D - 1] = offset
            for lvl in range(levels):
                sign = np.where((np.arange(2 ** levels) >> (levels - 1 - lvl)) & 1, 1.0, -1.0)
                centers[:, lvl] = scale0 / 2 ** lvl * sign
            k[b, n_fix:, h, :] = centers[c] + noise * rng.standard_normal((n_v, D)).astype(np.float32)
    return f32_to_bf16_bits(q), f32_to_bf16_bits(k), f32_to_bf16_bits(v), cid, n_fix
