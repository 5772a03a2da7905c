"""Split-by-split check of an adaptive partition (the oracle's step 9).

The size-balanced rule fixes where every group of the hierarchy sits in the
order: the root holds positions [n_fix, N), and a group of n > 64 rows gives
its first 64 * ceil(ceil(n / 64) / 2) positions to the left part and the rest
to the right.  So any order (the GPU's, or the oracle's own) can be cut back
into its tree level by level, and every split checked on its own members:
the oracle's projections of exactly those members (their mean, the power
steps from the lowest-numbered member, in fp64) must put every left row at or
below every right row, up to a band of ``band`` times the group's projection
range.  A wrong split anywhere in the hierarchy, at any level, fails.

Helper of the tests (no pytest marks here); it calls only the oracle.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from oracle import sol_ref


@dataclasses.dataclass
class SplitReport:
    groups: int = 0              # internal groups checked
    exact: int = 0               # groups whose left part equals the oracle's left part exactly
    worst: float = -np.inf       # max over groups of (max left projection - min right projection) / range
    levels: int = 0              # depth of the deepest internal group + 1


def check_splits(Q: np.ndarray, K: np.ndarray, perm: np.ndarray, prefix: int, band: float = 1e-4,
                 bs: int = 64) -> SplitReport:
    """Assert that ``perm`` [B, H, N] is a valid adaptive partition of (Q, K)
    (fp64 [B, N, H, D]) whose every split agrees with the oracle's projections
    outside the band; returns statistics of the agreement."""
    B, N, H, D = K.shape
    n_fix = min(N, bs * sol_ref.n_blocks(prefix, bs))
    n_v = N - n_fix
    perm = np.asarray(perm, dtype=np.int64).reshape(B, H, N)
    rep = SplitReport()
    for b in range(B):
        for h in range(H):
            row = perm[b, h]
            assert np.array_equal(np.sort(row), np.arange(N)), (b, h, "not a permutation")
            assert np.array_equal(row[:n_fix], np.arange(n_fix)), (b, h, "prefix blocks moved")
    if n_v == 0:
        return rep
    Y = sol_ref.whitened_unit_keys(K, sol_ref.second_moment_whitener(Q, prefix), n_fix)
    for b in range(B):
        for h in range(H):
            order = perm[b, h, n_fix:] - n_fix
            stack = [(0, n_v, 0)]
            while stack:
                start, n, lvl = stack.pop()
                part = order[start:start + n]
                if n <= bs:
                    assert np.all(np.diff(part) > 0), (b, h, start, "leaf rows not ascending")
                    continue
                rep.levels = max(rep.levels, lvl + 1)
                left = sol_ref.split_left_count(n, bs)
                members = np.sort(part)
                p = sol_ref.split_projections(Y[b, h], members)
                pos = np.searchsorted(members, part)          # members[pos] == part
                pl, pr = p[pos[:left]], p[pos[left:]]
                rng = float(p.max() - p.min())
                gap = float(pl.max() - pr.min())
                rep.worst = max(rep.worst, gap / rng if rng > 0 else 0.0)
                assert gap <= band * rng, (b, h, lvl, start, n, gap, rng)
                want = members[np.lexsort((members, p))[:left]]
                rep.exact += int(np.array_equal(np.sort(part[:left]), np.sort(want)))
                rep.groups += 1
                stack.append((start, left, lvl + 1))
                stack.append((start + left, n - left, lvl + 1))
    return rep
