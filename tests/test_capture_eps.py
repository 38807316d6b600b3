"""The stabiliser eps of the Box-Cox step: 1e-8 in the main text, 1e-10 in the appendix
(DAM review page, Referee Report minor comment 1).  What the choice changes, measured with
the oracle's capture (the library's capture is bit-exact to it at lambda = 1/2 and 1).

At lambda = 1/2 the transformed entry is sqrt(x + eps), and sqrt(x + eps) - sqrt(x) lies
in [0, sqrt(eps)], so eps moves the scaled value t of any entry by at most about
2 sqrt(eps) / (sqrt(max) - sqrt(min)) of its row, ~1e-3 for these maps; a decision flips
only for an entry that close to tau, and a pattern only when enough of its cells flip to
cross mu.  On the capture workload's maps (boost 4) and on sharper ones whose row minima
fall to 1e-15, far below both values, the two values keep the same lists at the pages'
setting and at lambda = 1."""

import numpy as np
import pytest

from structured_sparse_attention_b200 import inputs


@pytest.mark.parametrize("boost", [4.0, 16.0, 32.0])
def test_eps_1e10_keeps_the_patterns_of_eps_1e8(ora, boost):
    n, L = 32, 512
    seed = inputs.SEED_BASE + 2
    maps = inputs.averaged_maps(seed, n, L=L, n_samples=16, boost=boost)
    for lam, tau in ((0.5, 0.3), (0.5, 0.1), (0.5, 0.5), (1.0, 0.3)):
        a = ora.capture(maps, lam=lam, tau=tau, mu=0.8, eps=1e-8)
        b = ora.capture(maps, lam=lam, tau=tau, mu=0.8, eps=1e-10)
        for x, y in zip(a, b):
            np.testing.assert_array_equal(x, y, err_msg=f"boost {boost} lambda {lam} tau {tau}")


def test_row_minima_reach_below_eps_on_the_sharp_maps():
    # the sharpest maps above do test the regime where eps dominates the row minimum
    maps = inputs.averaged_maps(inputs.SEED_BASE + 2, 4, L=512, n_samples=16, boost=32.0)
    mins = [maps[m, i, :i + 1].min() for m in range(4) for i in range(1, 512)]
    assert np.median(mins) < 1e-12


def test_eps_over_the_sweep_grid(ora):
    # the capture workload's maps (128 of them, boost 4) over the whole sensitivity grid:
    # the lists differ only at lambda = 0 (log, where eps sets the bottom of the scale)
    # with tau <= 0.2, where nearly every candidate is kept, and there by a few patterns
    import bench
    n, L = 128, 512
    maps = inputs.averaged_maps(inputs.SEED_BASE + 2, n, L=L, n_samples=16)
    g = bench.SWEEP_GRID
    differs = []
    for scaling in g["scaling"]:
        for lam in g["lam"]:
            for tau in g["tau"]:
                for mu in g["mu"]:
                    a = ora.capture(maps, lam=lam, tau=tau, mu=mu, eps=1e-8, scaling=scaling)
                    b = ora.capture(maps, lam=lam, tau=tau, mu=mu, eps=1e-10, scaling=scaling)
                    if not all(np.array_equal(x, y) for x, y in zip(a, b)):
                        changed = sum(len(_kept(a, m, k) ^ _kept(b, m, k)) for m in range(n) for k in (0, 2))
                        kept = len(a[1]) + len(a[3])
                        differs.append((scaling, lam, tau, mu, changed, kept))
    assert all(lam == 0.0 and tau <= 0.2 for _, lam, tau, *_ in differs), differs
    # a handful of patterns out of the thousands kept at these settings
    assert len(differs) <= 5 and all(c <= 8 and k >= 10000 for *_, c, k in differs), differs


def _kept(lists, m, k):
    ptr, val = lists[k], lists[k + 1]
    return set(val[ptr[m]:ptr[m + 1]].tolist())
