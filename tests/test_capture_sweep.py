"""Host logic of the stage-one sensitivity sweep (bench.py --workload capture-sweep-*),
run on CPU with the oracle's capture standing in for the library's.

The sweep's rows must follow what the method fixes: a higher mu keeps a subset of the
patterns (gamma >= mu), and so does a higher tau (the true mask t >= tau only loses
entries, so every gamma can only fall) under either scaling of the transformed map; the
extended-mask density is a fraction of the causal pairs and falls with the kept set."""

import numpy as np
import pytest

import bench
from structured_sparse_attention_b200 import inputs

GRID = {"scaling": ("row", "map"), "lam": (0.0, 0.5, 1.0), "tau": (0.1, 0.3, 0.5), "mu": (0.5, 0.8, 0.95)}


def _capture_with(ora, maps):
    return lambda lam, tau, mu, scaling: ora.capture(maps, lam=lam, tau=tau, mu=mu, scaling=scaling)


@pytest.fixture(scope="module")
def rows(ora):
    n, L, S = 6, 128, 4096
    seed = 321
    maps = inputs.averaged_maps(seed, n, L=L, n_samples=4)
    planted = inputs.planted_map_patterns(seed, n, L)
    return bench.capture_sweep(_capture_with(ora, maps), planted, S, GRID)


def _at(rows, scaling, lam, tau, mu):
    return next(r for r in rows if (r["scaling"], r["lam"], r["tau"], r["mu"]) == (scaling, lam, tau, mu))


def test_one_row_per_grid_point(rows):
    assert len(rows) == 2 * 3 * 3 * 3
    assert len({(r["scaling"], r["lam"], r["tau"], r["mu"]) for r in rows}) == len(rows)
    for r in rows:
        assert 0.0 <= r["recall"] <= 1.0 and 0.0 <= r["precision"] <= 1.0
        assert 0.0 <= r["density_at_S"] <= 1.0


@pytest.mark.parametrize("scaling", GRID["scaling"])
@pytest.mark.parametrize("lam", GRID["lam"])
def test_kept_sets_shrink_with_mu_and_tau(rows, scaling, lam):
    for tau in GRID["tau"]:
        seq = [_at(rows, scaling, lam, tau, mu) for mu in GRID["mu"]]
        for a, b in zip(seq, seq[1:]):
            assert b["diags_per_map"] <= a["diags_per_map"] and b["cols_per_map"] <= a["cols_per_map"]
            assert b["density_at_S"] <= a["density_at_S"] + 1e-15
    for mu in GRID["mu"]:
        seq = [_at(rows, scaling, lam, tau, mu) for tau in GRID["tau"]]
        for a, b in zip(seq, seq[1:]):
            assert b["diags_per_map"] <= a["diags_per_map"] and b["cols_per_map"] <= a["cols_per_map"]


def test_grid_without_scaling_means_per_row(ora):
    n, L, S = 3, 64, 500
    maps = inputs.averaged_maps(77, n, L=L, n_samples=3)
    planted = inputs.planted_map_patterns(77, n, L)
    seen = []

    def cap(lam, tau, mu, scaling):
        seen.append(scaling)
        return ora.capture(maps, lam=lam, tau=tau, mu=mu, scaling=scaling)

    (row,) = bench.capture_sweep(cap, planted, S, {"lam": (0.5,), "tau": (0.3,), "mu": (0.8,)})
    assert seen == ["row"] and row["scaling"] == "row"


def test_density_matches_a_direct_count(ora):
    # the density of one setting recomputed cell by cell from the oracle's lists
    n, L, S = 2, 64, 300
    maps = inputs.averaged_maps(55, n, L=L, n_samples=3)
    planted = inputs.planted_map_patterns(55, n, L)
    grid = {"scaling": ("map",), "lam": (0.5,), "tau": (0.3,), "mu": (0.8,)}
    (row,) = bench.capture_sweep(_capture_with(ora, maps), planted, S, grid)
    dp, do, vp, vc = ora.capture(maps, scaling="map")
    total = 0
    for m in range(n):
        D, C = set(do[dp[m]:dp[m + 1]].tolist()), set(vc[vp[m]:vp[m + 1]].tolist())
        i, j = np.tril_indices(S)
        total += int(np.isin(i - j, list(D) or [-1]).__or__(np.isin(j, list(C) or [-1])).sum())
    assert row["density_at_S"] == pytest.approx(total / n / (S * (S + 1) / 2), rel=1e-12)
