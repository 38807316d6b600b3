"""Pins for the oracle's stage one (true mask, gamma, selection).

The definitions come from the DAM review page ("What carries the argument"): Box-Cox
with lambda, threshold tau to a binary true mask, gamma_k = sum(M P_k) / sum(P_k),
keep gamma_k >= mu.  These tests check the oracle against hand-derived fixtures,
closed forms and invariants; none of them re-types the oracle's own expression.
"""

import json
import os

import numpy as np
import pytest

from conftest import GOLDEN
from structured_sparse_attention_b200 import inputs


def _mask_from_rows(rows):
    L = len(rows)
    M = np.zeros((L, L), np.uint8)
    for i, s in enumerate(rows):
        for j, ch in enumerate(s):
            if ch == "1":
                assert j <= i, "fixture masks are causal"
                M[i, j] = 1
    return M


def test_hyperparameter_fixture_matches_defaults(ora):
    hp = json.load(open(os.path.join(GOLDEN, "hyperparams.json")))
    import inspect
    sig = inspect.signature(ora.capture)
    assert sig.parameters["lam"].default == hp["lambda"]
    assert sig.parameters["tau"].default == hp["tau"]
    assert sig.parameters["mu"].default == hp["mu"]
    assert sig.parameters["eps"].default == hp["eps"]


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "gamma_cases.json")))["cases"],
                         ids=lambda c: c["name"][:40])
def test_gamma_hand_cases(ora, case):
    M = _mask_from_rows(case["mask"])
    gd, gv = ora.gamma(M)
    exp_d = np.array([n / d for n, d in case["gamma_diag"]])
    exp_v = np.array([n / d for n, d in case["gamma_vert"]])
    np.testing.assert_array_equal(gd, exp_d)
    np.testing.assert_array_equal(gv, exp_v)
    kd, kv = ora.select(gd, gv, mu=0.8)
    assert kd.tolist() == case["kept_diag"]
    assert kv.tolist() == case["kept_vert"]


def test_boxcox_exact_row(ora):
    fx = json.load(open(os.path.join(GOLDEN, "boxcox_row.json")))
    row = np.array(fx["row"], np.float32)
    L = len(row)
    amap = np.zeros((L, L), np.float32)
    amap[L - 1] = row
    for c in fx["cases"]:
        M = ora.true_mask(amap, lam=c["lambda"], eps=0.0, tau=c["tau"])
        assert M[L - 1].tolist() == c["M"], c


def test_true_mask_matches_simplified_closed_form(ora):
    # With a row-wise min-max, ((z^l - 1)/l - ylo)/(yhi - ylo) simplifies to
    # (z^l - zmin^l) / (zmax^l - zmin^l): the -1 and the 1/l cancel.  Compare the
    # decisions wherever the closed form is not within 1e-9 of tau.
    maps = inputs.averaged_maps(5, 2, L=64, n_samples=4)
    for lam in (0.5, 1.0):
        for eps in (1e-8, 1e-10):
            for m in maps:
                M = ora.true_mask(m, lam=lam, eps=eps, tau=0.3)
                x = m.astype(np.float64)
                for i in range(1, 64):
                    z = x[i, :i + 1] + eps
                    zl = np.sqrt(z) if lam == 0.5 else z
                    lo, hi = zl.min(), zl.max()
                    t = (zl - lo) / (hi - lo)
                    ok = np.abs(t - 0.3) > 1e-9
                    np.testing.assert_array_equal(M[i, :i + 1][ok], (t >= 0.3)[ok].astype(np.uint8))
                    assert not M[i, i + 1:].any()


def test_true_mask_constant_row_is_all_set(ora):
    # row 0 has a single entry; a constant row counts as t = 1
    L = 8
    amap = np.zeros((L, L), np.float32)
    for i in range(L):
        amap[i, :i + 1] = 1.0 / (i + 1)
    M = ora.true_mask(amap)
    for i in range(L):
        assert M[i, :i + 1].all() and not M[i, i + 1:].any()


def test_true_mask_constant_map_is_all_set_under_per_map_scaling(ora):
    # per-map scaling (R19): a map whose causal entries are all equal has t = 1 at every
    # causal cell, so every candidate pattern has gamma = 1 and is kept (even at tau = 1)
    L = 8
    amap = np.tril(np.full((L, L), 0.25, np.float32))
    for tau in (0.3, 1.0):
        M = ora.true_mask(amap, tau=tau, scaling="map")
        assert (M == np.tril(np.ones((L, L), np.uint8))).all()
    dp, do, vp, vc = ora.capture(amap[None], tau=1.0, mu=1.0, scaling="map")
    assert do.tolist() == list(range(L)) and vc.tolist() == list(range(L))


def test_invariants_on_synthetic_maps(ora):
    maps = inputs.averaged_maps(11, 3, L=128, n_samples=4)
    L = 128
    # mu = 0 keeps every candidate; mu just above 1 keeps none
    dp, do, vp, vo = ora.capture(maps, mu=0.0)
    assert np.all(np.diff(dp) == L) and np.all(np.diff(vp) == L)
    dp, do, vp, vo = ora.capture(maps, mu=1.0 + 1e-9)
    assert dp[-1] == 0 and vp[-1] == 0
    # tau = 0 makes the true mask all ones, so every gamma is 1 and all are kept
    dp, do, vp, vo = ora.capture(maps, tau=0.0)
    assert np.all(np.diff(dp) == L) and np.all(np.diff(vp) == L)
    # raising tau never adds a pattern; raising mu never adds a pattern
    prev = None
    for tau in (0.1, 0.2, 0.3, 0.5, 0.8):
        cur = ora.capture(maps, tau=tau)
        if prev is not None:
            for a, b in ((0, 1), (2, 3)):
                for m in range(len(maps)):
                    s_new = set(cur[b][cur[a][m]:cur[a][m + 1]].tolist())
                    s_old = set(prev[b][prev[a][m]:prev[a][m + 1]].tolist())
                    assert s_new <= s_old
        prev = cur
    for m in maps:
        gd, gv = ora.gamma(ora.true_mask(m))
        assert ((gd >= 0) & (gd <= 1)).all() and ((gv >= 0) & (gv <= 1)).all()


@pytest.mark.parametrize("scaling,lam,tau", [("row", 0.5, 0.3), ("map", 0.5, 0.05), ("map", 0.25, 0.4)])
def test_capture_equals_stepwise_and_lists_sorted(ora, scaling, lam, tau):
    maps = inputs.averaged_maps(3, 4, L=96, n_samples=4)
    dp, do, vp, vo = ora.capture(maps, lam=lam, tau=tau, scaling=scaling)
    differs = False
    for m in range(len(maps)):
        kd, kv = ora.select(*ora.gamma(ora.true_mask(maps[m], lam=lam, tau=tau, scaling=scaling)), mu=0.8)
        assert do[dp[m]:dp[m + 1]].tolist() == kd.tolist()
        assert vo[vp[m]:vp[m + 1]].tolist() == kv.tolist()
        assert np.all(np.diff(kd) > 0) and np.all(np.diff(kv) > 0)
        other = "map" if scaling == "row" else "row"
        od, ov = ora.select(*ora.gamma(ora.true_mask(maps[m], lam=lam, tau=tau, scaling=other)), mu=0.8)
        differs |= od.tolist() != kd.tolist() or ov.tolist() != kv.tolist()
    assert differs  # the two readings keep different lists on these maps


def test_planted_patterns_are_recovered(ora):
    # Sanity rate (not a parity criterion): with 16 averaged samples the planted
    # diagonals and columns stand out after Box-Cox + row scaling.
    L = 512
    ids = [0, 1, 2, 3]
    maps = inputs.averaged_maps(inputs.SEED_BASE + 2, 8, L=L, n_samples=16, map_ids=ids)
    planted = inputs.planted_map_patterns(inputs.SEED_BASE + 2, 8, L)
    dp, do, vp, vo = ora.capture(maps)
    hit = tot = fp = 0
    for o, m in enumerate(ids):
        pd, pc = planted[m]
        kd = set(do[dp[o]:dp[o + 1]].tolist())
        kc = set(vo[vp[o]:vp[o + 1]].tolist())
        # a planted diagonal with very few cells can be missed or coincide with a column
        big_d = {r for r in pd.tolist() if L - r >= 32}
        big_c = {c for c in pc.tolist() if L - c >= 32}
        hit += len(big_d & kd) + len(big_c & kc)
        tot += len(big_d) + len(big_c)
        fp += len({r for r in kd if L - r >= 32} - set(pd.tolist()))
        fp += len({c for c in kc if L - c >= 32} - set(pc.tolist()))
    assert tot > 0 and hit / tot >= 0.9
    assert fp <= 2


def test_boxcox_eps_row(ora):
    fx = json.load(open(os.path.join(GOLDEN, "boxcox_row.json")))
    row = np.array(fx["eps_row"], np.float32)
    L = len(row)
    amap = np.zeros((L, L), np.float32)
    amap[L - 1] = row
    for c in fx["eps_cases"]:
        M = ora.true_mask(amap, lam=0.5, eps=c["eps"], tau=0.3)
        assert M[L - 1].tolist() == c["M"], c


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "scaling_cases.json")))["cases"],
                         ids=lambda c: f"l{c['lambda']}-t{c['tau']}-{c['scaling']}")
def test_scaling_readings_and_general_lambda_fixture(ora, case):
    # hand-derived masks (exact binary fractions) for the per-row and per-map readings
    # of the scaling before tau, at lambda 1/2, 1 and a general lambda (2, through pow)
    fx = json.load(open(os.path.join(GOLDEN, "scaling_cases.json")))
    amap = np.array(fx["map"], np.float32)
    M = ora.true_mask(amap, lam=case["lambda"], eps=0.0, tau=case["tau"], scaling=case["scaling"])
    assert [M[i, :i + 1].tolist() for i in range(len(amap))] == case["M"]
    assert not np.triu(M, 1).any()


def test_per_map_equals_per_row_when_every_row_spans_the_map(ora):
    # every row holds the map's minimum and maximum, so the two readings coincide
    g = np.random.default_rng(3)
    L = 48
    amap = np.tril(g.uniform(0.1, 0.9, size=(L, L))).astype(np.float32)
    amap[0, 0] = 1.0
    for i in range(1, L):
        amap[i, 0] = 0.0
        amap[i, i] = 1.0
    for lam in (0.5, 1.0, 1.7):
        for tau in (0.2, 0.5):
            np.testing.assert_array_equal(ora.true_mask(amap, lam=lam, tau=tau),
                                          ora.true_mask(amap, lam=lam, tau=tau, scaling="map"))


def test_per_map_scaling_invariants(ora):
    maps = inputs.averaged_maps(12, 3, L=96, n_samples=4)
    L = 96
    # tau = 0 keeps every candidate; raising tau never adds a pattern
    dp, do, vp, vo = ora.capture(maps, tau=0.0, scaling="map")
    assert np.all(np.diff(dp) == L) and np.all(np.diff(vp) == L)
    prev = None
    for tau in (0.001, 0.01, 0.05, 0.2):
        cur = ora.capture(maps, tau=tau, mu=0.5, scaling="map")
        if prev is not None:
            for a, b in ((0, 1), (2, 3)):
                for m in range(len(maps)):
                    assert set(cur[b][cur[a][m]:cur[a][m + 1]].tolist()) <= \
                        set(prev[b][prev[a][m]:prev[a][m + 1]].tolist())
        prev = cur
    # one global threshold per map: a cell is set iff its value's transform clears it,
    # so within a map the set cells are exactly the entries at or above one cut value
    for m in maps:
        M = ora.true_mask(m, tau=0.05, scaling="map")
        cells = np.tril(np.ones((L, L), bool))
        on, off = m[cells & (M == 1)], m[cells & (M == 0)]
        if on.size and off.size:
            assert on.min() > off.max()


@pytest.mark.parametrize("scaling", ["row", "map"])
def test_entries_above_the_diagonal_play_no_part(ora, scaling):
    # The pattern pool and the maps are causal: the true mask, its row (or map) min and
    # max, and so the capture depend on the entries j <= i only.  Values written above
    # the diagonal, larger and smaller than every causal entry, change nothing.
    L = 96
    maps = inputs.averaged_maps(31, 3, L=L, n_samples=3)
    junk = maps.copy()
    iu = np.triu_indices(L, 1)
    junk[:, iu[0], iu[1]] = np.where((iu[0] + iu[1]) % 2 == 0, 7.0, 1e-30).astype(np.float32)
    for m in range(3):
        for lam in (0.5, 1.0):
            a = ora.true_mask(maps[m], lam=lam, scaling=scaling)
            b = ora.true_mask(junk[m], lam=lam, scaling=scaling)
            np.testing.assert_array_equal(a, b)
            assert not a[iu].any()
    for x, y in zip(ora.capture(maps, scaling=scaling), ora.capture(junk, scaling=scaling)):
        np.testing.assert_array_equal(x, y)
