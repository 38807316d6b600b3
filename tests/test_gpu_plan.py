"""GPU parity of sparse_pattern_extend (extended lists and tile plan) against the
oracle: every integer array bit-exact."""

import numpy as np
import pytest

from gpu_util import lists_to_device
from structured_sparse_attention_b200 import inputs

pytestmark = pytest.mark.gpu

FIELDS = ("tile_ptr", "tile_key0", "tile_dmask", "tile_cmask", "tile_flags", "stripe_cnt")


def _gpu_plan(diags, verts, S):
    import structured_sparse_attention_b200 as ssa
    dev_lists, host_lists = lists_to_device(diags, verts)
    return ssa.extend(*dev_lists, S), host_lists


def _check_ext(ora, got, host_lists, S):
    ext = ora.extend(*host_lists, S)
    for a, b in zip(got["ext"], ext):
        np.testing.assert_array_equal(a, b)
    return ext


@pytest.mark.parametrize("seed", range(16))
def test_plan_fuzz_full(ora, seed):
    g = np.random.default_rng(seed)
    S = int(g.choice([1, 2, 127, 128, 129, 255, 256, 300, 640, 1000, 1500, 2047]))
    H = int(g.integers(1, 5))
    diags, verts = inputs.random_patterns(2000 + seed, H, S, max_diag=min(S, 400), max_vert=min(S, 60))
    plan, host = _gpu_plan(diags, verts, S)
    got = plan.to_numpy()
    ext = _check_ext(ora, got, host, S)
    ref = ora.plan(ext, S, "brute" if S <= 700 else "interval")
    assert plan.n_tiles == ref["n_tiles"]
    for k in FIELDS:
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)


def test_plan_lists_beyond_S_are_cut(ora):
    S = 300
    diags = [np.array([0, 5, 299, 300, 1000], np.int32), np.array([], np.int32)]
    verts = [np.array([7, 299, 300], np.int32), np.array([0, 400], np.int32)]
    plan, host = _gpu_plan(diags, verts, S)
    got = plan.to_numpy()
    ext = _check_ext(ora, got, host, S)
    ref = ora.plan(ext, S, "brute")
    for k in FIELDS:
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)


def test_plan_rejects_unsorted_lists():
    import structured_sparse_attention_b200 as ssa
    with pytest.raises(ssa.SSAError) as e:
        _gpu_plan([np.array([4, 2], np.int32)], [np.array([], np.int32)], 64)
    assert e.value.code == -1
    with pytest.raises(ssa.SSAError):
        _gpu_plan([np.array([1], np.int32)], [np.array([3, 3], np.int32)], 64)


def _sampled(ora, plan, ext, S, seed, n=48):
    nqb = (S + 127) // 128
    H = plan.n_heads
    g = np.random.default_rng(seed)
    items = {(h, q) for h in range(H) for q in (0, nqb - 1)}
    items.update((int(g.integers(0, H)), int(g.integers(0, nqb))) for _ in range(n))
    items = np.array(sorted(items), np.int32)
    ref = ora.plan_items(ext, S, items)
    got = plan.to_numpy()
    for a, (h, qb) in enumerate(items):
        g0, g1 = got["tile_ptr"][h * nqb + qb], got["tile_ptr"][h * nqb + qb + 1]
        r0, r1 = ref["item_ptr"][a], ref["item_ptr"][a + 1]
        for k in ("tile_key0", "tile_dmask", "tile_cmask", "tile_flags"):
            np.testing.assert_array_equal(got[k][g0:g1], ref[k][r0:r1], err_msg=f"{k} h={h} qb={qb}")
        assert got["stripe_cnt"][h * nqb + qb] == ref["stripe_cnt"][a]


def test_plan_single_head_512(ora):
    S = 512
    diags, verts = inputs.patterns_small_single_head()
    plan, host = _gpu_plan(diags, verts, S)
    got = plan.to_numpy()
    ext = _check_ext(ora, got, host, S)
    ref = ora.plan(ext, S, "brute")
    for k in FIELDS:
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)


def test_plan_gqa_16k(ora):
    S = 16384
    diags, verts = inputs.patterns_gqa_16k(inputs.SEED_BASE + 3)
    plan, host = _gpu_plan(diags, verts, S)
    got = plan.to_numpy()
    ext = _check_ext(ora, got, host, S)
    ref = ora.plan(ext, S, "interval")
    for k in FIELDS:
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)


def test_plan_band_64k(ora):
    S = 65536
    diags, verts = inputs.patterns_band_random(inputs.SEED_BASE + 4)
    plan, host = _gpu_plan(diags, verts, S)
    got = plan.to_numpy()
    ext = _check_ext(ora, got, host, S)
    ref = ora.plan(ext, S, "interval")
    for k in FIELDS:
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)


@pytest.mark.parametrize("density", ["0.5", "2", "10", "100"])
def test_plan_long_context_sampled(ora, density):
    S = 104000
    diags, verts = inputs.patterns_density(inputs.SEED_BASE + 5, density)
    plan, host = _gpu_plan(diags, verts, S)
    got = plan.to_numpy()
    ext = _check_ext(ora, got, host, S)
    _sampled(ora, plan, ext, S, seed=int(float(density) * 10))
    # total tile count against the closed form for a band of width W (every block
    # touches the tiles its band reaches; columns never empty a tile here)
    assert got["tile_ptr"][-1] == plan.n_tiles
