"""The seeded input generator (structured_sparse_attention_b200/inputs.py) against the
input recipe it implements: shapes, value ranges, pattern rules and realised densities
of the synthetic workloads, bf16 rounding, and reproducibility.  The generator draws
random numbers and lays them out; it holds none of the method's arithmetic."""

import numpy as np
import pytest
import torch

import bench
from structured_sparse_attention_b200 import inputs


def test_bf16_rounding_is_torchs_round_to_nearest_even():
    g = np.random.default_rng(5)
    x = g.standard_normal(100000).astype(np.float32) * np.float32(3.0)
    # exact ties: the 16 dropped bits are 0x8000, with both parities of the kept bit
    ties = (np.arange(1000, dtype=np.uint32) << np.uint32(16) | np.uint32(0x3F808000)).view(np.float32)
    x = np.concatenate([x, ties, -ties, np.float32([0.0, -0.0, 1.0, 65504.0, 1e-30])])
    got = inputs.bf16_bits_from_f32(x)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, want)
    back = inputs.f32_from_bf16_bits(got)
    np.testing.assert_array_equal(back, torch.from_numpy(got.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_qkv_shapes_distribution_and_reproducibility():
    q, k, v = inputs.qkv(123, 4, 2, 1000, 64)
    assert q.shape == (4, 1000, 64) and k.shape == v.shape == (2, 1000, 64)
    assert q.dtype == k.dtype == np.uint16
    xf = inputs.f32_from_bf16_bits(q).astype(np.float64)
    assert abs(xf.mean()) < 0.01 and abs(xf.std() - 1.0) < 0.01
    q2, k2, v2 = inputs.qkv(123, 4, 2, 1000, 64)
    assert np.array_equal(q, q2) and np.array_equal(k, k2) and np.array_equal(v, v2)
    assert not np.array_equal(q[0], q[1]) and not np.array_equal(k[0], v[0])


def _sorted_distinct(a, lo, hi):
    a = np.asarray(a)
    return a.dtype == np.int32 and (np.diff(a) > 0).all() and (len(a) == 0 or (a[0] >= lo and a[-1] < hi))


def test_layer_patterns_follow_their_rules():
    S = 65536
    diags, verts = inputs.patterns_band_random(7, n_heads=32, S=S)
    for D, C in zip(diags, verts):
        assert len(D) == 1024 and np.array_equal(D, np.arange(D[0], D[0] + 1024)) and 0 <= D[0] <= S - 1024
        assert len(C) == 128 and _sorted_distinct(C, 0, S)
    S = 16384
    diags, verts = inputs.patterns_gqa_16k(8, n_heads=32, S=S)
    for D, C in zip(diags, verts):
        assert np.array_equal(D, np.arange(512))
        assert 32 <= len(C) <= 64 and np.array_equal(C[:4], np.arange(4))
        assert _sorted_distinct(C, 0, S) and (C[4:] >= 512).all()


@pytest.mark.parametrize("density,target", [("0.5", 0.005), ("2", 0.02), ("10", 0.10)])
def test_long_context_densities(density, target):
    S = 104000
    diags, verts = inputs.patterns_density(9, density, n_heads=24, S=S)
    W, V = inputs.DENSITY_POINTS[density]
    assert all(np.array_equal(D, np.arange(W)) for D in diags)
    assert all(len(C) == V and _sorted_distinct(C, 0, S) for C in verts)
    dens = bench.nnz_per_head(diags, verts, S) / (S * (S + 1) / 2)
    assert np.all(np.abs(dens / target - 1.0) < 0.03), dens


def test_full_density_is_plain_causal():
    S = 1000
    diags, verts = inputs.patterns_density(9, "100", n_heads=2, S=S)
    assert all(np.array_equal(D, np.arange(S)) for D in diags) and all(len(C) == 0 for C in verts)
    assert (bench.nnz_per_head(diags, verts, S) == S * (S + 1) // 2).all()


def test_planted_patterns_and_averaged_maps():
    n, L = 6, 64
    planted = inputs.planted_map_patterns(11, n, L)
    for dg, cl in planted:
        assert 1 <= len(dg) <= 8 and 1 <= len(cl) <= 16
        assert _sorted_distinct(dg, 0, L) and _sorted_distinct(cl, 0, L)
    maps = inputs.averaged_maps(11, n, L=L, n_samples=3)
    assert maps.shape == (n, L, L) and maps.dtype == np.float32
    iu = np.triu_indices(L, 1)
    assert (maps[:, iu[0], iu[1]] == 0).all()
    # each row is a mean of probability rows over the causal keys
    np.testing.assert_allclose(maps.astype(np.float64).sum(axis=2), 1.0, atol=1e-5)
    assert (maps[:, np.tril_indices(L)[0], np.tril_indices(L)[1]] > 0).all()
    # any subset of maps reproduces the same maps as the full set
    sub = inputs.averaged_maps(11, n, L=L, n_samples=3, map_ids=[4, 1])
    np.testing.assert_array_equal(sub, maps[[4, 1]])


def test_csr_round_trip():
    lists = [np.array([0, 3, 9], np.int32), np.zeros(0, np.int32), np.array([5], np.int32)]
    ptr, vals = inputs.to_csr(lists)
    assert ptr.tolist() == [0, 3, 3, 4] and vals.tolist() == [0, 3, 9, 5]
    back = inputs.from_csr(ptr, vals)
    assert all(np.array_equal(a, b) for a, b in zip(lists, back))


def test_qk_samples_plant_what_capture_recovers(ora):
    # the maps workload's rows (L = 512, 16 samples, d = 64): the oracle's averaged maps,
    # captured at the pages' setting, keep every planted column and the main diagonal
    n, B, L, d = 4, 16, 512, 64
    q, k = inputs.qk_samples(inputs.SEED_BASE + 1, n, B, L=L, d=d)
    assert q.shape == k.shape == (n, B, L, d)
    maps = ora.attn_maps(q, k, d ** -0.5).astype(np.float32)
    dp, do, vp, vc = ora.capture(maps)
    planted = inputs.planted_map_patterns(inputs.SEED_BASE + 1, n, L)
    for m in range(n):
        assert 0 in do[dp[m]:dp[m + 1]].tolist()
        assert set(planted[m][1].tolist()) <= set(vc[vp[m]:vp[m + 1]].tolist())
