"""Pins of the oracle's averaged attention maps (CPU only).

The maps are the input of stage one (DAM review page, "What carries the argument":
attention maps averaged over a calibration corpus at capture length L).  Each map is
the mean over samples of the causal row softmax of scale * Q K^T.  These tests pin the
oracle to closed forms and invariants rather than to a second copy of the formula:
uniform rows when every key is zero, the two-token logistic form, the hard-max limit,
invariance under a shift shared by all keys, and linearity in the samples.
"""

import math

import numpy as np
import pytest

from oracle import oracle as O
from structured_sparse_attention_b200 import inputs


def bf16(x):
    return inputs.bf16_bits_from_f32(np.asarray(x, dtype=np.float32))


def test_zero_keys_give_uniform_causal_rows():
    # every logit is 0, so row i spreads 1/(i+1) over keys 0..i
    L, d = 37, 8
    q = bf16(np.random.default_rng(1).standard_normal((2, 3, L, d)))
    k = bf16(np.zeros((2, 3, L, d)))
    maps = O.attn_maps(q, k, 0.3)
    i, j = np.meshgrid(np.arange(L), np.arange(L), indexing="ij")
    want = np.where(j <= i, 1.0 / (i + 1), 0.0)
    np.testing.assert_allclose(maps, np.broadcast_to(want, maps.shape), rtol=0, atol=1e-15)


def test_two_tokens_logistic_form():
    # row 1 holds softmax(scale q1 k0, scale q1 k1): p0 = 1 / (1 + exp(scale q1 (k1 - k0)))
    q = bf16([[[[0.75], [1.5]]]])
    k = bf16([[[[0.5], [-0.25]]]])
    scale = 0.7
    maps = O.attn_maps(q, k, scale)[0]
    p0 = 1.0 / (1.0 + math.exp(scale * 1.5 * (-0.25 - 0.5)))
    assert maps[0, 0] == 1.0 and maps[0, 1] == 0.0
    assert abs(maps[1, 0] - p0) < 1e-15
    assert abs(maps[1, 1] - (1.0 - p0)) < 1e-15


def test_hard_max_limit_picks_the_largest_logit():
    # a large scale turns each row into a one-hot at the argmax of q_i . k_j (j <= i);
    # logits far beyond exp's range also check that the row max is subtracted
    rng = np.random.default_rng(2)
    L, d = 24, 4
    qv = rng.integers(-3, 4, size=(1, 1, L, d)).astype(np.float32)
    kv = rng.integers(-3, 4, size=(1, 1, L, d)).astype(np.float32)
    dots = qv[0, 0] @ kv[0, 0].T
    maps = O.attn_maps(bf16(qv), bf16(kv), 400.0)[0]
    assert np.isfinite(maps).all()
    for i in range(L):
        row = dots[i, : i + 1]
        best = np.flatnonzero(row == row.max())
        if len(best) == 1:  # a unique maximum: one-hot there
            want = np.zeros(L)
            want[best[0]] = 1.0
            np.testing.assert_allclose(maps[i], want, atol=1e-12)
        else:  # ties share the mass equally
            np.testing.assert_allclose(maps[i, best], 1.0 / len(best), atol=1e-12)


def test_rows_are_distributions_and_causal():
    q, k = inputs.qk_samples(11, 2, 3, L=64, d=16)
    maps = O.attn_maps(q, k, 0.25)
    i, j = np.meshgrid(np.arange(64), np.arange(64), indexing="ij")
    assert (maps[:, j > i] == 0).all()
    assert (maps[:, j <= i] > 0).all()
    np.testing.assert_allclose(maps.sum(axis=2), 1.0, atol=1e-13)


def test_shift_shared_by_all_keys_changes_nothing():
    # k_j + delta for every j adds q_i . delta to every logit of row i: same softmax.
    # Values on a 1/4 grid keep q, k and k + delta exact in bf16.
    rng = np.random.default_rng(3)
    L, d = 20, 6
    qv = rng.integers(-6, 7, size=(1, 2, L, d)).astype(np.float32) / 4
    kv = rng.integers(-6, 7, size=(1, 2, L, d)).astype(np.float32) / 4
    delta = rng.integers(-4, 5, size=d).astype(np.float32) / 4
    a = O.attn_maps(bf16(qv), bf16(kv), 0.4)
    b = O.attn_maps(bf16(qv), bf16(kv + delta), 0.4)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)


def test_average_over_samples_is_the_mean_of_single_samples():
    q, k = inputs.qk_samples(12, 1, 3, L=48, d=8)
    whole = O.attn_maps(q, k, 0.35)[0]
    parts = [O.attn_maps(q[:, b:b + 1], k[:, b:b + 1], 0.35)[0] for b in range(3)]
    np.testing.assert_allclose(whole, sum(parts) / 3, rtol=0, atol=1e-15)


def test_query_and_key_roles_are_not_swapped():
    # s_ij uses query row i and key row j: with one non-zero key the column of that key
    # (and only it) stands out in every row that can see it
    L, d = 10, 2
    q = np.ones((1, 1, L, d), np.float32)
    k = np.zeros((1, 1, L, d), np.float32)
    k[0, 0, 3] = [2.0, 2.0]
    maps = O.attn_maps(bf16(q), bf16(k), 1.0)[0]
    for i in range(3, L):
        e = math.exp(4.0)
        np.testing.assert_allclose(maps[i, 3], e / (e + i), atol=1e-14)
        np.testing.assert_allclose(maps[i, 0], 1.0 / (e + i), atol=1e-14)


@pytest.mark.parametrize("bad", [dict(B=0), dict(L=0), dict(d=0)])
def test_rejects_empty_shapes(bad):
    shape = dict(n=1, B=1, L=4, d=2)
    shape.update(bad)
    q = np.zeros((shape["n"], shape["B"], shape["L"], shape["d"]), np.uint16)
    with pytest.raises(RuntimeError):
        O.attn_maps(q, q, 1.0)
