"""Pins for the oracle's attention (list-driven and dense-mask routines).

What the page fixes: the kept patterns are applied to QK^T / sqrt(d_k) before the
softmax, leaving only the retained connections (DAM review page, "What carries the
argument", Referee Report summary, "Circularity Check" step 2).  Reading: masked
logits are removed from the softmax (-inf), empty rows give O = 0, LSE = -inf.

Pins: torch's scaled_dot_product_attention / logsumexp in float64 on a boolean mask
built by enumerating the pattern cells (a library routine), closed forms for r = 0
and c = 0, the normalisation invariant, and agreement of the two oracle routines.
"""

import numpy as np
import pytest
import torch

from structured_sparse_attention_b200 import inputs


def _ext(ora, diags, verts, S):
    dp, do = inputs.to_csr(diags)
    vp, vo = inputs.to_csr(verts)
    return ora.extend(dp, do, vp, vo, S)


def _f64(bits):
    return inputs.f32_from_bf16_bits(bits).astype(np.float64)


def _cell_mask(diags, verts, h, S):
    M = np.zeros((S, S), bool)
    for r in diags[h]:
        for i in range(r, S):
            M[i, i - r] = True
    for c in verts[h]:
        for i in range(c, S):
            M[i, c] = True
    return M


@pytest.mark.parametrize("seed", range(4))
def test_matches_torch_sdpa_on_enumerated_mask(ora, seed):
    g = np.random.default_rng(seed)
    Hq, Hkv, d = 4, 2, 16
    S = int(g.integers(20, 160))
    diags, verts = inputs.random_patterns(77 + seed, Hq, S, max_diag=S // 2, max_vert=8)
    q, k, v = inputs.qkv(500 + seed, Hq, Hkv, S, d)
    scale = 1.0 / np.sqrt(d)
    ext = _ext(ora, diags, verts, S)
    O, LSE = ora.attn_rows(q, k, v, ext, scale, np.arange(S))
    Qt, Kt, Vt = (torch.from_numpy(_f64(a)) for a in (q, k, v))
    for h in range(Hq):
        kvh = h // (Hq // Hkv)
        M = torch.from_numpy(_cell_mask(diags, verts, h, S))
        nonempty = M.any(dim=1)
        ref = torch.nn.functional.scaled_dot_product_attention(
            Qt[h][None, None], Kt[kvh][None, None], Vt[kvh][None, None], attn_mask=M[None, None],
            scale=scale)[0, 0]
        logits = (Qt[h] @ Kt[kvh].T) * scale
        lse = torch.logsumexp(logits.masked_fill(~M, -torch.inf), dim=1)
        ne = nonempty.numpy()
        np.testing.assert_allclose(O[h][ne], ref.numpy()[ne], rtol=0, atol=1e-12)
        np.testing.assert_allclose(LSE[h][ne], lse.numpy()[ne], rtol=0, atol=1e-12)
        assert (O[h][~ne] == 0).all() and np.isneginf(LSE[h][~ne]).all()


def test_full_causal_equals_causal_sdpa(ora):
    Hq, Hkv, S, d = 2, 1, 130, 32
    q, k, v = inputs.qkv(9, Hq, Hkv, S, d)
    ext = _ext(ora, [np.arange(S, dtype=np.int32)] * Hq, [np.zeros(0, np.int32)] * Hq, S)
    O, LSE = ora.attn_dense(q, k, v, ext, 0.125)
    Qt, Kt, Vt = (torch.from_numpy(_f64(a)) for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(Qt, Kt.expand(Hq, -1, -1), Vt.expand(Hq, -1, -1),
                                                           is_causal=True, scale=0.125)
    np.testing.assert_allclose(O, ref.numpy(), rtol=0, atol=1e-12)


def test_diagonal_zero_returns_own_value(ora):
    Hq, S, d = 1, 300, 64
    q, k, v = inputs.qkv(21, Hq, 1, S, d)
    scale = 0.125
    ext = _ext(ora, [np.array([0], np.int32)], [np.zeros(0, np.int32)], S)
    O, LSE = ora.attn_rows(q, k, v, ext, scale, np.arange(S))
    np.testing.assert_array_equal(O[0], _f64(v[0]))
    qk = np.array([scale * np.dot(_f64(q[0, i]), _f64(k[0, i])) for i in range(S)])
    np.testing.assert_allclose(LSE[0], qk, rtol=0, atol=1e-12)


def test_column_zero_returns_first_value(ora):
    S, d = 257, 64
    q, k, v = inputs.qkv(22, 1, 1, S, d)
    ext = _ext(ora, [np.zeros(0, np.int32)], [np.array([0], np.int32)], S)
    O, LSE = ora.attn_rows(q, k, v, ext, 0.125, np.arange(S))
    np.testing.assert_array_equal(O[0], np.broadcast_to(_f64(v[0, 0]), (S, d)))
    qk0 = np.array([0.125 * np.dot(_f64(q[0, i]), _f64(k[0, 0])) for i in range(S)])
    np.testing.assert_allclose(LSE[0], qk0, rtol=0, atol=1e-12)


def test_weights_sum_to_one(ora):
    # with every value row equal to 1, O is the sum of the softmax weights
    Hq, S, d = 2, 200, 16
    q, k, _ = inputs.qkv(23, Hq, 1, S, d)
    v = np.full((1, S, d), 0x3F80, np.uint16)  # bf16 1.0
    diags, verts = inputs.random_patterns(5, Hq, S, 60, 10)
    ext = _ext(ora, diags, verts, S)
    O, LSE = ora.attn_rows(q, k, v, ext, 0.25, np.arange(S))
    nonempty = np.isfinite(LSE)
    assert np.abs(O[nonempty] - 1.0).max() <= 1e-12


@pytest.mark.parametrize("seed", range(3))
def test_list_driven_equals_dense_mask(ora, seed):
    Hq, Hkv, d = 4, 1, 32
    S = 64 + 50 * seed
    diags, verts = inputs.random_patterns(300 + seed, Hq, S, max_diag=S, max_vert=12)
    q, k, v = inputs.qkv(40 + seed, Hq, Hkv, S, d)
    ext = _ext(ora, diags, verts, S)
    Od, Ld = ora.attn_dense(q, k, v, ext, 0.2)
    Or, Lr = ora.attn_rows(q, k, v, ext, 0.2, np.arange(S))
    np.testing.assert_allclose(Or, Od, rtol=0, atol=1e-12)
    fin = np.isfinite(Ld)
    assert (np.isfinite(Lr) == fin).all()
    np.testing.assert_allclose(Lr[fin], Ld[fin], rtol=0, atol=1e-12)


def test_explicit_kv_map_equals_default_grouping(ora):
    Hq, Hkv, S, d = 4, 2, 90, 16
    q, k, v = inputs.qkv(60, Hq, Hkv, S, d)
    diags, verts = inputs.random_patterns(61, Hq, S, 40, 6)
    ext = _ext(ora, diags, verts, S)
    O1, L1 = ora.attn_rows(q, k, v, ext, 0.3, np.arange(S))
    O2, L2 = ora.attn_rows(q, k, v, ext, 0.3, np.arange(S), kv_map=np.array([0, 0, 1, 1], np.int32))
    np.testing.assert_array_equal(O1, O2)
    # a different map changes the answer for heads 1 and 2
    O3, _ = ora.attn_rows(q, k, v, ext, 0.3, np.arange(S), kv_map=np.array([0, 1, 0, 1], np.int32))
    assert not np.array_equal(O1[1], O3[1])


def test_empty_rows_before_band(ora):
    S, d = 200, 16
    q, k, v = inputs.qkv(70, 1, 1, S, d)
    ext = _ext(ora, [np.arange(100, 110, dtype=np.int32)], [np.array([150], np.int32)], S)
    O, LSE = ora.attn_rows(q, k, v, ext, 0.25, np.arange(S))
    assert np.isneginf(LSE[0, :100]).all() and (O[0, :100] == 0).all()
    assert np.isfinite(LSE[0, 100:]).all()
