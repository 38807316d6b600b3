"""GPU parity of sparse_attn_maps (averaged causal attention maps) against the fp64 oracle.

The oracle routine attn_maps is pinned in test_oracle_maps.py.  Tolerance, from the
arithmetic: the kernel forms the logits from the same bf16 inputs with fp32
accumulation on the tensor cores (relative error of a logit ~ d * 2^-24 of the sum of
|q_k k_k|), takes 2^x with the hardware approximation (a few ulp of fp32) and sums
and averages in fp32.  A probability p then carries an error of about p * 1e-5 at
most; the bound used is |gpu - oracle| <= 2e-6 + 1e-4 * oracle, elementwise.  Entries
above the diagonal must be exactly 0.
"""

import numpy as np
import pytest
import torch

from gpu_util import t_bf16
from structured_sparse_attention_b200 import inputs

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-6, 1e-4


def _maps(q, k, scale):
    import structured_sparse_attention_b200 as ssa
    out = ssa.attn_maps(t_bf16(q), t_bf16(k), scale)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def _compare(got, want):
    L = got.shape[-1]
    i, j = np.meshgrid(np.arange(L), np.arange(L), indexing="ij")
    assert (got[:, j > i] == 0).all(), "entries above the diagonal must be 0"
    err = np.abs(got - want)
    bound = ATOL + RTOL * np.abs(want)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert (err <= bound).all(), f"max excess at {worst}: got {got[worst]}, want {want[worst]}"


@pytest.mark.parametrize("n, B, L, d, planted", [
    (3, 3, 384, 64, True),     # three row blocks, diagonal chunks masked
    (2, 2, 256, 128, False),   # d = 128 (two 64-column boxes per operand)
    (1, 1, 128, 64, False),    # one block, one sample
    (2, 32, 256, 64, True),    # the largest sample count per call
    (5, 4, 512, 64, True),     # the capture length of the pages, several maps
])
def test_maps_match_oracle(ora, n, B, L, d, planted):
    q, k = inputs.qk_samples(900 + n * 7 + B, n, B, L=L, d=d, planted=planted)
    scale = d ** -0.5
    _compare(_maps(q, k, scale), ora.attn_maps(q, k, scale))


def test_zero_keys_uniform_rows():
    # closed form: every logit 0, row i is 1/(i+1) on keys 0..i
    L = 256
    q = inputs.bf16_bits_from_f32(np.random.default_rng(5).standard_normal((2, 3, L, 64)).astype(np.float32))
    k = np.zeros_like(q)
    got = _maps(q, k, 0.125)
    i, j = np.meshgrid(np.arange(L), np.arange(L), indexing="ij")
    want = np.where(j <= i, 1.0 / (i + 1), 0.0)
    np.testing.assert_allclose(got, np.broadcast_to(want, got.shape), rtol=1e-6, atol=0)


def test_full_size_properties_and_sampled_maps(ora):
    # 512 maps (16 layers x 32 heads) x 16 samples x L = 512, d = 64: every row sums to
    # 1, nothing above the diagonal; four maps compared with the oracle in full
    n, B, L, d = 512, 16, 512, 64
    q, k = inputs.qk_samples(20261202, n, B, L=L, d=d)
    got = _maps(q, k, d ** -0.5)
    i, j = np.meshgrid(np.arange(L), np.arange(L), indexing="ij")
    assert np.isfinite(got).all()
    assert (got[:, j > i] == 0).all()
    assert (got >= 0).all()
    assert np.abs(got.sum(axis=2) - 1.0).max() < 1e-4
    pick = [0, 137, 300, 511]
    _compare(got[pick], ora.attn_maps(q[pick], k[pick], d ** -0.5))


def test_maps_feed_capture(ora):
    # produced maps go straight into capture: the lists equal the oracle's capture of the
    # same maps, and the planted columns and the local diagonal are found
    import structured_sparse_attention_b200 as ssa
    n, B, L = 8, 8, 512
    q, k = inputs.qk_samples(31, n, B, L=L, d=64)
    maps = ssa.attn_maps(t_bf16(q), t_bf16(k))
    lists = ssa.capture(maps)
    got = [t.cpu().numpy() for t in (lists["diag_ptr"], lists["diag_offsets"], lists["vert_ptr"], lists["vert_cols"])]
    want = ora.capture(maps.cpu().numpy())
    for g, w in zip(got, want):
        np.testing.assert_array_equal(g[:len(w)], w)
    dp, do, vp, vc = want
    planted = inputs.planted_map_patterns(31, n, L)
    for m in range(n):
        assert 0 in do[dp[m]:dp[m + 1]]
        assert set(planted[m][1]) <= set(vc[vp[m]:vp[m + 1]].tolist())


@pytest.mark.parametrize("kw, code", [
    (dict(L=200), -1),     # L not a multiple of 128
    (dict(B=33), -1),      # more samples than one call takes
    (dict(d=96), -2),      # unsupported head dimension
])
def test_maps_argument_errors(kw, code):
    import structured_sparse_attention_b200 as ssa
    shape = dict(n=1, B=2, L=128, d=64)
    shape.update(kw)
    q = torch.zeros((shape["n"], shape["B"], shape["L"], shape["d"]), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ssa.SSAError) as e:
        ssa.attn_maps(q, q)
    assert e.value.code == code
