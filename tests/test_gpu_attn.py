"""GPU parity of sparse_attn_fwd against the fp64 oracle.

Tolerances: O max-abs <= 2e-2 and mean-abs <= 2e-3, LSE max-abs <= 1e-3; rows with no
retained key must give O = 0 and LSE = -inf exactly."""

import numpy as np
import pytest
import torch

from gpu_util import compare_attn, lists_to_device, sample_rows, t_bf16, t_i32
from structured_sparse_attention_b200 import inputs

pytestmark = pytest.mark.gpu


def _run(diags, verts, S, Hq, Hkv, d, seed, kv_map=None, scale=None, rows=None, dense=False, ora=None):
    import structured_sparse_attention_b200 as ssa
    dev_lists, host = lists_to_device(diags, verts)
    plan = ssa.extend(*dev_lists, S)
    q, k, v = inputs.qkv(seed, Hq, Hkv, S, d)
    scale = d ** -0.5 if scale is None else scale
    km = None if kv_map is None else t_i32(kv_map)
    O, LSE = ssa.attn_fwd(t_bf16(q), t_bf16(k), t_bf16(v), plan, kv_map=km, scale=scale)
    ext = ora.extend(*host, S)
    if dense:
        Oref, Lref = ora.attn_dense(q, k, v, ext, scale, kv_map=kv_map)
        return compare_attn(O, LSE, Oref, Lref), (O, LSE, q, k, v)
    rows = np.arange(S, dtype=np.int32) if rows is None else rows
    Oref, Lref = ora.attn_rows(q, k, v, ext, scale, rows, kv_map=kv_map)
    return compare_attn(O, LSE, Oref, Lref, rows), (O, LSE, q, k, v)


def test_single_head_512(ora):
    diags, verts = inputs.patterns_small_single_head()
    _run(diags, verts, 512, 1, 1, 64, inputs.SEED_BASE, scale=0.125, dense=True, ora=ora)


@pytest.mark.parametrize("seed", range(10))
def test_fuzz_small(ora, seed):
    g = np.random.default_rng(100 + seed)
    S = int(g.choice([1, 7, 100, 128, 129, 256, 300, 513, 777]))
    d = int(g.choice([64, 128]))
    Hkv = int(g.integers(1, 3))
    Hq = Hkv * int(g.integers(1, 3))
    diags, verts = inputs.random_patterns(300 + seed, Hq, S, max_diag=S, max_vert=min(S, 140))
    _run(diags, verts, S, Hq, Hkv, d, 900 + seed, dense=S <= 1024, ora=ora)


@pytest.mark.parametrize("d", [64, 128])
def test_full_causal_and_ragged(ora, d):
    S = 333
    diags = [np.arange(S, dtype=np.int32)] * 2
    verts = [np.zeros(0, np.int32), np.array([0, 5, 200], np.int32)]
    _run(diags, verts, S, 2, 1, d, 5, dense=True, ora=ora)


def test_main_diagonal_returns_values(ora):
    S, d = 300, 128
    stats, (O, LSE, q, k, v) = _run([np.array([0], np.int32)], [np.zeros(0, np.int32)], S, 1, 1, d, 8,
                                    dense=True, ora=ora)
    # P = 2^(s*scale - m) for the only retained key is 1 up to the rounding residual of
    # the fused s*scale - m, so O = V within one bf16 ulp (the tolerance check above holds)
    got = O[0].float().cpu().numpy()
    want = inputs.f32_from_bf16_bits(v[0])
    assert (np.abs(got - want) <= np.abs(want) * 2.0 ** -7).all()


def test_stripes_only_and_empty_rows(ora):
    S, d = 700, 64
    diags = [np.zeros(0, np.int32), np.arange(400, 420, dtype=np.int32)]
    verts = [np.array([0], np.int32), np.array([650], np.int32)]
    stats, (O, LSE, q, k, v) = _run(diags, verts, S, 2, 2, d, 9, dense=True, ora=ora)
    # c = 0 only: every row returns V[0] (within one bf16 ulp, as above)
    got = O[0].float().cpu().numpy()
    want = np.broadcast_to(inputs.f32_from_bf16_bits(v[0, 0]), got.shape)
    assert (np.abs(got - want) <= np.abs(want) * 2.0 ** -7).all()
    assert np.isneginf(LSE[1, :400].cpu().numpy()).all()


def test_explicit_kv_map(ora):
    S, d = 400, 64
    diags, verts = inputs.random_patterns(77, 4, S, 200, 20)
    _run(diags, verts, S, 4, 2, d, 12, kv_map=np.array([1, 0, 1, 0], np.int32), dense=True, ora=ora)


def test_gqa_16k(ora):
    S = 16384
    diags, verts = inputs.patterns_gqa_16k(inputs.SEED_BASE + 3)
    rows = sample_rows(S, 256, 1)
    _run(diags, verts, S, 32, 8, 64, inputs.SEED_BASE + 3, rows=rows, ora=ora)


def test_band_64k(ora):
    S = 65536
    diags, verts = inputs.patterns_band_random(inputs.SEED_BASE + 4)
    rows = sample_rows(S, 192, 2)
    _run(diags, verts, S, 32, 8, 128, inputs.SEED_BASE + 4, rows=rows, ora=ora)


@pytest.mark.parametrize("density", ["0.5", "2", "10", "100"])
def test_long_context(ora, density):
    S = 104000
    diags, verts = inputs.patterns_density(inputs.SEED_BASE + 5, density)
    n = {"0.5": 128, "2": 128, "10": 32, "100": 8}[density]
    rows = sample_rows(S, n, 3)
    if density == "100":
        rows = np.unique(np.concatenate([rows[::16], rows[-64:]])).astype(np.int32)
    _run(diags, verts, S, 24, 8, 128, inputs.SEED_BASE + 5, rows=rows, ora=ora)


def test_bad_kv_map_reports_invalid(ora):
    import structured_sparse_attention_b200 as ssa
    S, d = 256, 64
    dev_lists, _ = lists_to_device([np.arange(10, dtype=np.int32)] * 2, [np.zeros(0, np.int32)] * 2)
    plan = ssa.extend(*dev_lists, S)
    q, k, v = inputs.qkv(3, 2, 1, S, d)
    with pytest.raises(ssa.SSAError) as e:
        ssa.attn_fwd(t_bf16(q), t_bf16(k), t_bf16(v), plan, kv_map=t_i32([0, 5]))
    assert e.value.code == -1
    # the context stays usable
    O, LSE = ssa.attn_fwd(t_bf16(q), t_bf16(k), t_bf16(v), plan)
    assert torch.isfinite(LSE).all()
