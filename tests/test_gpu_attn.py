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


def _scaled_run(ora, diags, verts, S, d, q32, k32, v, scale):
    """Attention on explicit (float32 -> bf16) Q/K and bf16-bit V against the dense oracle."""
    import structured_sparse_attention_b200 as ssa
    dev_lists, host = lists_to_device(diags, verts)
    plan = ssa.extend(*dev_lists, S)
    q = inputs.bf16_bits_from_f32(q32)
    k = inputs.bf16_bits_from_f32(k32)
    O, LSE = ssa.attn_fwd(t_bf16(q), t_bf16(k), t_bf16(v), plan, scale=scale)
    ext = ora.extend(*host, S)
    Oref, Lref = ora.attn_dense(q, k, v, ext, scale)
    return compare_attn(O, LSE, Oref, Lref), (O, LSE, Oref, Lref)


@pytest.mark.parametrize("d", [64, 128])
def test_large_negative_logits(ora, d):
    """The only retained key of every row (r = 0) scores about -32 sqrt(d), below the natural
    log of 2^-126: its exponential underflows unless the row max is the reference, so a
    wrong reference shows up as an empty row."""
    S = 300
    _, k, v = inputs.qkv(21, 1, 1, S, d)
    k32 = inputs.f32_from_bf16_bits(k)
    stats, (O, LSE, Oref, Lref) = _scaled_run(ora, [np.array([0], np.int32)], [np.zeros(0, np.int32)], S, d,
                                              -32.0 * k32, k32, v, d ** -0.5)
    assert np.isfinite(Lref).all() and (Lref < -126 * np.log(2)).all()
    got = O[0].float().cpu().numpy()
    want = inputs.f32_from_bf16_bits(v[0])
    assert (np.abs(got - want) <= np.abs(want) * 2.0 ** -7).all()


@pytest.mark.parametrize("d", [64, 128])
def test_growing_logits(ora, d):
    """Key norms grow along the sequence, so a row's max rises across its key tiles by far
    more than the lazy-rescale threshold (2^8): exercises the rescale of O and the redo of a
    tile whose stale reference is too small."""
    S = 700
    q, k, v = inputs.qkv(22, 2, 1, S, d)
    q32 = 3.0 * inputs.f32_from_bf16_bits(q)
    k32 = inputs.f32_from_bf16_bits(k) * (0.25 + 6.0 * np.arange(S, dtype=np.float32) / S)[None, :, None]
    diags = [np.arange(0, 400, dtype=np.int32), np.array([0, 3, 130, 131, 260, 500], np.int32)]
    verts = [np.array([5, 300], np.int32), np.array([0, 1, 2, 650], np.int32)]
    _scaled_run(ora, diags, verts, S, d, q32, np.ascontiguousarray(k32), v, d ** -0.5)


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


def test_trailing_empty_items(ora):
    """The first half of the query blocks of every head has no retained key, so the last
    half of the work schedule (which runs from the last query blocks down) is items with
    no tile at all, in long runs after every CTA's last non-empty item.  The step sequence
    must still move past them: the last PVs of the preceding items (which their
    epilogues wait for) may not depend on a later item being scheduled."""
    S, Hq, Hkv, d = 8192, 48, 8, 128
    g = np.random.default_rng(31)
    diags = [np.arange(4096 + int(g.integers(0, 512)), 4096 + 600, dtype=np.int32) for _ in range(Hq)]
    diags = [x[x < S] for x in diags]
    verts = [np.sort(g.choice(np.arange(4096, S), size=3, replace=False)).astype(np.int32) for _ in range(Hq)]
    rows = np.unique(np.concatenate([sample_rows(S, 96, 4), np.arange(4000, 4200)])).astype(np.int32)
    for _ in range(3):  # several launches: the stall depended on timing
        _run(diags, verts, S, Hq, Hkv, d, 41, rows=rows, ora=ora)


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
