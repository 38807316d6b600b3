"""GPU parity of sparse_attn_decode against the fp64 oracle.

The decoding query of sequence b sits at position pos[b] and attends to row pos[b] of
the extended mask over that sequence's cache, so the oracle's row routine (attn_rows,
pinned in test_oracle_attn.py) run on the same cache with the query placed in row
pos[b] gives the expected O and LSE.  Tolerances as for prefill: O max-abs <= 2e-2 and
mean-abs <= 2e-3, LSE max-abs <= 1e-3; an empty key set must give O = 0, LSE = -inf.
"""

import numpy as np
import pytest
import torch

from gpu_util import compare_attn, lists_to_device, t_bf16, t_i32
from structured_sparse_attention_b200 import inputs

pytestmark = pytest.mark.gpu


def _case(ora, diags, verts, S, Hq, Hkv, d, positions, seed, kv_map=None):
    import structured_sparse_attention_b200 as ssa
    dev_lists, host = lists_to_device(diags, verts)
    plan = ssa.extend(*dev_lists, S)
    ext = ora.extend(*host, S)
    scale = d ** -0.5
    B = len(positions)
    qs, ks, vs = [], [], []
    Oref = np.zeros((B, Hq, d))
    Lref = np.zeros((B, Hq))
    for b, pos in enumerate(positions):
        q, k, v = inputs.qkv(seed + b, Hq, Hkv, S, d)
        o, lse = ora.attn_rows(q, k, v, ext, scale, np.array([pos], np.int32), kv_map=kv_map)
        Oref[b], Lref[b] = o[:, 0], lse[:, 0]
        qs.append(q[:, pos])
        ks.append(k)
        vs.append(v)
    km = None if kv_map is None else t_i32(kv_map)
    O, LSE = ssa.attn_decode(t_bf16(np.stack(qs)), t_bf16(np.stack(ks)), t_bf16(np.stack(vs)),
                             t_i32(positions), plan, kv_map=km, scale=scale)
    return compare_attn(O, LSE, Oref, Lref), (O, LSE)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("seed", range(3))
def test_decode_random_patterns(ora, d, seed):
    S = 700
    diags, verts = inputs.random_patterns(500 + seed, 4, S, max_diag=300, max_vert=40)
    _case(ora, diags, verts, S, 4, 2, d, [0, 1, 350, 699], 70 + seed)


def test_decode_band_keys_that_are_columns_count_once(ora):
    # D = {0..127}, pos = 500: the band reaches keys 373..500, and every column lies in it
    S = 512
    diags = [np.arange(128, dtype=np.int32)] * 2
    verts = [np.array([400, 450, 480, 500], np.int32), np.array([0, 373, 374, 501], np.int32)]
    _case(ora, diags, verts, S, 2, 1, 128, [500, 373], 11)


def test_decode_empty_key_set(ora):
    # D = {300}, C = {400}: a query at position 100 has no retained key
    S = 512
    stats, (O, LSE) = _case(ora, [np.array([300], np.int32)], [np.array([400], np.int32)], S, 1, 1, 64,
                            [100, 450], 5)
    assert torch.isneginf(LSE[0, 0]).item() and (O[0].float() == 0).all().item()
    assert torch.isfinite(LSE[1, 0]).item()


def test_decode_explicit_kv_map(ora):
    S = 600
    diags, verts = inputs.random_patterns(77, 4, S, max_diag=200, max_vert=30)
    _case(ora, diags, verts, S, 4, 2, 128, [599, 300], 21, kv_map=np.array([1, 0, 1, 0], np.int32))


def test_decode_long_cache(ora):
    # the 64K layer's pattern rule (1024 contiguous diagonals at a random offset + 128
    # columns), 8 heads, two sequences at different positions
    S = 65536
    diags, verts = inputs.patterns_band_random(inputs.SEED_BASE + 4, n_heads=8, S=S)
    _case(ora, diags, verts, S, 8, 2, 128, [S - 1, 40000], 31)


def test_decode_bad_position_reports_invalid(ora):
    import structured_sparse_attention_b200 as ssa
    S, d = 256, 64
    dev_lists, _ = lists_to_device([np.arange(10, dtype=np.int32)], [np.zeros(0, np.int32)])
    plan = ssa.extend(*dev_lists, S)
    q, k, v = inputs.qkv(3, 1, 1, S, d)
    with pytest.raises(ssa.SSAError) as e:
        ssa.attn_decode(t_bf16(q[None, :, 0]), t_bf16(k[None]), t_bf16(v[None]), t_i32([S]), plan)
    assert e.value.code == -1
    O, LSE = ssa.attn_decode(t_bf16(q[None, :, 5]), t_bf16(k[None]), t_bf16(v[None]), t_i32([5]), plan)
    assert torch.isfinite(LSE).all()
