"""The Case-2 extension on the GPU (DAM review page, Referee Report major comment 2;
Appendix A, "Case 2"): the captured L x L true mask verbatim in the first block, the kept
patterns elsewhere.  The capture's true-mask bitmap feeds sparse_pattern_extend_case2;
its plan is compared field by field with the oracle's brute-force Case-2 plan
(plan_case2, element-bitmap tiles included), and the attention over it with the
oracle's dense Case-2 attention (ora_attn_dense_case2) at the stated tolerances.
"""

import numpy as np
import pytest
import torch

import structured_sparse_attention_b200 as ssa
from structured_sparse_attention_b200 import inputs
from gpu_util import compare_attn, dev, lists_to_device, t_bf16

pytestmark = pytest.mark.gpu


def _bits_to_masks(bits, L):
    w = bits.astype(np.uint32)
    j = np.arange(L)
    return ((w[..., j // 32] >> (j % 32).astype(np.uint32)) & 1).astype(np.uint8)


def _capture_case2(maps):
    out = ssa.capture(torch.from_numpy(maps).to(dev()), true_mask=True)
    return out


def _check_plan(pg, pref):
    for k in ("tile_ptr", "tile_key0", "tile_dmask", "tile_cmask", "tile_flags", "stripe_cnt"):
        np.testing.assert_array_equal(pg[k], pref[k], err_msg=k)
    np.testing.assert_array_equal(pg["tile_bits"], pref["tile_bits"], err_msg="tile_bits")


@pytest.mark.parametrize("S,L,d", [(512, 512, 64), (1000, 512, 128), (4096, 512, 64), (700, 300, 128)])
def test_case2_plan_and_attention_match_oracle(ora, S, L, d):
    H = 2
    maps = inputs.averaged_maps(inputs.SEED_BASE + 40 + S, H, L=L, n_samples=4)
    cap = _capture_case2(maps)
    tm = _bits_to_masks(cap["true_mask"].cpu().numpy(), L)
    for m in range(H):  # the bitmap is the oracle's true mask
        np.testing.assert_array_equal(tm[m], ora.true_mask(maps[m]))
    plan = ssa.extend(cap["diag_ptr"], cap["diag_offsets"], cap["vert_ptr"], cap["vert_cols"], S,
                      true_mask=cap["true_mask"])
    dp, do, vp, vc = ora.capture(maps)
    ext = ora.extend(dp, do, vp, vc, S)
    _check_plan(plan.to_numpy(), ora.plan_case2(ext, S, tm))
    q, k, v = inputs.qkv(inputs.SEED_BASE + 41, H, H, S, d)
    O, LSE = ssa.attn_fwd(t_bf16(q), t_bf16(k), t_bf16(v), plan)
    Oref, Lref = ora.attn_dense_case2(q, k, v, ext, d ** -0.5, tm)
    compare_attn(O, LSE, Oref, Lref)


def test_case2_hand_mask_with_patterns_past_the_block(ora):
    # a hand-made true mask (random cells, one empty row, one full row) and lists that
    # reach past L; L not a multiple of 128, so one query block straddles L
    S, L, d, H = 600, 200, 64, 1
    rng = np.random.default_rng(5)
    tm = np.tril(rng.random((H, L, L)) < 0.2).astype(np.uint8)
    tm[0, 77] = 0
    tm[0, 150, :151] = 1
    words = np.zeros((H, L, (L + 31) // 32), np.uint32)
    for j in range(L):
        words[..., j // 32] |= tm[..., j].astype(np.uint32) << np.uint32(j % 32)
    diags = [np.array([0, 5, 130, 400], np.int32)]
    verts = [np.array([3, 250], np.int32)]
    (dpt, dot, vpt, vot), host = lists_to_device(diags, verts)
    plan = ssa.extend(dpt, dot, vpt, vot, S, true_mask=torch.from_numpy(words.view(np.int32)).to(dev()))
    ext = ora.extend(*host, S)
    _check_plan(plan.to_numpy(), ora.plan_case2(ext, S, tm))
    q, k, v = inputs.qkv(42, H, H, S, d)
    O, LSE = ssa.attn_fwd(t_bf16(q), t_bf16(k), t_bf16(v), plan)
    Oref, Lref = ora.attn_dense_case2(q, k, v, ext, d ** -0.5, tm)
    compare_attn(O, LSE, Oref, Lref)
    assert torch.isneginf(LSE[0, 77])  # the empty row
