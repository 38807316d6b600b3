"""End-to-end paths on the GPU that the other files cover only in parts.

* Case 1 (S <= L; DAM review page, "Circularity Check" step 1, the patterns cropped to the
  sequence): maps captured at L = 512 on the GPU, their lists extended to S = 300 < L and
  S = 512 = L, attention over them against the oracle's capture, crop and attention.
* Case 2 with grouped-query heads and the per-map scaling (Referee Report major comment
  2; the scaling is the other reading of the unstated normalisation): the GPU capture's
  true masks (per-map scaling, lambda = 1) feed sparse_pattern_extend_case2 for 4 query
  heads over 2 key/value heads at d = 128, with S past L and not a multiple of 128; the
  plan is compared with the oracle's brute-force Case-2 plan and the attention with
  ora_attn_dense_case2.
Lists and plans are compared exactly, attention at the stated tolerances.
"""

import numpy as np
import pytest
import torch

import structured_sparse_attention_b200 as ssa
from structured_sparse_attention_b200 import inputs
from gpu_util import compare_attn, dev, t_bf16

pytestmark = pytest.mark.gpu


def _lists(cap):
    dp, vp = cap["diag_ptr"].cpu().numpy(), cap["vert_ptr"].cpu().numpy()
    return dp, cap["diag_offsets"].cpu().numpy()[:dp[-1]], vp, cap["vert_cols"].cpu().numpy()[:vp[-1]]


@pytest.mark.parametrize("S,d", [(300, 64), (512, 128)])
def test_case1_capture_crop_attention(ora, S, d):
    L, H = 512, 3
    maps = inputs.averaged_maps(inputs.SEED_BASE + 60 + S, H, L=L, n_samples=4)
    cap = ssa.capture(torch.from_numpy(maps).to(dev()))
    want = ora.capture(maps)
    for a, b in zip(_lists(cap), want):
        np.testing.assert_array_equal(a, b)
    plan = ssa.extend(cap["diag_ptr"], cap["diag_offsets"], cap["vert_ptr"], cap["vert_cols"], S)
    ext = ora.extend(*want, S)
    # the crop keeps r < S and c < S only
    edp, edo, evp, evc = ext[:4]
    assert (np.asarray(edo) < S).all() and (np.asarray(evc) < S).all()
    q, k, v = inputs.qkv(inputs.SEED_BASE + 61 + S, H, H, S, d)
    O, LSE = ssa.attn_fwd(t_bf16(q), t_bf16(k), t_bf16(v), plan)
    Oref, Lref = ora.attn_dense(q, k, v, ext, d ** -0.5)
    compare_attn(O, LSE, Oref, Lref)


def test_case2_gqa_per_map_scaling(ora):
    L, S, Hq, Hkv, d, lam = 384, 1500, 4, 2, 128, 1.0
    maps = inputs.averaged_maps(inputs.SEED_BASE + 70, Hq, L=L, n_samples=4)
    tau = 0.05  # per-map scaling keeps few cells at the pages' tau (see the sweep)
    cap = ssa.capture(torch.from_numpy(maps).to(dev()), lam=lam, tau=tau, mu=0.5, scaling="map",
                      true_mask=True)
    want = ora.capture(maps, lam=lam, tau=tau, mu=0.5, scaling="map")
    for a, b in zip(_lists(cap), want):
        np.testing.assert_array_equal(a, b)
    w = cap["true_mask"].cpu().numpy().astype(np.uint32)
    j = np.arange(L)
    tm = ((w[..., j // 32] >> (j % 32).astype(np.uint32)) & 1).astype(np.uint8)
    for m in range(Hq):
        np.testing.assert_array_equal(tm[m], ora.true_mask(maps[m], lam=lam, tau=tau, scaling="map"))
    plan = ssa.extend(cap["diag_ptr"], cap["diag_offsets"], cap["vert_ptr"], cap["vert_cols"], S,
                      true_mask=cap["true_mask"])
    ext = ora.extend(*want, S)
    pg, pref = plan.to_numpy(), ora.plan_case2(ext, S, tm)
    for key in ("tile_ptr", "tile_key0", "tile_dmask", "tile_cmask", "tile_flags", "stripe_cnt", "tile_bits"):
        np.testing.assert_array_equal(pg[key], pref[key], err_msg=key)
    q, k, v = inputs.qkv(inputs.SEED_BASE + 71, Hq, Hkv, S, d)
    O, LSE = ssa.attn_fwd(t_bf16(q), t_bf16(k), t_bf16(v), plan)
    Oref, Lref = ora.attn_dense_case2(q, k, v, ext, d ** -0.5, tm)
    compare_attn(O, LSE, Oref, Lref)
