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


def test_path_replayed_from_cuda_graph_matches_eager(ora):
    # capture -> extension fill pass -> attention, captured once into a CUDA graph: every
    # call is capture-safe (no host synchronisation), and a replay on new queries gives
    # exactly the eager results, which match the oracle
    L, S, H, d = 256, 2048, 4, 64
    maps_h = inputs.averaged_maps(inputs.SEED_BASE + 80, H, L=L, n_samples=3)
    q_a, k_h, v_h = inputs.qkv(inputs.SEED_BASE + 82, H, H, S, d)
    q_b = inputs.qkv(inputs.SEED_BASE + 83, H, H, S, d)[0]
    maps = torch.from_numpy(maps_h).to(dev())
    q, k, v = t_bf16(q_a), t_bf16(k_h), t_bf16(v_h)
    cap = ssa.capture(maps)
    ws = torch.empty(max(ssa.load().sparse_pattern_capture_ws_bytes(H, L), 16), dtype=torch.uint8, device=dev())
    plan = ssa.extend(cap["diag_ptr"], cap["diag_offsets"], cap["vert_ptr"], cap["vert_cols"], S)
    O = torch.empty_like(q)
    LSE = torch.empty((H, S), dtype=torch.float32, device=dev())
    aws = torch.empty(max(ssa.attn_ws_bytes(plan, d), 16), dtype=torch.uint8, device=dev())
    status = torch.zeros(1, dtype=torch.int32, device=dev())

    def step():
        ssa.capture(maps, out=cap, ws=ws, status=status, check=False)
        ssa.refill(plan, cap["diag_ptr"], cap["diag_offsets"], cap["vert_ptr"], cap["vert_cols"], status=status)
        ssa.attn_fwd(q, k, v, plan, out=O, lse=LSE, ws=aws, status=status, check=False)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    q.copy_(t_bf16(q_b))  # new queries, same maps: the replay recomputes the whole path
    graph.replay()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    O_g, L_g = O.clone(), LSE.clone()
    step()
    torch.cuda.synchronize()
    assert torch.equal(O_g, O) and torch.equal(L_g, LSE)
    ext = ora.extend(*ora.capture(maps_h), S)
    Oref, Lref = ora.attn_dense(q_b, k_h, v_h, ext, d ** -0.5)
    compare_attn(O_g, L_g, Oref, Lref)
    del graph


def test_refill_beyond_the_plan_reports_capacity(ora):
    # a fill pass whose new plan needs more than the plan was sized for changes nothing in
    # the plan and reports SSA_ERR_CAPACITY (-3): more diagonals in total; more columns
    # for one head than the plan's max_vert; lists of the same lengths whose diagonals lie
    # further apart, so that only the tile count grows (30 -> 51 tiles)
    from gpu_util import lists_to_device
    S, d = 1024, 64
    diags = [np.arange(0, 40, dtype=np.int32), np.array([0, 7], np.int32)]
    verts = [np.array([3, 99], np.int32), np.array([5], np.int32)]
    dev_lists, host = lists_to_device(diags, verts)
    plan = ssa.extend(*dev_lists, S)
    before = plan.to_numpy()
    spread = [np.arange(0, 1000, 25, dtype=np.int32), np.array([0, 7], np.int32)]
    n_ref = ora.plan(ora.extend(*host, S), S)["n_tiles"]
    n_spread = ora.plan(ora.extend(*lists_to_device(spread, verts)[1], S), S)["n_tiles"]
    assert len(spread[0]) == len(diags[0]) and n_spread > n_ref == len(before["tile_key0"])
    bigger = [
        ([np.arange(0, 90, dtype=np.int32), np.array([0, 7], np.int32)], verts),
        (diags, [np.array([3, 99], np.int32), np.array([5, 6, 9], np.int32)]),
        (spread, verts),
    ]
    for dg, vt in bigger:
        status = torch.zeros(1, dtype=torch.int32, device=dev())
        lists_b, _ = lists_to_device(dg, vt)
        ssa.refill(plan, *lists_b, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == -3
        after = plan.to_numpy()
        for key in before:
            pairs = zip(before[key], after[key]) if key == "ext" else [(before[key], after[key])]
            for a, b in pairs:
                np.testing.assert_array_equal(a, b, err_msg=key)
    # the plan still serves the lists it was sized for
    q, k, v = inputs.qkv(inputs.SEED_BASE + 90, 2, 2, S, d)
    O, LSE = ssa.attn_fwd(t_bf16(q), t_bf16(k), t_bf16(v), plan)
    Oref, Lref = ora.attn_dense(q, k, v, ora.extend(*host, S), d ** -0.5)
    compare_attn(O, LSE, Oref, Lref)


def test_case2_refill_goes_through_the_bitmap_fill(ora):
    # refilling a Case-2 plan with a true mask that keeps a random half of the captured
    # cells (so the new plan fits) gives the plan a fresh sparse_pattern_extend_case2
    # makes from it, the oracle's Case-2 plan, and attention that matches the oracle;
    # a refill without a mask reuses the one the plan holds
    L, S, H, d = 256, 600, 2, 64
    maps = inputs.averaged_maps(inputs.SEED_BASE + 74, H, L=L, n_samples=3)
    cap = ssa.capture(torch.from_numpy(maps).to(dev()), true_mask=True)
    lists = (cap["diag_ptr"], cap["diag_offsets"], cap["vert_ptr"], cap["vert_cols"])
    plan = ssa.extend(*lists, S, true_mask=cap["true_mask"])
    g = np.random.default_rng(inputs.SEED_BASE + 75)
    keep = g.integers(0, 2 ** 32, size=tuple(cap["true_mask"].shape), dtype=np.uint64).astype(np.uint32)
    tm_sub = cap["true_mask"] & torch.from_numpy(keep.view(np.int32)).to(dev())
    for mask in (tm_sub, None):
        status = torch.zeros(1, dtype=torch.int32, device=dev())
        ssa.refill(plan, *lists, true_mask=mask, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        got, fresh = plan.to_numpy(), ssa.extend(*lists, S, true_mask=tm_sub).to_numpy()
        n = int(fresh["tile_ptr"][-1])
        assert n <= plan.n_tiles
        for key in ("tile_ptr", "stripe_cnt", "tile_bits"):
            np.testing.assert_array_equal(got[key], fresh[key], err_msg=key)
        for key in ("tile_key0", "tile_dmask", "tile_cmask", "tile_flags"):
            np.testing.assert_array_equal(got[key][:n], fresh[key][:n], err_msg=key)
    w = tm_sub.cpu().numpy().astype(np.uint32)
    j = np.arange(L)
    tmb = ((w[..., j // 32] >> (j % 32).astype(np.uint32)) & 1).astype(np.uint8)
    ext = ora.extend(*ora.capture(maps), S)
    pref = ora.plan_case2(ext, S, tmb)
    for key in ("tile_ptr", "stripe_cnt", "tile_bits"):
        np.testing.assert_array_equal(got[key], pref[key], err_msg=key)
    q, k, v = inputs.qkv(inputs.SEED_BASE + 76, H, H, S, d)
    O, LSE = ssa.attn_fwd(t_bf16(q), t_bf16(k), t_bf16(v), plan)
    Oref, Lref = ora.attn_dense_case2(q, k, v, ext, d ** -0.5, tmb)
    compare_attn(O, LSE, Oref, Lref)
