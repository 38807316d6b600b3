"""Pins of the oracle's Case-2 extended mask (CPU only).

Case 2 reads the extension to S > L (DAM review page, Referee Report major comment 2:
the patterns are pasted beyond the first L tokens) with the captured L x L true mask
kept verbatim in the first block and the union of the kept patterns everywhere else.
The routine is pinned by reductions to the already pinned dense routine and by the
cases whose output is known outright.
"""

import numpy as np
import pytest

from structured_sparse_attention_b200 import inputs


def _ext(ora, diags, verts, S):
    dp, do = inputs.to_csr(diags)
    vp, vo = inputs.to_csr(verts)
    return ora.extend(dp, do, vp, vo, S)


def _pattern_block(diags, verts, L):
    """The patterns' own cells in the first L x L block, as a mask."""
    out = []
    i, j = np.meshgrid(np.arange(L), np.arange(L), indexing="ij")
    for D, C in zip(diags, verts):
        m = np.isin(i - j, D) | np.isin(j, C)
        out.append((m & (j <= i)).astype(np.uint8))
    return np.stack(out)


def test_pattern_block_reduces_to_case_one(ora):
    # a true mask equal to the patterns' cells gives the plain extended mask exactly
    S, L, d, H = 300, 128, 16, 2
    diags = [np.array([0, 3, 40]), np.array([1, 2])]
    verts = [np.array([5, 130]), np.array([0, 200])]
    ext = _ext(ora, diags, verts, S)
    q, k, v = inputs.qkv(5, H, H, S, d)
    o1, l1 = ora.attn_dense(q, k, v, ext, 0.25)
    o2, l2 = ora.attn_dense_case2(q, k, v, ext, 0.25, _pattern_block(diags, verts, L))
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_rows_past_the_block_use_the_patterns_only(ora):
    S, L, d = 260, 128, 8
    diags, verts = [np.array([0, 7])], [np.array([3])]
    ext = _ext(ora, diags, verts, S)
    q, k, v = inputs.qkv(6, 1, 1, S, d)
    rng = np.random.default_rng(1)
    tm = (rng.random((1, L, L)) < 0.3).astype(np.uint8)
    o1, l1 = ora.attn_dense(q, k, v, ext, 0.3)
    o2, l2 = ora.attn_dense_case2(q, k, v, ext, 0.3, tm)
    assert np.array_equal(o1[:, L:], o2[:, L:]) and np.array_equal(l1[:, L:], l2[:, L:])
    assert not np.array_equal(o1[:, :L], o2[:, :L])  # the block itself did change


def test_single_key_rows_copy_that_value(ora):
    # one marked key j0 in row i, no patterns: O[i] = V[j0], LSE[i] = scale * q_i . k_j0
    S, L, d = 128, 128, 8
    ext = _ext(ora, [np.array([], np.int64)], [np.array([], np.int64)], S)
    q, k, v = inputs.qkv(7, 1, 1, S, d)
    tm = np.zeros((1, L, L), np.uint8)
    picks = {10: 3, 50: 50, 127: 0}
    for i, j0 in picks.items():
        tm[0, i, j0] = 1
    O, LSE = ora.attn_dense_case2(q, k, v, ext, 0.5, tm)
    f = lambda a: inputs.f32_from_bf16_bits(a).astype(np.float64)
    for i, j0 in picks.items():
        np.testing.assert_array_equal(O[0, i], f(v[0, j0]))
        assert LSE[0, i] == pytest.approx(0.5 * float(f(q[0, i]) @ f(k[0, j0])), abs=1e-12)
    # rows with no marked key and no pattern: O = 0, LSE = -inf
    assert (O[0, 11] == 0).all() and LSE[0, 11] == -np.inf


def test_full_block_is_causal_attention(ora):
    # every causal cell of the block marked, S = L: the same as the all-diagonals mask
    S = L = 96
    d = 16
    q, k, v = inputs.qkv(8, 1, 1, S, d)
    empty = _ext(ora, [np.array([], np.int64)], [np.array([], np.int64)], S)
    full = _ext(ora, [np.arange(S)], [np.array([], np.int64)], S)
    o1, l1 = ora.attn_dense(q, k, v, full, 0.25)
    o2, l2 = ora.attn_dense_case2(q, k, v, empty, 0.25, np.ones((1, L, L), np.uint8))
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_entries_above_the_diagonal_are_ignored(ora):
    S, L, d = 200, 128, 8
    ext = _ext(ora, [np.array([0, 2])], [np.array([9])], S)
    q, k, v = inputs.qkv(9, 1, 1, S, d)
    rng = np.random.default_rng(2)
    tm = (rng.random((1, L, L)) < 0.2).astype(np.uint8)
    up = tm.copy()
    up[0][np.triu_indices(L, 1)] = 1
    a = ora.attn_dense_case2(q, k, v, ext, 0.2, tm)
    b = ora.attn_dense_case2(q, k, v, ext, 0.2, up)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_captured_true_mask_feeds_the_block(ora):
    # the block comes from stage one: the true mask of an averaged map
    L, S, d = 128, 256, 16
    maps = inputs.averaged_maps(12, 1, L=L, n_samples=3)
    tm = ora.true_mask(maps[0]).astype(np.uint8)[None]
    dp, do, vp, vc = ora.capture(maps)
    ext = ora.extend(dp, do, vp, vc, S)
    q, k, v = inputs.qkv(10, 1, 1, S, d)
    O, LSE = ora.attn_dense_case2(q, k, v, ext, 0.25, tm)
    assert np.isfinite(O).all()
    # row 0 always marks its only key (a constant row counts as t = 1)
    f = lambda a: inputs.f32_from_bf16_bits(a).astype(np.float64)
    np.testing.assert_array_equal(O[0, 0], f(v[0, 0]))


def test_block_replaces_the_patterns_there(ora):
    # inside the block the true mask decides alone: a pattern cell it leaves out is dropped
    S, L, d = 160, 128, 8
    ext = _ext(ora, [np.array([0])], [np.array([], np.int64)], S)
    q, k, v = inputs.qkv(11, 1, 1, S, d)
    O, LSE = ora.attn_dense_case2(q, k, v, ext, 0.3, np.zeros((1, L, L), np.uint8))
    assert (O[0, :L] == 0).all() and (LSE[0, :L] == -np.inf).all()
    f = lambda a: inputs.f32_from_bf16_bits(a).astype(np.float64)
    np.testing.assert_array_equal(O[0, L:], f(v[0, L:]))  # past the block: the diagonal r = 0


# --- the Case-2 tile plan (element-bitmap tiles over the first block) -------------------

def _plan_cells(pl, S, ext, h):
    """The (i, j) cells a plan retains for head h, cell by cell from its tiles: bitmap
    tiles by their bits, band windows by the diagonal and column masks, stripe tiles by
    the stripe counts (columns c <= i among the first stripe_cnt kept columns)."""
    T, nqb = 128, pl["nqb"]
    dp, do, vp, vo = ext
    C = vo[vp[h]:vp[h + 1]]
    cells = set()
    for qb in range(nqb):
        it = h * nqb + qb
        for t in range(pl["tile_ptr"][it], pl["tile_ptr"][it + 1]):
            k0 = int(pl["tile_key0"][t])
            for il in range(T):
                i = T * qb + il
                if i >= S:
                    break
                for jl in range(T):
                    j = k0 + jl
                    if pl["tile_flags"][t] & 2:
                        w = pl["tile_bits"][int(pl["tile_dmask"][t][0]), il, jl // 64]
                        on = (int(w) >> (jl % 64)) & 1
                    else:
                        tt = il - jl + 127
                        dm = int(pl["tile_dmask"][t][tt // 64])
                        cm = int(pl["tile_cmask"][t][jl // 64])
                        on = ((dm >> (tt % 64)) & 1) and not ((cm >> (jl % 64)) & 1)
                    if on:
                        assert j <= i and (i, j) not in cells
                        cells.add((i, j))
        sc = int(pl["stripe_cnt"][it])
        for il in range(T):
            i = T * qb + il
            if i >= S:
                break
            for c in C[:sc]:
                if c <= i:
                    assert (i, int(c)) not in cells
                    cells.add((i, int(c)))
    return cells


def _case2_cells(diags_h, verts_h, tm_h, L, S):
    D, Cs = set(np.asarray(diags_h).tolist()), set(np.asarray(verts_h).tolist())
    out = set()
    for i in range(S):
        for j in range(i + 1):
            if i < L:
                if tm_h[i, j]:
                    out.add((i, j))
            elif (i - j) in D or j in Cs:
                out.add((i, j))
    return out


@pytest.mark.parametrize("L,S", [(128, 300), (200, 300), (256, 256), (100, 90), (300, 700)])
def test_case2_plan_retains_exactly_the_case2_cells(ora, L, S):
    rng = np.random.default_rng(L + S)
    diags = [np.array([0, 3, 40, 129]), np.array([1, 2, 255])]
    verts = [np.array([5, 130, 260]), np.array([0, 200])]
    diags = [d[d < S] for d in diags]
    verts = [c[c < S] for c in verts]
    ext = _ext(ora, diags, verts, S)
    tm = (rng.random((2, L, L)) < 0.25).astype(np.uint8)
    pl = ora.plan_case2(ext, S, tm)
    for h in range(2):
        assert _plan_cells(pl, S, ext, h) == _case2_cells(diags[h], verts[h], tm[h], L, S)


def test_case2_plan_with_pattern_block_matches_case_one(ora):
    # a true mask equal to the patterns' cells: the same cells as the plain plan
    S, L = 400, 256
    diags = [np.array([0, 3, 40, 129])]
    verts = [np.array([5, 130])]
    ext = _ext(ora, diags, verts, S)
    pl2 = ora.plan_case2(ext, S, _pattern_block(diags, verts, L))
    pl1 = ora.plan(ext, S)
    pl1["tile_bits"] = np.zeros((1, 128, 2), np.uint64)
    assert _plan_cells(pl2, S, ext, 0) == _plan_cells(pl1, S, ext, 0)
    # past the first block the plan is the plain one, tile for tile
    nqb, nL = pl1["nqb"], 2
    a1, a2 = pl1["tile_ptr"][nL], pl2["tile_ptr"][nL]
    np.testing.assert_array_equal(pl1["tile_key0"][a1:], pl2["tile_key0"][a2:])
    np.testing.assert_array_equal(pl1["tile_flags"][a1:], pl2["tile_flags"][a2:])
    assert (pl2["tile_flags"][:a2] == 2).all() and (pl2["stripe_cnt"][:nL] == 0).all()


@pytest.mark.parametrize("L,S,nL", [(512, 300, 3), (512, 1000, 4), (384, 1500, 3), (200, 100, 1), (128, 128, 1)])
def test_case2_bitmap_layout(ora, L, S, nL):
    # bitmap blocks are the query blocks holding a row below min(L, S): nL of them, with a
    # slot per (qb, kb <= qb), slot = h * slots + qb (qb + 1) / 2 + kb; listed tiles are
    # those with a set cell, and every slot of a listed tile is its own
    H = 2
    slots = nL * (nL + 1) // 2
    assert ora.case2_bitmap_slots(L, S) == (nL, slots)
    diags = [np.array([0, 3]), np.array([1])]
    verts = [np.array([5]), np.array([0])]
    ext = _ext(ora, [d[d < S] for d in diags], [c[c < S] for c in verts], S)
    tm = (np.random.default_rng(L * S).random((H, L, L)) < 0.3).astype(np.uint8)
    pl = ora.plan_case2(ext, S, tm)
    assert pl["bitmap_slots"] == slots and pl["tile_bits"].shape == (H * slots, 128, 2)
    nqb = pl["nqb"]
    seen = set()
    for h in range(H):
        for qb in range(min(nL, nqb)):
            it = h * nqb + qb
            for t in range(pl["tile_ptr"][it], pl["tile_ptr"][it + 1]):
                kb = int(pl["tile_key0"][t]) // 128
                slot = int(pl["tile_dmask"][t][0])
                assert pl["tile_flags"][t] == 2 and slot == h * slots + qb * (qb + 1) // 2 + kb
                assert pl["tile_bits"][slot].any() and slot not in seen
                seen.add(slot)


def test_case2_empty_bitmap_tile_is_not_listed(ora):
    # L = S = 256 and a true mask of the main diagonal only: block 1's key block 0 (rows
    # 128..255, keys 0..127) holds no cell, so block 1 lists key block 1 alone
    L = S = 256
    ext = _ext(ora, [np.array([], np.int64)], [np.array([], np.int64)], S)
    tm = np.eye(L, dtype=np.uint8)[None]
    pl = ora.plan_case2(ext, S, tm)
    assert pl["tile_key0"][pl["tile_ptr"][0]:pl["tile_ptr"][1]].tolist() == [0]
    assert pl["tile_key0"][pl["tile_ptr"][1]:pl["tile_ptr"][2]].tolist() == [128]
