"""Pins for the oracle's extension and canonical tile plan.

Extension: the extended mask is the union of the kept patterns over the S x S causal
square (DAM review page, "What carries the argument" and "Circularity Check" step 1),
i.e. diagonals r < S and columns c < S.  The tile plan is this library's own data
structure; its two oracle routines (brute force and interval arithmetic) must agree,
and the element counts it implies must equal the retained pairs counted by brute
force over the dense mask.
"""

import numpy as np
import pytest

from structured_sparse_attention_b200 import inputs

T = 128


def _ext(ora, diags, verts, S):
    dp, do = inputs.to_csr(diags)
    vp, vo = inputs.to_csr(verts)
    return ora.extend(dp, do, vp, vo, S)


def _dense_mask(diags, verts, h, S):
    M = np.zeros((S, S), bool)
    for r in diags[h]:
        if r < S:
            idx = np.arange(r, S)
            M[idx, idx - r] = True
    for c in verts[h]:
        if c < S:
            M[c:, c] = True
    return M


def _active_count_from_plan(plan, ext, h, S):
    """Count retained pairs implied by the plan: band elements of listed tiles
    (dmask & ~cmask & i < S) plus stripe elements (C_h[k] <= i)."""
    nqb = plan["nqb"]
    C = ext[3][ext[2][h]:ext[2][h + 1]]
    total = 0
    for qb in range(nqb):
        a, b = plan["tile_ptr"][h * nqb + qb], plan["tile_ptr"][h * nqb + qb + 1]
        for t in range(a, b):
            dm = plan["tile_dmask"][t]
            cm = plan["tile_cmask"][t]
            for il in range(T):
                i = T * qb + il
                if i >= S:
                    break
                for jl in range(T):
                    tb = il - jl + T - 1
                    if (int(dm[tb >> 6]) >> (tb & 63)) & 1 and not (int(cm[jl >> 6]) >> (jl & 63)) & 1:
                        total += 1
        for il in range(T):
            i = T * qb + il
            if i >= S:
                break
            total += int(np.sum(C[:plan["stripe_cnt"][h * nqb + qb]] <= i))
    return total


def test_extend_filters_and_validates(ora):
    diags = [np.array([0, 3, 9, 16, 20], np.int32), np.array([], np.int32)]
    verts = [np.array([1, 10, 16], np.int32), np.array([0, 15, 16], np.int32)]
    edp, edo, evp, evo = _ext(ora, diags, verts, 16)
    assert edo[edp[0]:edp[1]].tolist() == [0, 3, 9]
    assert edo[edp[1]:edp[2]].tolist() == []
    assert evo[evp[0]:evp[1]].tolist() == [1, 10]
    assert evo[evp[1]:evp[2]].tolist() == [0, 15]
    with pytest.raises(RuntimeError):
        _ext(ora, [np.array([3, 3], np.int32)], [np.array([], np.int32)], 16)
    with pytest.raises(RuntimeError):
        _ext(ora, [np.array([5, 2], np.int32)], [np.array([], np.int32)], 16)
    with pytest.raises(RuntimeError):
        _ext(ora, [np.array([-1], np.int32)], [np.array([], np.int32)], 16)


def test_plan_main_diagonal_only(ora):
    # D = {0}: each query block has exactly one window, starting at its own first row
    # and holding only the local diagonal t = 127; never FULL; no stripes.
    for S in (256, 300):
        ext = _ext(ora, [np.array([0], np.int32)], [np.array([], np.int32)], S)
        p = ora.plan(ext, S)
        nqb = (S + T - 1) // T
        assert p["n_tiles"] == nqb
        assert p["tile_key0"].tolist() == [T * qb for qb in range(nqb)]
        for t in range(nqb):
            assert p["tile_dmask"][t].tolist() == [0, 1 << 63, 0, 0]
            assert p["tile_cmask"][t].tolist() == [0, 0]
            assert p["tile_flags"][t] == 0
        assert not p["stripe_cnt"].any()


@pytest.mark.parametrize("routine", ["brute", "interval"])
def test_plan_full_causal(ora, routine):
    S = 512
    ext = _ext(ora, [np.arange(S, dtype=np.int32)], [np.array([], np.int32)], S)
    p = ora.plan(ext, S, routine)
    assert p["n_tiles"] == 4 * 5 // 2
    for qb in range(4):
        a, b = p["tile_ptr"][qb], p["tile_ptr"][qb + 1]
        assert p["tile_key0"][a:b].tolist() == [T * kb for kb in range(qb + 1)]
        for t in range(a, b):
            kb = p["tile_key0"][t] // T
            assert p["tile_flags"][t] == (1 if kb < qb else 0)
            if kb == qb:
                # only r >= 0, i.e. t >= 127
                assert p["tile_dmask"][t].tolist() == [0, 0xFFFFFFFFFFFFFFFF << 63 & 0xFFFFFFFFFFFFFFFF,
                                                       0xFFFFFFFFFFFFFFFF, 0x7FFFFFFFFFFFFFFF]


@pytest.mark.parametrize("routine", ["brute", "interval"])
def test_plan_column_owned_by_stripes(ora, routine):
    # D = {128}, C = {0..127}: the only window of block 1 (keys 0..127) holds band
    # elements in columns of C only, so it is not listed; the stripe phase owns them.
    S = 256
    ext = _ext(ora, [np.array([128], np.int32)], [np.arange(128, dtype=np.int32)], S)
    p = ora.plan(ext, S, routine)
    assert p["n_tiles"] == 0
    assert p["stripe_cnt"].tolist() == [128, 128]
    # one excluded column stops a tile from being FULL but keeps it listed: the window
    # of block 1 at keys 0..127 sees every diagonal (r = 1..255), column 5 excludes one
    ext = _ext(ora, [np.arange(S, dtype=np.int32)], [np.array([5], np.int32)], S)
    p = ora.plan(ext, S, routine)
    t = p["tile_ptr"][1]
    assert p["tile_key0"][t] == 0 and p["tile_flags"][t] == 0
    assert p["tile_cmask"][t].tolist() == [1 << 5, 0]
    assert p["tile_dmask"][t].tolist() == [2**64 - 1, 2**64 - 1, 2**64 - 1, 2**63 - 1]


@pytest.mark.parametrize("routine", ["brute", "interval"])
def test_plan_ragged_tail_is_not_full(ora, routine):
    S = 200  # second block has 72 rows
    ext = _ext(ora, [np.arange(S, dtype=np.int32)], [np.array([], np.int32)], S)
    p = ora.plan(ext, S, routine)
    a, b = p["tile_ptr"][1], p["tile_ptr"][2]
    assert p["tile_key0"][a:b].tolist() == [0, T]
    assert p["tile_flags"][a:b].tolist() == [0, 0]
    # S = 400: the ragged block 3 (rows 384..399) has windows that see all 255 diagonals
    # and no column (keys 0..127 and 128..255: r = 257..511 and 129..383, all kept up
    # to S - 1 = 399 for the second); FULL needs the whole block inside S, so none is
    S = 400
    ext = _ext(ora, [np.arange(S, dtype=np.int32)], [np.array([], np.int32)], S)
    p = ora.plan(ext, S, routine)
    a, b = p["tile_ptr"][3], p["tile_ptr"][4]
    assert p["tile_key0"][a:b].tolist() == [0, T, 2 * T, 3 * T]
    assert p["tile_dmask"][a + 1].tolist() == [2**64 - 1, 2**64 - 1, 2**64 - 1, 2**63 - 1]
    assert p["tile_flags"][a:b].tolist() == [0, 0, 0, 0]
    # the same window in the whole block 2 (rows 256..383, keys 0..127: r = 129..383) is FULL
    a2 = p["tile_ptr"][2]
    assert p["tile_key0"][a2] == 0 and p["tile_flags"][a2] == 1


@pytest.mark.parametrize("seed", range(12))
def test_plan_routines_agree_and_count_pairs(ora, seed):
    g = np.random.default_rng(seed)
    S = int(g.integers(1, 700))
    H = 3
    diags, verts = inputs.random_patterns(1000 + seed, H, S, max_diag=min(S, 200), max_vert=min(S, 40))
    ext = _ext(ora, diags, verts, S)
    pb = ora.plan(ext, S, "brute")
    pi = ora.plan(ext, S, "interval")
    for k in ("tile_ptr", "tile_key0", "tile_dmask", "tile_cmask", "tile_flags", "stripe_cnt"):
        np.testing.assert_array_equal(pb[k], pi[k], err_msg=k)
    nnz = ora.nnz(ext, S)
    for h in range(H):
        dense = int(_dense_mask(diags, verts, h, S).sum())
        assert nnz[h] == dense
        if S <= 400:
            assert _active_count_from_plan(pb, ext, h, S) == dense


def test_plan_items_equals_full_plan(ora):
    S = 1000
    diags, verts = inputs.random_patterns(4242, 3, S, max_diag=300, max_vert=30)
    ext = _ext(ora, diags, verts, S)
    full = ora.plan(ext, S, "interval")
    nqb = full["nqb"]
    items = np.array([[h, qb] for h in (2, 0) for qb in (7, 0, 3)], np.int32)
    sel = ora.plan_items(ext, S, items)
    for a, (h, qb) in enumerate(items):
        f0, f1 = full["tile_ptr"][h * nqb + qb], full["tile_ptr"][h * nqb + qb + 1]
        s0, s1 = sel["item_ptr"][a], sel["item_ptr"][a + 1]
        for k in ("tile_key0", "tile_dmask", "tile_cmask", "tile_flags"):
            np.testing.assert_array_equal(full[k][f0:f1], sel[k][s0:s1])
        assert full["stripe_cnt"][h * nqb + qb] == sel["stripe_cnt"][a]


def test_plan_windows_follow_an_unaligned_band(ora):
    # D = {100..399} (300 contiguous offsets).  Block 5 (rows 640..767) reaches keys
    # 640 - 399 = 241 .. 767 - 100 = 667, i.e. 427 keys: four windows starting at 241,
    # 369, 497, 625 (key tiles aligned to multiples of 128 would need five: 1..5).
    S = 1024
    ext = _ext(ora, [np.arange(100, 400, dtype=np.int32)], [np.array([], np.int32)], S)
    for routine in ("brute", "interval"):
        p = ora.plan(ext, S, routine)
        a, b = p["tile_ptr"][5], p["tile_ptr"][6]
        assert p["tile_key0"][a:b].tolist() == [241, 369, 497, 625]
        # window 241: r = 640 - 241 + t - 127 = 272 + t, so bits t = 0..127 (r 272..399)
        assert p["tile_dmask"][a].tolist() == [2**64 - 1, 2**64 - 1, 0, 0]
        # window 625: r = t - 112, so bits t = 212..254 (r 100..142)
        want = 0
        for t in range(212, 255):
            want |= 1 << t
        assert p["tile_dmask"][a + 3].tolist() == [(want >> (64 * w)) & (2**64 - 1) for w in range(4)]
        # window 369 sees r = 144..398, all in D: FULL; windows 241 (r 272..526), 497
        # (r 16..270) and 625 (r -112..142) see D only partly
        assert p["tile_flags"][a:b].tolist() == [0, 1, 0, 0]
        # block 0 (rows 0..127) reaches keys 0..27 only (r = 100 from rows 100..127)
        assert p["tile_key0"][p["tile_ptr"][0]:p["tile_ptr"][1]].tolist() == [0]


def test_plan_windows_skip_gaps_between_diagonal_runs(ora):
    # Two runs far apart, D = {0, 1} and {700}: block 7 (rows 896..1023) reaches keys
    # 196..323 from r = 700 and 895..1023 from the first run; nothing is listed in the
    # gap, and the 129 keys of the first run take two windows (895 and 1023).
    S = 1024
    ext = _ext(ora, [np.array([0, 1, 700], np.int32)], [np.array([], np.int32)], S)
    for routine in ("brute", "interval"):
        p = ora.plan(ext, S, routine)
        a, b = p["tile_ptr"][7], p["tile_ptr"][8]
        assert p["tile_key0"][a:b].tolist() == [196, 895, 1023]


@pytest.mark.parametrize("routine", ["brute", "interval"])
def test_plan_runs_128_and_129_apart(ora, routine):
    # Block 2 (rows 256..383).  D = {0, 128}: the keys reached by r = 128 (128..255) and by
    # r = 0 (256..383) touch, so the windows are 128 and 256.  D = {0, 129}: r = 129
    # reaches 127..254 and r = 0 reaches 256..383; key 255 is needed by no row (it would
    # need r in 1..128), so the second window starts at 256, not at 255: 127 and 256.
    S = 512
    for D, want in (([0, 128], [128, 256]), ([0, 129], [127, 256])):
        ext = _ext(ora, [np.array(D, np.int32)], [np.array([], np.int32)], S)
        p = ora.plan(ext, S, routine)
        a, b = p["tile_ptr"][2], p["tile_ptr"][3]
        assert p["tile_key0"][a:b].tolist() == want, (D, routine)


def test_stripe_counts_at_block_ends(ora):
    # columns exactly at a block's last row (127, 383) and at S - 1 = 999: block qb
    # counts the columns c <= min(S - 1, 128 qb + 127), the same in every routine
    S = 1000
    ext = _ext(ora, [np.array([0], np.int32)], [np.array([127, 383, 999], np.int32)], S)
    want = {0: 1, 1: 1, 2: 2, 3: 2, 6: 2, 7: 3}
    for routine in ("brute", "interval"):
        p = ora.plan(ext, S, routine)
        assert {qb: int(p["stripe_cnt"][qb]) for qb in want} == want
    items = np.array([[0, qb] for qb in want], np.int32)
    sel = ora.plan_items(ext, S, items)
    assert sel["stripe_cnt"].tolist() == list(want.values())
