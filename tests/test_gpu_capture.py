"""GPU parity of sparse_pattern_capture against the oracle: kept lists bit-exact."""

import numpy as np
import pytest
import torch

from structured_sparse_attention_b200 import inputs

pytestmark = pytest.mark.gpu


def _run(maps, **kw):
    import structured_sparse_attention_b200 as ssa
    out = ssa.capture(torch.from_numpy(np.ascontiguousarray(maps, np.float32)).to("cuda:0"), **kw)
    dp = out["diag_ptr"].cpu().numpy()
    vp = out["vert_ptr"].cpu().numpy()
    return dp, out["diag_offsets"].cpu().numpy()[:dp[-1]], vp, out["vert_cols"].cpu().numpy()[:vp[-1]]


def _same(a, b):
    for x, y, name in zip(a, b, ("diag_ptr", "diag_offsets", "vert_ptr", "vert_cols")):
        np.testing.assert_array_equal(x, y, err_msg=name)


@pytest.mark.parametrize("L", [1, 5, 37, 128, 300, 512, 700, 1024])
def test_capture_matches_oracle_sizes(ora, L):
    maps = inputs.averaged_maps(100 + L, 3, L=L, n_samples=2)
    _same(_run(maps), ora.capture(maps))


@pytest.mark.parametrize("lam,eps,tau,mu", [(0.5, 1e-8, 0.3, 0.8), (0.5, 1e-10, 0.3, 0.8), (1.0, 1e-8, 0.3, 0.8),
                                            (0.5, 0.0, 0.05, 0.5), (0.5, 1e-8, 0.6, 0.2), (1.0, 0.0, 0.01, 0.9),
                                            (0.5, 1e-8, 0.0, 0.8), (0.5, 1e-8, 1.0, 0.0), (0.5, 1e-8, 1.5, 0.0)])
def test_capture_matches_oracle_parameters(ora, lam, eps, tau, mu):
    maps = inputs.averaged_maps(7, 4, L=256, n_samples=3)
    _same(_run(maps, lam=lam, eps=eps, tau=tau, mu=mu), ora.capture(maps, lam=lam, eps=eps, tau=tau, mu=mu))


def test_capture_exact_ties_and_degenerate_rows(ora):
    # binary fractions put many entries exactly on the tau boundary; constant rows,
    # zeros, repeated values and tiny values near eps exercise the cut search
    L = 64
    g = np.random.default_rng(5)
    maps = np.zeros((6, L, L), np.float32)
    for m in range(6):
        for i in range(L):
            n = i + 1
            if m == 0:
                maps[m, i, :n] = g.choice([0.0, 0.0625, 0.140625, 0.25, 1.0], size=n)
            elif m == 1:
                maps[m, i, :n] = 1.0 / n
            elif m == 2:
                maps[m, i, :n] = g.choice([0.0, 5e-9, 3e-8, 1e-8], size=n)
            elif m == 3:
                maps[m, i, :n] = g.integers(0, 3, size=n) * 0.5
            elif m == 4:
                maps[m, i, :n] = np.float32(0.3) + g.integers(0, 2, size=n) * np.float32(1e-7)
            else:
                maps[m, i, :n] = g.random(n, dtype=np.float32) ** 8
    for tau in (0.3, 0.375, 0.5):
        for lam in (0.5, 1.0):
            for eps in (0.0, 1e-8):
                _same(_run(maps, lam=lam, tau=tau, eps=eps), ora.capture(maps, lam=lam, tau=tau, eps=eps))


def test_capture_full_model_maps(ora):
    # 16 layers x 32 heads at L = 512, averaged over 16 samples
    maps = inputs.averaged_maps(inputs.SEED_BASE + 2, 512, L=512, n_samples=16)
    _same(_run(maps), ora.capture(maps))


def test_capture_rejects_negative_entries():
    import structured_sparse_attention_b200 as ssa
    maps = inputs.averaged_maps(1, 2, L=32, n_samples=1)
    maps[1, 20, 3] = -1e-3
    with pytest.raises(ssa.SSAError) as e:
        _run(maps)
    assert e.value.code == -1


# --- the optional readings and outputs of sparse_pattern_capture_ex ---------------------

def _bits_to_mask(bits, L):
    """uint32 words [L][ceil(L/32)] (as int32) -> uint8 [L, L]."""
    w = bits.astype(np.uint32)
    j = np.arange(L)
    return ((w[:, j // 32] >> (j % 32).astype(np.uint32)) & 1).astype(np.uint8)


@pytest.mark.parametrize("L", [37, 128, 512])
@pytest.mark.parametrize("lam", [0.5, 1.0])
def test_capture_per_map_scaling_matches_oracle(ora, L, lam):
    maps = inputs.averaged_maps(200 + L, 4, L=L, n_samples=3)
    for tau, mu in ((0.02, 0.5), (0.1, 0.3), (0.3, 0.05)):
        _same(_run(maps, lam=lam, tau=tau, mu=mu, scaling="map"),
              ora.capture(maps, lam=lam, tau=tau, mu=mu, scaling="map"))


@pytest.mark.parametrize("lam", [0.0, 0.25, 0.7, 1.5, 2.0, 3.0])
def test_capture_general_lambda_matches_oracle(ora, lam):
    # pow / log are not correctly rounded on either side; on these maps no entry lies
    # within their error of tau, so the lists agree exactly
    maps = inputs.averaged_maps(17, 4, L=256, n_samples=3)
    for scaling in ("row", "map"):
        tau = 0.3 if scaling == "row" else 0.05
        _same(_run(maps, lam=lam, tau=tau, mu=0.5, scaling=scaling),
              ora.capture(maps, lam=lam, tau=tau, mu=0.5, scaling=scaling))


def test_capture_scaling_fixture_true_masks(ora):
    # the hand-derived fixture (exact binary fractions, ties on tau), through the bitmap
    import json
    import os

    import structured_sparse_attention_b200 as ssa
    from conftest import GOLDEN
    fx = json.load(open(os.path.join(GOLDEN, "scaling_cases.json")))
    amap = np.array(fx["map"], np.float32)[None]
    for c in fx["cases"]:
        out = ssa.capture(torch.from_numpy(amap).to("cuda:0"), lam=c["lambda"], tau=c["tau"], eps=0.0,
                          scaling=c["scaling"], true_mask=True)
        M = _bits_to_mask(out["true_mask"][0].cpu().numpy(), 4)
        assert [M[i, :i + 1].tolist() for i in range(4)] == c["M"], c
        assert not np.triu(M, 1).any()


@pytest.mark.parametrize("L", [5, 100, 512, 700])
def test_capture_true_mask_bitmap_matches_oracle(ora, L):
    import structured_sparse_attention_b200 as ssa
    maps = inputs.averaged_maps(300 + L, 3, L=L, n_samples=2)
    for scaling in ("row", "map"):
        tau = 0.3 if scaling == "row" else 0.05
        out = ssa.capture(torch.from_numpy(maps).to("cuda:0"), tau=tau, scaling=scaling, true_mask=True)
        got = out["true_mask"].cpu().numpy()
        for m in range(len(maps)):
            np.testing.assert_array_equal(_bits_to_mask(got[m], L), ora.true_mask(maps[m], tau=tau, scaling=scaling))
        # the lists of the same call are those of the oracle
        dp = out["diag_ptr"].cpu().numpy()
        vp = out["vert_ptr"].cpu().numpy()
        _same((dp, out["diag_offsets"].cpu().numpy()[:dp[-1]], vp, out["vert_cols"].cpu().numpy()[:vp[-1]]),
              ora.capture(maps, tau=tau, scaling=scaling))


@pytest.mark.parametrize("scaling", ["row", "map"])
def test_capture_unaligned_maps_take_the_direct_loads(ora, scaling):
    # maps whose base is 4 bytes past a 16-byte boundary: rows are not staged by bulk
    # copies (they need 16-byte aligned rows) but loaded directly; same lists either way
    import structured_sparse_attention_b200 as ssa
    n, L = 5, 512
    maps = inputs.averaged_maps(41, n, L=L, n_samples=2)
    buf = torch.zeros(n * L * L + 4, dtype=torch.float32, device="cuda:0")
    view = buf[1:1 + n * L * L].view(n, L, L)
    view.copy_(torch.from_numpy(maps))
    assert view.data_ptr() % 16 == 4
    out = ssa.capture(view, scaling=scaling)
    dp, vp = out["diag_ptr"].cpu().numpy(), out["vert_ptr"].cpu().numpy()
    got = (dp, out["diag_offsets"].cpu().numpy()[:dp[-1]], vp, out["vert_cols"].cpu().numpy()[:vp[-1]])
    _same(got, ora.capture(maps, scaling=scaling))
    _same(got, _run(maps, scaling=scaling))
