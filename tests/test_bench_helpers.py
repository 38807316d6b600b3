"""Host helpers of bench.py that its numbers rest on, checked on CPU.

* nnz_per_head: the retained pairs of the extended mask from the list form, by integer
  counting with the cells on both a diagonal and a column counted once; against a cell
  by cell count of the mask (DAM review page, "Circularity Check" step 1: the mask is the
  union of the kept patterns).
* profiled_traffic: the DRAM bytes per launch are taken from the machine-readable ncu
  record only while the attention sources hash to the value recorded with it.
"""

import json

import numpy as np
import pytest

import bench


def _brute_nnz(D, C, S):
    i, j = np.tril_indices(S)
    on = np.isin(i - j, D) | np.isin(j, C)
    return int(on.sum())


@pytest.mark.parametrize("seed", range(6))
def test_nnz_per_head_matches_a_cell_count(seed):
    g = np.random.default_rng(seed)
    S = int(g.integers(1, 300))
    diags, verts = [], []
    for _ in range(3):
        D = np.unique(g.integers(0, S + 20, size=int(g.integers(0, 40)))).astype(np.int32)
        C = np.unique(g.integers(0, S + 20, size=int(g.integers(0, 20)))).astype(np.int32)
        diags.append(D)
        verts.append(C)
    got = bench.nnz_per_head(diags, verts, S)
    want = [_brute_nnz(D[D < S], C[C < S], S) for D, C in zip(diags, verts)]
    assert got.tolist() == want


def test_nnz_per_head_closed_forms():
    S = 1000
    # every diagonal: all causal pairs; one column c: the S - c rows at or below it
    assert bench.nnz_per_head([np.arange(S, dtype=np.int32)], [np.zeros(0, np.int32)], S)[0] == S * (S + 1) // 2
    assert bench.nnz_per_head([np.zeros(0, np.int32)], [np.array([7], np.int32)], S)[0] == S - 7
    # the main diagonal and column 0 share the cell (0, 0) only
    assert bench.nnz_per_head([np.array([0], np.int32)], [np.array([0], np.int32)], S)[0] == S + S - 1


def test_profiled_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "attn_source_hash", lambda: "0123456789abcdef")
    assert bench.profiled_traffic("w") is None  # no record
    rec = {"traffic_bytes_per_launch": 12345, "source_sha256_16": "0123456789abcdef"}
    (prof / "sparse_attn_fwd_w_dram.json").write_text(json.dumps(rec))
    assert bench.profiled_traffic("w") == 12345.0
    rec["source_sha256_16"] = "ffffffffffffffff"  # taken on other sources: not reported
    (prof / "sparse_attn_fwd_w_dram.json").write_text(json.dumps(rec))
    assert bench.profiled_traffic("w") is None


def test_committed_traffic_record_is_current():
    # the record in profiles/ was taken on the attention sources as committed
    assert bench.profiled_traffic("llama3-8b-layer-64k") is not None


def test_peaks_measured_else_the_stated_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_peaks() == (6650.0, 1590.0, 1400.0, "fallback")
    assert bench.sm_max_mhz() == 1965.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6545.9, "bf16_tflops": 1667.7, "bf16_tflops_sustained": 1368.0, "sm_max_mhz": 1950.0}))
    assert bench.load_peaks() == (6545.9, 1667.7, 1368.0, "measured")
    assert bench.sm_max_mhz() == 1950.0
