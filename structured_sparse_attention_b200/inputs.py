"""Seeded synthetic inputs shared by the tests, the benchmark and the CPU oracle.

This module only draws random numbers and lays them out.  It holds none of the
arithmetic of the method (no Box-Cox, no thresholding, no scoring, no attention),
so that both the CUDA path and the oracle can be fed from it without sharing any
of the computation they are compared on.

Workload shapes follow the DAM review page ("DAM: Dynamic Attention Mask for
Long-Context Large Language Model Inference Acceleration", pith review of arXiv
2506.11104): a pattern capture length L = 512 ("What carries the argument",
"Assumptions & free parameters"), LLaMA-3.2-1B / LLaMA-3-8B shaped layers and
prefill lengths of 16K, 64K and up to 104K tokens ("The reading", "If this is
right").  The pages evaluate on Multi-News, LongEval and LV-Eval with trained
weights; none of those are available, so seeded Gaussian Q/K/V and seeded
planted-pattern attention maps stand in for them.

Conventions
-----------
* Q, K, V are returned as raw bf16 bit patterns (``uint16``), layout ``[H][S][d]``,
  obtained from float32 N(0, 1) samples by round-to-nearest-even.
* Pattern lists are per-head sorted, duplicate-free int32 arrays: ``diag`` holds the
  diagonal offsets r (key j = i - r), ``vert`` the vertical columns c (key j = c,
  for queries i >= c).  ``to_csr`` packs them as (ptr, values) pairs.
* Every generator takes an explicit seed; sub-streams come from
  ``numpy.random.SeedSequence(seed).spawn`` driving NumPy's SFC64 bit generator.
  The split into sub-streams (one per head / map) is fixed, so the values do not
  depend on how many threads fill them.
"""

from __future__ import annotations

import concurrent.futures as _cf
import os

import numpy as np

SEED_BASE = 20261200

#: Row-block / key-tile edge used by the tile plan (fixed by the CUDA kernels).
BLOCK = 128


def _gen(ss) -> np.random.Generator:
    return np.random.Generator(np.random.SFC64(ss))


def _streams(seed: int, n: int) -> list[np.random.Generator]:
    return [_gen(s) for s in np.random.SeedSequence(seed).spawn(n)]


def _pmap(fn, items):
    workers = max(1, min(len(items), os.cpu_count() or 1, 32))
    if workers == 1:
        return [fn(x) for x in items]
    with _cf.ThreadPoolExecutor(workers) as ex:
        return list(ex.map(fn, items))


# --------------------------------------------------------------------------------------
# bf16 bit handling (layout only: float32 <-> bf16 storage conversion)
# --------------------------------------------------------------------------------------

def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    rounded = u + np.uint32(0x7FFF) + lsb
    return (rounded >> np.uint32(16)).astype(np.uint16)


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(seed: int, H: int, S: int, d: int) -> np.ndarray:
    """[H, S, d] bf16 bits of i.i.d. N(0,1) float32 samples, one sub-stream per head."""
    out = np.empty((H, S, d), np.uint16)
    seqs = np.random.SeedSequence(seed).spawn(H)

    def fill(h):
        out[h] = bf16_bits_from_f32(_gen(seqs[h]).standard_normal((S, d), dtype=np.float32))

    _pmap(fill, list(range(H)))
    return out


def qkv(seed: int, H_q: int, H_kv: int, S: int, d: int):
    """Q [H_q,S,d], K [H_kv,S,d], V [H_kv,S,d] as bf16 bits from i.i.d. N(0,1)."""
    sq, sk, sv = (int(x.generate_state(1)[0]) for x in np.random.SeedSequence(seed).spawn(3))
    return normal_bf16(sq, H_q, S, d), normal_bf16(sk, H_kv, S, d), normal_bf16(sv, H_kv, S, d)


# --------------------------------------------------------------------------------------
# Pattern lists
# --------------------------------------------------------------------------------------

def to_csr(lists: list[np.ndarray]) -> tuple[np.ndarray, np.ndarray]:
    ptr = np.zeros(len(lists) + 1, dtype=np.int32)
    for h, a in enumerate(lists):
        ptr[h + 1] = ptr[h] + len(a)
    vals = np.concatenate([np.asarray(a, dtype=np.int32) for a in lists]) if lists else np.zeros(0, np.int32)
    return ptr, np.ascontiguousarray(vals, dtype=np.int32)


def from_csr(ptr: np.ndarray, vals: np.ndarray) -> list[np.ndarray]:
    return [np.asarray(vals[ptr[h]:ptr[h + 1]], dtype=np.int32) for h in range(len(ptr) - 1)]


def _distinct_sorted(g: np.random.Generator, lo: int, hi: int, n: int) -> np.ndarray:
    n = min(n, hi - lo)
    return np.sort(g.choice(np.arange(lo, hi, dtype=np.int64), size=n, replace=False)).astype(np.int32)


def random_patterns(seed: int, n_heads: int, S: int, max_diag: int, max_vert: int):
    """Fuzz patterns: per head a random number of distinct diagonals and columns in [0, S).

    Offsets near 0 and S-1 are drawn with extra weight so edge tiles get exercised.
    """
    gs = _streams(seed, n_heads)
    diags, verts = [], []
    for g in gs:
        nd = int(g.integers(0, max_diag + 1))
        nv = int(g.integers(0, max_vert + 1))
        d = set(_distinct_sorted(g, 0, S, nd).tolist())
        if g.random() < 0.5:
            d.add(0)
        if g.random() < 0.3:
            d.add(S - 1)
        v = set(_distinct_sorted(g, 0, S, nv).tolist())
        if g.random() < 0.3:
            v.add(S - 1)
        if g.random() < 0.3:
            v.add(0)
        diags.append(np.array(sorted(d), dtype=np.int32))
        verts.append(np.array(sorted(v), dtype=np.int32))
    return diags, verts


def patterns_small_single_head():
    """Single head at S=512, d=64: diagonals r = 0..63 and columns c = 0..3."""
    return [np.arange(64, dtype=np.int32)], [np.arange(4, dtype=np.int32)]


def patterns_gqa_16k(seed: int, n_heads: int = 32, S: int = 16384):
    """LLaMA-3.2-1B-shaped layer at S=16384: diagonals 0..511 for every head; columns
    {0,1,2,3} plus n_h - 4 distinct columns drawn from [512, S) with n_h ~ U{32..64}."""
    gs = _streams(seed, n_heads)
    diags, verts = [], []
    for g in gs:
        n_h = int(g.integers(32, 65))
        extra = _distinct_sorted(g, 512, S, n_h - 4)
        diags.append(np.arange(512, dtype=np.int32))
        verts.append(np.concatenate([np.arange(4, dtype=np.int32), extra]).astype(np.int32))
    return diags, verts


def patterns_band_random(seed: int, n_heads: int = 32, S: int = 65536, width: int = 1024, n_vert: int = 128):
    """LLaMA-3-8B-shaped layer: per head a contiguous run of `width` diagonals starting at
    r0 ~ U{0..S-width} and `n_vert` distinct columns drawn uniformly from [0, S)."""
    gs = _streams(seed, n_heads)
    diags, verts = [], []
    for g in gs:
        r0 = int(g.integers(0, S - width + 1))
        diags.append(np.arange(r0, r0 + width, dtype=np.int32))
        verts.append(_distinct_sorted(g, 0, S, n_vert))
    return diags, verts


#: (band width W, number of columns V) for the long-context density sweep; the
#: ratio V ~ W/8 follows the 64K layer.  None marks full causal attention.
DENSITY_POINTS = {"0.5": (245, 31), "2": (984, 123), "10": (5038, 630), "100": None}


def patterns_density(seed: int, density: str, n_heads: int = 24, S: int = 104000):
    """Long-context sweep: diagonals 0..W-1 for every head and V distinct random columns
    per head; density "100" is plain causal attention (all diagonals, no columns)."""
    point = DENSITY_POINTS[density]
    if point is None:
        return ([np.arange(S, dtype=np.int32) for _ in range(n_heads)],
                [np.zeros(0, dtype=np.int32) for _ in range(n_heads)])
    W, V = point
    gs = _streams(seed, n_heads)
    diags = [np.arange(W, dtype=np.int32) for _ in range(n_heads)]
    verts = [_distinct_sorted(g, 0, S, V) for g in gs]
    return diags, verts


# --------------------------------------------------------------------------------------
# Averaged attention maps for pattern capture
# --------------------------------------------------------------------------------------

def planted_map_patterns(seed: int, n_maps: int, L: int = 512):
    """Per map the planted diagonals (n_d ~ U{1..8}) and columns (n_c ~ U{1..16})."""
    gs = _streams(seed, n_maps)
    out = []
    for g in gs:
        nd = int(g.integers(1, 9))
        nc = int(g.integers(1, 17))
        out.append((_distinct_sorted(g, 0, L, nd), _distinct_sorted(g, 0, L, nc)))
    return out


def averaged_maps(seed: int, n_maps: int, L: int = 512, n_samples: int = 16, boost: float = 4.0,
                  map_ids=None) -> np.ndarray:
    """Synthetic batch-averaged causal attention maps, float32 [n, L, L].

    Map m is the mean over `n_samples` draws of a causal row-softmax of N(0,1) logits
    with `boost` added on the planted diagonals and columns of map m.  Entries above
    the diagonal are 0.  Each map has its own random stream, so any subset
    (`map_ids`) reproduces exactly the same maps as the full set.
    """
    ids = list(range(n_maps)) if map_ids is None else list(map_ids)
    planted = planted_map_patterns(seed, n_maps, L)
    sample_seeds = np.random.SeedSequence(seed + 7919).spawn(n_maps)
    ii, jj = np.meshgrid(np.arange(L), np.arange(L), indexing="ij")
    causal = jj <= ii
    out = np.zeros((len(ids), L, L), dtype=np.float32)

    def one(o):
        m = ids[o]
        dg, cl = planted[m]
        bonus = np.zeros((L, L), dtype=np.float32)
        for r in dg:
            bonus[(ii - jj) == r] = boost
        bonus[:, cl] = boost
        bonus[~causal] = -np.inf
        g = _gen(sample_seeds[m])
        acc = np.zeros((L, L), dtype=np.float64)
        for _ in range(n_samples):
            z = g.standard_normal((L, L), dtype=np.float32) + bonus
            z -= z.max(axis=1, keepdims=True)
            e = np.exp(z)
            acc += e / e.sum(axis=1, keepdims=True)
        out[o] = (acc / n_samples).astype(np.float32)

    _pmap(one, list(range(len(ids))))
    return out


# --------------------------------------------------------------------------------------
# Per-head query/key samples for producing the averaged maps on the GPU
# --------------------------------------------------------------------------------------

def qk_samples(seed: int, n_maps: int, B: int, L: int = 512, d: int = 64, planted: bool = True,
               map_ids=None):
    """Query and key rows of B calibration samples per map, bf16 bits [n, B, L, d] each.

    Entries are N(0, 1).  With `planted`, map m gets its planted columns
    (`planted_map_patterns`) as keys that every query favours: a unit direction u_m is
    added (x 4.5) to every query row and to the key rows of those columns; and a local
    diagonal: each key row also gets 0.35 x its own query row.  Each map has its own
    random stream, so a subset (`map_ids`) reproduces the same rows as the full set.
    """
    ids = list(range(n_maps)) if map_ids is None else list(map_ids)
    pl = planted_map_patterns(seed, n_maps, L)
    streams = np.random.SeedSequence(seed + 104729).spawn(n_maps)
    q_out = np.empty((len(ids), B, L, d), np.uint16)
    k_out = np.empty((len(ids), B, L, d), np.uint16)

    def one(o):
        m = ids[o]
        g = _gen(streams[m])
        u = g.standard_normal(d).astype(np.float32)
        u /= np.float32(np.linalg.norm(u))
        for b in range(B):
            q = g.standard_normal((L, d), dtype=np.float32)
            k = g.standard_normal((L, d), dtype=np.float32)
            if planted:
                q += np.float32(4.5) * u
                k[pl[m][1]] += np.float32(4.5) * u
                k += np.float32(0.35) * q
            q_out[o, b] = bf16_bits_from_f32(q)
            k_out[o, b] = bf16_bits_from_f32(k)

    _pmap(one, list(range(len(ids))))
    return q_out, k_out
