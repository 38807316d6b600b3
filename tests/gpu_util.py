"""Helpers shared by the GPU parity tests (host <-> device marshalling only)."""

import numpy as np
import torch

from structured_sparse_attention_b200 import inputs

# Tolerances on the attention outputs against the fp64 oracle (bf16 in, fp32 accumulate).
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3


def dev():
    return torch.device("cuda:0")


def t_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev())


def t_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev()).view(torch.bfloat16)


def lists_to_device(diags, verts):
    dp, do = inputs.to_csr(diags)
    vp, vo = inputs.to_csr(verts)
    if len(do) == 0:
        do = np.zeros(1, np.int32)
    if len(vo) == 0:
        vo = np.zeros(1, np.int32)
    return (t_i32(dp), t_i32(do), t_i32(vp), t_i32(vo)), (dp, do[:dp[-1]], vp, vo[:vp[-1]])


def sample_rows(S, n, seed):
    """Seeded rows covering the first block, the last full block, the tail and random rows."""
    g = np.random.default_rng(seed)
    rows = set(range(min(S, 128)))
    last_full = (S // 128) * 128
    rows.update(range(max(0, last_full - 128), last_full))
    rows.update(range(last_full, S))
    rows.update(g.integers(0, S, size=n).tolist())
    return np.array(sorted(rows), dtype=np.int32)


def compare_attn(O, LSE, Oref, Lref, rows=None):
    """O [H,S,d] bf16 / LSE [H,S] from the GPU vs oracle fp64 arrays on the given rows."""
    o = O.float().cpu().numpy().astype(np.float64)
    l = LSE.cpu().numpy().astype(np.float64)
    if rows is not None:
        o = o[:, rows]
        l = l[:, rows]
    empty = np.isneginf(Lref)
    assert (np.isneginf(l) == empty).all(), "empty-row pattern differs"
    assert (o[empty] == 0).all(), "empty rows must give O = 0"
    err = np.abs(o - Oref)
    lerr = np.abs(l[~empty] - Lref[~empty]) if (~empty).any() else np.zeros(1)
    stats = dict(o_max=float(err.max()), o_mean=float(err.mean()), lse_max=float(lerr.max()))
    assert stats["o_max"] <= O_MAX_ABS and stats["o_mean"] <= O_MEAN_ABS, stats
    assert stats["lse_max"] <= LSE_MAX_ABS, stats
    return stats
