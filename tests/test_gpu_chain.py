"""The whole path on the GPU: capture -> extend -> attention, fed by the GPU's own lists.

The averaged maps of one layer (32 heads at L = 512, 16 samples) are captured on the
GPU; the device lists go straight into sparse_pattern_extend at S = 16384 and then into
sparse_attn_fwd (32 Q / 8 KV heads, d = 64).  The oracle takes the same maps through its
own capture, extension and row-wise attention (DAM page, "What carries the argument":
patterns captured at L, pasted onto the long sequence).  Lists are compared exactly,
attention on sampled rows within the stated tolerances.
"""

import numpy as np
import pytest

import structured_sparse_attention_b200 as ssa
from structured_sparse_attention_b200 import inputs
from gpu_util import compare_attn, dev, sample_rows, t_bf16

pytestmark = pytest.mark.gpu


def test_capture_extend_attention_chain(ora):
    import torch
    L, S, Hq, Hkv, d = 512, 16384, 32, 8, 64
    maps = inputs.averaged_maps(inputs.SEED_BASE + 2, 512, L=L, n_samples=16, map_ids=range(Hq))
    cap = ssa.capture(torch.from_numpy(maps).to(dev()))
    dp, do, vp, vc = ora.capture(maps)
    got = [cap[k].cpu().numpy() for k in ("diag_ptr", "diag_offsets", "vert_ptr", "vert_cols")]
    assert np.array_equal(got[0], dp) and np.array_equal(got[2], vp)
    assert np.array_equal(got[1][:dp[-1]], do) and np.array_equal(got[3][:vp[-1]], vc)
    # the capture's device lists feed the extension directly
    plan = ssa.extend(cap["diag_ptr"], cap["diag_offsets"], cap["vert_ptr"], cap["vert_cols"], S)
    q, k, v = inputs.qkv(inputs.SEED_BASE + 33, Hq, Hkv, S, d)
    O, LSE = ssa.attn_fwd(t_bf16(q), t_bf16(k), t_bf16(v), plan)
    ext = ora.extend(dp, do, vp, vc, S)
    rows = sample_rows(S, 256, 9)
    Oref, Lref = ora.attn_rows(q, k, v, ext, d ** -0.5, rows)
    compare_attn(O, LSE, Oref, Lref, rows)
