"""Failure detection on the GPU without a fault: the bounded waits run out on purpose.

Every wait in the attention, averaged-maps and capture kernels gives up after the limit set by
ssa_set_wait_limit_ns.  With the limit at 0 the first wait that is not already complete
gives up; the kernel then records SSA_ERR_TIMEOUT (-5) in dev_status, stops every role,
drains its own copies and MMAs, frees tensor memory and returns.  The tests check that
the call returns with that status and that the same context then runs a normal call
that matches the oracle (nothing was left hung or corrupted).
"""

import numpy as np
import pytest
import torch

import structured_sparse_attention_b200 as ssa
from structured_sparse_attention_b200 import inputs
from gpu_util import compare_attn, dev, lists_to_device, t_bf16

pytestmark = pytest.mark.gpu

SSA_ERR_TIMEOUT = -5


class _zero_wait_limit:
    """ssa_set_wait_limit_ns(0) for the duration of a block, restored on exit."""

    def __enter__(self):
        self.old = ssa.set_wait_limit_ns(0)
        return self

    def __exit__(self, *exc):
        ssa.set_wait_limit_ns(self.old)
        return False


@pytest.mark.parametrize("d", [64, 128])
def test_attention_wait_expiry_returns_timeout_then_recovers(ora, d):
    S = 256
    diags = [np.arange(0, 96, dtype=np.int32)]
    verts = [np.array([0, 5, 200], np.int32)]
    (dp, do, vp, vo), host = lists_to_device(diags, verts)
    plan = ssa.extend(dp, do, vp, vo, S)
    q, k, v = inputs.qkv(31, 1, 1, S, d)
    tq, tk, tv = (t_bf16(a) for a in (q, k, v))
    status = torch.zeros(1, dtype=torch.int32, device=dev())
    with _zero_wait_limit():
        ssa.attn_fwd(tq, tk, tv, plan, status=status, check=False)
        torch.cuda.synchronize()
    assert int(status.item()) == SSA_ERR_TIMEOUT
    # the context is still usable: a normal call on it matches the oracle
    O, LSE = ssa.attn_fwd(tq, tk, tv, plan)
    ext = ora.extend(*host, S)
    Oref, Lref = ora.attn_dense(q, k, v, ext, d ** -0.5)
    compare_attn(O, LSE, Oref, Lref)


def test_maps_wait_expiry_returns_timeout_then_recovers(ora):
    n, B, L, d = 2, 2, 256, 64
    qs, ks = inputs.qk_samples(inputs.SEED_BASE + 1, n, B, L=L, d=d)
    tq, tk = t_bf16(qs), t_bf16(ks)
    status = torch.zeros(1, dtype=torch.int32, device=dev())
    with _zero_wait_limit():
        ssa.attn_maps(tq, tk, status=status, check=False)
        torch.cuda.synchronize()
    assert int(status.item()) == SSA_ERR_TIMEOUT
    got = ssa.attn_maps(tq, tk).cpu().numpy().astype(np.float64)
    want = ora.attn_maps(qs, ks, d ** -0.5)
    assert (np.abs(got - want) <= 2e-6 + 1e-4 * np.abs(want)).all()


def test_capture_wait_expiry_returns_timeout_then_recovers(ora):
    # rows are staged by bulk copies (16-byte aligned maps, L a multiple of 4) whose
    # waits share the limit; after an expired wait the CTA still waits (a fixed 1 s) for
    # its copies in flight before it exits
    n, L = 64, 512
    maps = inputs.averaged_maps(inputs.SEED_BASE + 11, n, L=L, n_samples=2)
    tm = torch.from_numpy(maps).to(dev())
    assert tm.data_ptr() % 16 == 0
    status = torch.zeros(1, dtype=torch.int32, device=dev())
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev())
    flush.fill_(1)  # the maps leave L2, so the row copies take DRAM latency
    with _zero_wait_limit():
        ssa.capture(tm, status=status, check=False)
        torch.cuda.synchronize()
    assert int(status.item()) == SSA_ERR_TIMEOUT
    out = ssa.capture(tm)
    dp, vp = out["diag_ptr"].cpu().numpy(), out["vert_ptr"].cpu().numpy()
    want = ora.capture(maps)
    np.testing.assert_array_equal(dp, want[0])
    np.testing.assert_array_equal(out["diag_offsets"].cpu().numpy()[:dp[-1]], want[1])
    np.testing.assert_array_equal(vp, want[2])
    np.testing.assert_array_equal(out["vert_cols"].cpu().numpy()[:vp[-1]], want[3])
