"""The allocation-free capture entry point (sparse_pattern_capture_noalloc).

Some callers cannot allocate device memory: a plugin host that only hands the library
its input and output buffers has no allocator to lend it, and a serving process that
must not call cudaMalloc/cudaFree after start-up (they can synchronise the device and
stall other streams) cannot let the library allocate either.  This entry point keeps
its scratch in a fixed device array inside the library instead of a caller workspace.

The test calls it through the C ABI and checks that calls in a row (the second keeping
fewer patterns than the first from the same number of maps) give exactly the kept lists
of the oracle and of the regular entry point (lists are integers: bit-exact), and that
a size beyond the fixed scratch is rejected.  It must pass alone in a fresh process and
after the rest of the suite, so it creates everything it needs itself.
"""

import ctypes as C

import numpy as np
import pytest
import torch

from structured_sparse_attention_b200 import inputs

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 8 << 20  # SSA_CAPTURE_NOALLOC_SCRATCH_BYTES


def _lib():
    import structured_sparse_attention_b200 as ssa
    lib = ssa.load()
    V, I, D = C.c_void_p, C.c_int, C.c_double
    lib.sparse_pattern_capture_noalloc.argtypes = [V, I, I, D, D, D, D, V, V, V, V, V, V]
    lib.sparse_pattern_capture_noalloc.restype = I
    return ssa, lib


def _noalloc(lib, maps_dev, lam=0.5, tau=0.3, mu=0.8, eps=1e-8):
    n, L, _ = maps_dev.shape
    dev = maps_dev.device
    # outputs pre-filled with garbage so stale values cannot pass for results
    out = [torch.full((n + 1,), -7, dtype=torch.int32, device=dev),
           torch.full((n * L,), -7, dtype=torch.int32, device=dev),
           torch.full((n + 1,), -7, dtype=torch.int32, device=dev),
           torch.full((n * L,), -7, dtype=torch.int32, device=dev)]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    p = lambda t: C.c_void_p(t.data_ptr())
    rc = lib.sparse_pattern_capture_noalloc(p(maps_dev), n, L, lam, tau, mu, eps, p(out[0]), p(out[1]),
                                            p(out[2]), p(out[3]), p(status), C.c_void_p(stream.cuda_stream))
    assert rc == 0, lib.ssa_last_error()
    stream.synchronize()
    assert int(status.item()) == 0
    dp, vp = out[0].cpu().numpy(), out[2].cpu().numpy()
    return dp, out[1].cpu().numpy()[:dp[-1]], vp, out[3].cpu().numpy()[:vp[-1]]


def _regular(ssa, maps_dev, **kw):
    out = ssa.capture(maps_dev, **kw)
    dp, vp = out["diag_ptr"].cpu().numpy(), out["vert_ptr"].cpu().numpy()
    return dp, out["diag_offsets"].cpu().numpy()[:dp[-1]], vp, out["vert_cols"].cpu().numpy()[:vp[-1]]


def test_noalloc_capture_matches_oracle_and_regular_on_calls_in_a_row():
    from oracle import oracle as ora
    ora.build()
    ssa, lib = _lib()
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    # call 1: a model's worth of maps at L = 512; call 2: the same maps with stricter
    # thresholds, so it keeps fewer patterns per map with the same map count (staging
    # or counts left by call 1 must not leak into its lists); call 3: another size
    a_h = inputs.averaged_maps(inputs.SEED_BASE + 2, 64, L=512, n_samples=4)
    b_h = inputs.averaged_maps(991, 40, L=300, n_samples=3)
    a, b = torch.from_numpy(a_h).to(dev), torch.from_numpy(b_h).to(dev)
    calls = ((a, a_h, {}), (a, a_h, dict(tau=0.5, mu=0.97)), (b, b_h, dict(tau=0.25, mu=0.7)))
    kept = []
    for maps, maps_h, kw in calls:
        got = _noalloc(lib, maps, **kw)
        want = ora.capture(maps_h, **kw)
        regular = _regular(ssa, maps, **kw)
        for x, y, z, name in zip(got, want, regular, ("diag_ptr", "diag_offsets", "vert_ptr", "vert_cols")):
            np.testing.assert_array_equal(x, y, err_msg=name)
            np.testing.assert_array_equal(x, z, err_msg=name)
        assert got[0][-1] > 0 and got[2][-1] > 0
        kept.append(int(got[0][-1]) + int(got[2][-1]))
    assert kept[1] < kept[0], kept  # the second call keeps fewer patterns than the first


def test_noalloc_rejects_sizes_beyond_the_scratch():
    ssa, lib = _lib()
    n, L = 1024, 512  # 1024 * (4 * 512 + 2) * 4 bytes > 8 MiB
    assert lib.sparse_pattern_capture_ws_bytes(n, L) > SCRATCH_BYTES
    assert lib.sparse_pattern_capture_ws_bytes(1023, L) <= SCRATCH_BYTES
    dummy = C.c_void_p(256)  # never dereferenced: the size check comes first
    rc = lib.sparse_pattern_capture_noalloc(dummy, n, L, 0.5, 0.3, 0.8, 1e-8, dummy, dummy, dummy, dummy,
                                            None, None)
    assert rc == -3
    assert b"scratch" in lib.ssa_last_error()
