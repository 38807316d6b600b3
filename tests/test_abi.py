"""The C ABI library builds, loads without a GPU and exports every symbol that
include/ssa.h declares; host-side argument checks return their documented codes."""

import ctypes as C
import os
import re

import pytest

from conftest import ROOT


@pytest.fixture(scope="module")
def lib():
    from structured_sparse_attention_b200 import binding, build
    build.build()
    return binding.load()


def _declared():
    src = open(os.path.join(ROOT, "include", "ssa.h")).read()
    return re.findall(r"SSA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)


def test_exports_every_declared_symbol(lib):
    from structured_sparse_attention_b200 import binding
    names = _declared()
    assert len(names) >= 9
    assert sorted(names) == sorted(binding.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_sizes(lib):
    assert lib.ssa_version() >= 100
    assert lib.sparse_pattern_capture_ws_bytes(512, 512) == 512 * (4 * 512 + 2) * 4
    # 256 bytes of scheduling counter + the gathered stripe keys and values
    assert lib.sparse_attn_fwd_ws_bytes(32, 128, 128) == 256 + 2 * 32 * 128 * 128 * 2
    assert lib.sparse_attn_fwd_ws_bytes(32, 129, 64) == 256 + 2 * 32 * 256 * 64 * 2
    assert lib.sparse_attn_fwd_ws_bytes(4, 0, 128) == 256
    assert lib.sparse_pattern_extend_ws_bytes(32, 65536) > 32 * 512 * 8


def test_host_argument_checks(lib):
    from structured_sparse_attention_b200 import binding
    P = C.c_void_p
    dummy = P(256)
    # lambda outside [0, 64], an unknown scaling and an unsupported L are rejected
    # before any device work
    rc = lib.sparse_pattern_capture(dummy, 1, 16, -0.5, 0.3, 0.8, 1e-8, dummy, dummy, dummy, dummy,
                                    dummy, 1 << 20, None, None)
    assert rc == -1 and b"lambda" in lib.ssa_last_error()
    rc = lib.sparse_pattern_capture_ex(dummy, 1, 16, 0.5, 0.3, 0.8, 1e-8, 2, dummy, dummy, dummy, dummy,
                                       None, dummy, 1 << 20, None, None)
    assert rc == -1 and b"scaling" in lib.ssa_last_error()
    rc = lib.sparse_pattern_capture(dummy, 1, 2048, 0.5, 0.3, 0.8, 1e-8, dummy, dummy, dummy, dummy,
                                    dummy, 1 << 30, None, None)
    assert rc == -2
    rc = lib.sparse_pattern_capture(None, 1, 16, 0.5, 0.3, 0.8, 1e-8, dummy, dummy, dummy, dummy,
                                    dummy, 1 << 20, None, None)
    assert rc == -1
    rc = lib.sparse_pattern_capture(dummy, 4, 16, 0.5, 0.3, 0.8, 1e-8, dummy, dummy, dummy, dummy,
                                    dummy, 10, None, None)
    assert rc == -3
    # head dimension other than 64 / 128
    plan = binding.PlanStruct()
    plan.S, plan.n_heads, plan.nqb = 256, 1, 2
    rc = lib.sparse_attn_fwd(dummy, dummy, dummy, 1, 1, 256, 96, C.byref(plan), None, 0.1, dummy, dummy,
                             None, 0, None, None)
    assert rc == -2
    # plan / shape mismatch
    rc = lib.sparse_attn_fwd(dummy, dummy, dummy, 1, 1, 300, 64, C.byref(plan), None, 0.1, dummy, dummy,
                             None, 0, None, None)
    assert rc == -1 and b"plan" in lib.ssa_last_error()
    # averaged maps: sizes and head dimension are checked before any device work
    for n, B, L, d, want in [(1, 2, 200, 64, -1), (1, 0, 128, 64, -1), (1, 33, 128, 64, -1),
                             (1, 2, 128, 96, -2), (1, 2, 8192, 64, -1), (1 << 20, 1, 4096, 64, -1)]:
        rc = lib.sparse_attn_maps(dummy, dummy, n, B, L, d, 0.125, dummy, None, None)
        assert rc == want, (n, B, L, d, rc)
    rc = lib.sparse_attn_maps(dummy, dummy, 1, 2, 128, 64, 0.0, dummy, None, None)
    assert rc == -1 and b"scale" in lib.ssa_last_error()
    rc = lib.sparse_attn_maps(P(8), dummy, 1, 2, 128, 64, 0.125, dummy, None, None)
    assert rc == -1 and b"aligned" in lib.ssa_last_error()
    # extend: bad sizes
    sizes = binding.PlanSizes()
    rc = lib.sparse_pattern_extend(0, dummy, dummy, dummy, dummy, 10, C.byref(sizes), None, dummy, 1 << 20,
                                   None, None)
    assert rc == -1


def test_decode_rejects_case2_plans_before_any_device_work(lib):
    # element-bitmap tiles are a prefill-only plan form: decoding says so on the host
    from structured_sparse_attention_b200 import binding
    dummy = C.c_void_p(256)
    plan = binding.PlanStruct()
    plan.S, plan.n_heads, plan.nqb, plan.bitmap_slots = 256, 1, 2, 3
    pos = C.c_void_p(256)
    rc = lib.sparse_attn_decode(dummy, dummy, dummy, 1, 1, 1, 256, 64, pos, C.byref(plan), None, 0.1, dummy,
                                dummy, dummy, 1 << 20, None, None)
    assert rc == -2 and b"Case-2" in lib.ssa_last_error()


def test_wait_limit_knob(lib):
    old = lib.ssa_set_wait_limit_ns(12345)
    assert lib.ssa_set_wait_limit_ns(old) == 12345


def test_product_path_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "structured_sparse_attention_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"(from|import)\s+oracle|libssa_oracle|ssa_oracle|\bora_\w+\(", txt), f


def test_binding_rejects_host_tensors_before_any_call(lib):
    # the binding marshals CUDA tensors only: host tensors fail loudly, nothing falls back
    import torch

    from structured_sparse_attention_b200 import binding
    q = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16)
    with pytest.raises(binding.SSAError) as e:
        binding.attn_maps(q, q)
    assert e.value.code == -1 and "CUDA" in str(e.value)
    with pytest.raises(binding.SSAError):
        binding.capture(torch.zeros((1, 16, 16), dtype=torch.float32))
    with pytest.raises(binding.SSAError):
        binding.extend(*(torch.zeros(2, dtype=torch.int32) for _ in range(4)), 64)
    with pytest.raises(binding.SSAError) as e:
        binding.refill(object(), *(torch.zeros(2, dtype=torch.int32) for _ in range(4)))
    assert e.value.code == -1 and "CUDA" in str(e.value)


def test_oracle_shares_no_code_with_the_library():
    # the oracle includes only the C standard library and imports nothing of the package
    src = open(os.path.join(ROOT, "oracle", "ssa_oracle.c")).read()
    assert set(re.findall(r"#include\s*<([^>]+)>", src)) <= {"math.h", "stdint.h", "stdlib.h", "string.h"}
    assert not re.search(r'#include\s*"', src)
    py = open(os.path.join(ROOT, "oracle", "oracle.py")).read()
    assert not re.search(r"structured_sparse_attention_b200|libssa\.so|import\s+ssa\b", py)
