"""Register and spill budgets of the kernels, from the compiler's resource report
(nvcc -Xptxas -v for sm_100a), checked on the CPU.  Each launch relies on them:

* sparse_attn_fwd_kernel is launched with exactly kLaunchRegs registers per thread; its
  warpgroups then move registers between them with setmaxnreg, which can only hand out
  what the launch gave (the host refuses any other count at run time);
* capture_hits_kernel is planned at three CTAs of 256 threads per SM;
* attn_maps_kernel runs one CTA of 576 threads per SM.
The hot kernels must not spill; only the general-lambda transform of the capture (pow /
log, TR_POW), which the pages' settings never take, may.
"""

import concurrent.futures as cf
import os
import re
import shutil
import subprocess

import pytest

from conftest import ROOT

CSRC = os.path.join(ROOT, "structured_sparse_attention_b200", "csrc")
INCLUDE = os.path.join(ROOT, "include")
NVCC = "/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else shutil.which("nvcc")
REGS_PER_SM = 65536

pytestmark = pytest.mark.skipif(NVCC is None, reason="nvcc is not installed")


def _report(src, out_dir):
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-I", INCLUDE,
           "-Xptxas", "-v", "-c", os.path.join(CSRC, src), "-o", os.path.join(out_dir, src + ".o")]
    err = subprocess.run(cmd, capture_output=True, text=True, check=True).stderr
    kernels, cur = {}, None
    for line in err.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            cur = m.group(1)
            kernels[cur] = {"spill": 0}
            continue
        if cur is None:
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m:
            kernels[cur]["spill"] = int(m.group(1)) + int(m.group(2))
        m = re.search(r"Used (\d+) registers", line)
        if m:
            kernels[cur]["regs"] = int(m.group(1))
    return kernels


@pytest.fixture(scope="module")
def reports(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("ptxas"))
    files = ("attn_fwd.cu", "capture.cu", "maps.cu")
    with cf.ThreadPoolExecutor(max_workers=len(files)) as ex:
        futs = {f: ex.submit(_report, f, out) for f in files}
        return {f: fut.result() for f, fut in futs.items()}


def _constant(src, name):
    text = open(os.path.join(CSRC, src)).read()
    return int(re.search(rf"\b{name} = (\d+)", text).group(1))


def _select(report, name):
    found = {k: v for k, v in report.items() if name in k}
    assert found, f"no {name} in the compiler's report"
    return found


def test_attention_gets_exactly_the_launch_registers(reports):
    want = _constant("attn_fwd.cu", "kLaunchRegs")
    threads = _constant("attn_fwd.cu", "kThreads")
    assert threads * want <= REGS_PER_SM
    kernels = _select(reports["attn_fwd.cu"], "sparse_attn_fwd_kernel")
    assert len(kernels) == 2  # head dimensions 64 and 128
    for k, v in kernels.items():
        assert v["regs"] == want and v["spill"] == 0, (k, v)
    for k, v in _select(reports["attn_fwd.cu"], "stripe_gather_kernel").items():
        assert v["spill"] == 0, (k, v)


def test_capture_fits_three_ctas_per_sm(reports):
    threads = _constant("capture.cu", "kCaptureThreads")
    kernels = _select(reports["capture.cu"], "capture_hits_kernel")
    assert len(kernels) == 12  # 2 block counts x 3 transforms x 2 staging modes
    for k, v in kernels.items():
        assert 3 * threads * v["regs"] <= REGS_PER_SM, (k, v)
        transform = int(re.search(r"capture_hits_kernelILi\d+ELi(\d)E", k).group(1))
        if transform != 2:  # sqrt (lambda 1/2) and linear (lambda 1): no spills
            assert v["spill"] == 0, (k, v)


def test_maps_kernel_fits_one_cta_of_576_threads(reports):
    kernels = _select(reports["maps.cu"], "attn_maps_kernel")
    assert len(kernels) == 2
    for k, v in kernels.items():
        # 576 threads are 18 warps; the SM grants registers per warp in units of 256
        # and to warps in groups of four, so 20 warps' worth must fit (a 104-register
        # build, 20 x 3328 > 65536, was refused at launch; 96 registers fit)
        per_warp = -(-32 * v["regs"] // 256) * 256
        assert 20 * per_warp <= REGS_PER_SM, (k, v)
