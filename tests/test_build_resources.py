"""Build-time resource checks of every kernel (nvcc -Xptxas -v, no GPU):
no kernel spills registers or keeps a stack frame (a register array indexed
by a runtime bound once moved the GEMM epilogue's accumulator to local memory
and halved its speed), and the 384-thread tcgen05 GEMM stays within the
register file (384 x 168 <= 65,536)."""
import os
import re
import shutil
import subprocess
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sign_muon_optimizer_b200", "csrc")
SOURCES = ["ns_tc.cu", "kernels_elem.cu", "kernels_ternary.cu", "ns_simt.cu", "noalloc.cu"]


def _nvcc():
    for cand in ("/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    return None


def _ptxas_report(nvcc, src, out_dir):
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "--expt-relaxed-constexpr",
           "-I", os.path.join(ROOT, "include"), "-Xptxas", "-v", "-c", os.path.join(CSRC, src),
           "-o", os.path.join(out_dir, src + ".o")]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-2000:]
    kernels = {}
    for block in res.stderr.split("Compiling entry function")[1:]:
        name = re.search(r"'([^']+)'", block).group(1)
        frame = re.search(r"(\d+) bytes stack frame, (\d+) bytes spill stores, (\d+) bytes spill loads", block)
        regs = re.search(r"Used (\d+) registers", block)
        kernels[name] = (tuple(int(x) for x in frame.groups()), int(regs.group(1)))
    return kernels


@pytest.mark.skipif(_nvcc() is None, reason="no nvcc")
def test_no_kernel_spills_or_keeps_a_stack_frame(tmp_path):
    nvcc = _nvcc()
    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        reports = list(ex.map(lambda s: _ptxas_report(nvcc, s, str(tmp_path)), SOURCES))
    found = {}
    for rep in reports:
        found.update(rep)
    assert len(found) >= 30
    for name, (frame, regs) in found.items():
        assert frame == (0, 0, 0), f"{name}: stack frame / spill stores / spill loads = {frame}"
    gemm = [regs for name, (_, regs) in found.items() if "k_gemm_tc" in name]
    assert gemm and max(gemm) * 384 <= 65536
