"""The GEMMs' tile decoding, run on the CPU: tests/cpu_tile_decode.cu compiles
decode_tile / problem_id (ns_tiles.cuh, host-callable) with the planner
(plan.cpp) and checks that every output tile of every problem comes out
exactly once and in range, for the nanoGPT shapes and random shape mixes."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sign_muon_optimizer_b200", "csrc")


def _nvcc():
    for cand in ("/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    return None


@pytest.mark.skipif(_nvcc() is None, reason="no nvcc")
def test_every_output_tile_is_decoded_exactly_once(tmp_path):
    exe = str(tmp_path / "tile_decode")
    cmd = [_nvcc(), "-std=c++17", "-O1", "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           os.path.join(ROOT, "tests", "cpu_tile_decode.cu"), os.path.join(CSRC, "plan.cpp"), "-o", exe]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-3000:]
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "tile decode ok" in run.stdout
