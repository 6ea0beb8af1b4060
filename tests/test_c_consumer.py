"""The C ABI from plain C: tests/c_consumer.c is compiled as C99 against
include/signmuon.h, linked with libsignmuon.so and run (host-only calls; no
GPU needed)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "sign_muon_optimizer_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c99_program_plans_through_the_c_abi(tmp_path):
    if not os.path.exists(os.path.join(LIBDIR, "libsignmuon.so")):
        pytest.skip("libsignmuon.so is not built")
    exe = str(tmp_path / "c_consumer")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_consumer.c"), "-L", LIBDIR, "-lsignmuon", "-Wl,-rpath," + LIBDIR, "-o", exe]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, f"check {run.returncode} failed: {run.stdout}{run.stderr}"
    assert "c consumer ok: d=84934656 packed=10616832" in run.stdout
