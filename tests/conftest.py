import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 and the built CUDA library")
    # a fresh checkout has no libsignmuon.so (built files are not committed):
    # build it once before any test imports the package, when nvcc is here
    lib = os.path.join(ROOT, "sign_muon_optimizer_b200", "libsignmuon.so")
    if not os.path.exists(lib) and (shutil.which("nvcc") or os.path.exists("/usr/local/cuda/bin/nvcc")):
        import importlib.util
        spec = importlib.util.spec_from_file_location(
            "signmuon_build", os.path.join(ROOT, "sign_muon_optimizer_b200", "build.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod.build()
