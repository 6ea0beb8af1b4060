"""CPU-side checks of the C ABI: the library loads, exports every symbol the
header declares, and the host-only planner validates and sizes plans like
signmuon_init would (no GPU calls)."""
import ctypes
import os
import re

import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "signmuon.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(signmuon_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    import sign_muon_optimizer_b200 as smo
    lib = ctypes.CDLL(smo.LIB_PATH)
    names = _declared()
    assert len(names) >= 20
    for n in names:
        assert hasattr(lib, n), f"{n} declared in signmuon.h but not exported"
    assert sorted(smo.EXPORTED) == names


def test_plan_sizes_for_the_workloads():
    import sign_muon_optimizer_b200 as smo
    p = smo.signmuon_plan(synth.NANOGPT_SHAPES, 8, 5, "spectral", 2)
    assert p["d"] == 84_934_656 and p["packed_bytes"] == 10_616_832 and p["groups"] == 4
    p = smo.signmuon_plan(synth.RESNET50_SHAPES, 4, 5, "spectral", 2)
    assert p["d"] == 25_502_912 and p["n_mats"] == 54
    p = smo.signmuon_plan(synth.LLAMA_LAYER_SHAPES, 16, flags=smo.SIGNMUON_VOTE_ONLY)
    assert p["d"] == 717_225_984 and p["packed_bytes"] == 89_653_248 and p["device_bytes"] == 0
    p = smo.signmuon_plan([(3, 5)], 1)
    assert p["packed_bytes"] == 2  # ceil(15/8)


@pytest.mark.parametrize("shapes,M,K,scale,P,flags,status", [
    ([(3, 0)], 2, 5, "fro", 1, 0, 1),
    ([(3, 3)], 0, 5, "fro", 1, 0, 1),
    ([(3, 3)], 257, 5, "fro", 1, 0, 1),
    ([(3, 3)], 2, -1, "fro", 1, 0, 1),
    ([(3, 3)], 2, 5, "spectral", 0, 0, 1),
    ([(3, 3)], 128, 5, "fro", 1, 1 << 3, 2),
    ([(70000, 70000)], 1, 5, "fro", 1, 0, 1),
])
def test_plan_rejects_invalid(shapes, M, K, scale, P, flags, status):
    import sign_muon_optimizer_b200 as smo
    with pytest.raises(smo.SignMuonError) as e:
        smo.signmuon_plan(shapes, M, K, scale, P, flags)
    assert e.value.status == status
    assert smo.signmuon_last_error(None)


def test_init_validation_without_gpu():
    # argument checks run before any CUDA call
    import sign_muon_optimizer_b200 as smo
    for kw in (dict(beta=1.0), dict(beta=-0.1), dict(lam=-1.0), dict(eps=0.0)):
        args = dict(beta=0.9, lam=0.0, K=5, eps=1e-7, scale="fro", P=1)
        args.update(kw)
        with pytest.raises(smo.SignMuonError) as e:
            smo.signmuon_init([(4, 4)], 2, args["beta"], args["lam"], args["K"], args["eps"], args["scale"],
                              args["P"])
        assert e.value.status == smo.SIGNMUON_E_INVALID


def test_status_strings():
    import sign_muon_optimizer_b200 as smo
    for s in range(8):
        assert smo.signmuon_status_string(s)


# POLAR_AFTER_ONLY (1 << 8) without POST_POLAR (1 << 2); MUON_MEAN (1 << 9)
# with the post-vote polar step or a sign wire flag (TERNARY 1 << 10,
# NORMALIZED_SIGN 1 << 11); NORMALIZED_SIGN with POST_POLAR
BAD_FLAG_SETS = [1 << 8, (1 << 9) | (1 << 2), (1 << 9) | (1 << 8) | (1 << 2), (1 << 9) | (1 << 10),
                 (1 << 9) | (1 << 11), (1 << 11) | (1 << 2), (1 << 11) | (1 << 8) | (1 << 2)]


@pytest.mark.parametrize("flags", BAD_FLAG_SETS)
def test_init_rejects_variant_flag_combinations(flags):
    # checked before any CUDA call: runs without a GPU
    import sign_muon_optimizer_b200 as smo
    assert smo.SIGNMUON_POLAR_AFTER_ONLY == 1 << 8 and smo.SIGNMUON_MUON_MEAN == 1 << 9
    assert smo.SIGNMUON_TERNARY == 1 << 10 and smo.SIGNMUON_NORMALIZED_SIGN == 1 << 11
    with pytest.raises(smo.SignMuonError) as e:
        smo.SignMuon([(8, 8)], 2, flags=flags)
    assert e.value.status == smo.SIGNMUON_E_INVALID
    with pytest.raises(smo.SignMuonError) as e:
        smo.signmuon_plan([(8, 8)], 2, flags=flags)
    assert e.value.status == smo.SIGNMUON_E_INVALID


def test_plan_accepts_the_sign_wire_variants_and_counts_ternary_bytes():
    import sign_muon_optimizer_b200 as smo
    shapes = [(8, 24), (40, 16)]
    base = smo.signmuon_plan(shapes, 5, 5, "spectral", 2)
    for flags in (1 << 10, 1 << 11, (1 << 10) | (1 << 11), (1 << 10) | (1 << 2), (1 << 10) | (1 << 8) | (1 << 2)):
        p = smo.signmuon_plan(shapes, 5, 5, "spectral", 2, flags)
        # one int8 per entry and worker, at the library's 64-entry padded stride
        extra = 5 * ((p["d"] + 63) // 64 * 64) if flags & (1 << 10) else 0
        assert p["device_bytes"] == base["device_bytes"] + extra
    # the warm power-iteration state of one problem set: min(rows, cols) floats per matrix
    assert smo.SIGNMUON_PI_WARM == 1 << 12
    assert smo.SIGNMUON_NS_GRAM == 1 << 13
    p = smo.signmuon_plan(shapes, 5, 5, "spectral", 2, 1 << 12)
    assert p["device_bytes"] == base["device_bytes"] + 4 * (8 + 16)


_NULL_HANDLE_CALLS = """
import ctypes, sys
sys.path.insert(0, {root!r})
import sign_muon_optimizer_b200 as smo
L = smo._lib
pp = (ctypes.c_void_p * 1)()
calls = {{
    "signmuon_step": (None, None, pp, 0.1), "signmuon_step_host": (None, None, pp, 0.1),
    "signmuon_local_signs": (None, None, pp, None, 16), "signmuon_vote_step": (None, None, None, 16, 2, 0.1),
    "signmuon_sums_step": (None, None, None, 0.1), "signmuon_vote": (None, pp, 8, None, None),
    "signmuon_vote_ternary": (None, pp, 8, None, None), "signmuon_pack": (None, None, 8, None),
    "signmuon_sign_ternary": (None, None, 8, None), "signmuon_apply_update": (None, None, None, 8, 0.1),
    "signmuon_polar": (None, pp, pp), "signmuon_get_momentum": (None, 0, None),
    "signmuon_set_momentum": (None, 0, None), "signmuon_get_pi_state": (None, 0, None),
    "signmuon_set_pi_state": (None, 0, None), "signmuon_get_polar": (None, 0, None),
    "signmuon_get_signs": (None, 0, None), "signmuon_get_ternary_signs": (None, 0, None),
    "signmuon_get_direction": (None, None), "signmuon_get_scales": (None, None),
    "signmuon_set_ns_coeffs": (None, None, 2), "signmuon_sync": (None,), "signmuon_info": (None, None, 6),
    "signmuon_profile": (None, 1), "signmuon_profile_read": (None, None, None, 1),
    "signmuon_get_gram": (None, 0, 0, None), "signmuon_vote_step_ptrs": (None, None, pp, 2, 0.1),
}}
bad = []
for name, args in calls.items():
    rc = getattr(L, name)(*args)
    if rc != smo.SIGNMUON_E_INVALID or not L.signmuon_last_error(None):
        bad.append((name, rc))
# the handle-free IPC calls reject null pointers the same way
off = ctypes.c_int64()
for name, args in {{"signmuon_ipc_get_handle": (None, None, ctypes.byref(off)), "signmuon_ipc_open": (None, None),
                    "signmuon_ipc_close": (None,)}}.items():
    rc = getattr(L, name)(*args)
    if rc != smo.SIGNMUON_E_INVALID or not L.signmuon_last_error(None):
        bad.append((name, rc))
L.signmuon_destroy(None)
print("BAD", bad) if bad else print("ALL", len(calls))
"""


def test_every_entry_point_rejects_a_null_handle():
    # in a child process, so that a crash would fail this test, not the run
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, "-c", _NULL_HANDLE_CALLS.format(root=root)], capture_output=True,
                         text=True, timeout=120)
    assert res.returncode == 0, res.stderr[-2000:]
    assert res.stdout.strip().startswith("ALL"), res.stdout
    import sign_muon_optimizer_b200 as smo
    declared = [n for n in smo.EXPORTED if n not in (
        "signmuon_init", "signmuon_plan", "signmuon_plan_tables", "signmuon_kernel_launches",
        "signmuon_last_error", "signmuon_status_string", "signmuon_destroy", "signmuon_spectral_norm_noalloc",
        "signmuon_ipc_get_handle", "signmuon_ipc_open", "signmuon_ipc_close")]
    assert int(res.stdout.split()[1]) == len(declared)   # every handle-taking call is covered
