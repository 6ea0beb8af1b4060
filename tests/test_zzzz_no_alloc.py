"""signmuon_spectral_norm_noalloc: the allocation-free spectral-norm call.

It exists for callers that cannot allocate device memory (code under CUDA
graph capture, frameworks that own all device memory, real-time paths).  Its
result must equal, within the fp32 tolerance of the other parity tests, the
spectral scale that the regular entry points compute for the same matrix
(signmuon_polar with SIGNMUON_NS_FP32 and spectral scaling, read back with
signmuon_get_scales), and the oracle's power iteration in float64.  The size
limit is checked on both sides of the bound.  This file is collected last on
purpose.
"""
import numpy as np
import pytest

import synth
from oracle import signmuon_ref as ref

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import sign_muon_optimizer_b200 as smo  # noqa: E402

REL_TOL = 1e-4  # the fp32 tolerance of the polar-factor parity tests


def _existing_sigma(shape, x, P):
    h = smo.SignMuon([shape], 1, beta=0.9, lam=0.0, K=0, eps=1e-7, scale="spectral", P=P,
                     flags=smo.SIGNMUON_NS_FP32)
    X = torch.from_numpy(x).cuda()
    U = torch.zeros_like(X)
    h.polar([X], [U])
    s = float(h.get_scales()[0, 0])
    h.close()
    return s


@pytest.mark.parametrize("P", [1, 2, 5])
def test_noalloc_matches_existing_entry_point_two_calls_in_a_row(P):
    shapes = [(130, 70), (96, 300)]
    xs = [synth.gaussian_matrices([s], 1, config_id=900 + i)[0] for i, s in enumerate(shapes)]
    sig = torch.zeros(4, device="cuda")
    got = []
    for (r, c), x in zip(shapes, xs):  # two calls in a row, same static scratch
        smo.signmuon_spectral_norm_noalloc(torch.from_numpy(x).cuda(), r, c, P, sig)
        torch.cuda.synchronize()
        got.append(float(sig[0].item()))
    for (r, c), x, g in zip(shapes, xs, got):
        want = _existing_sigma((r, c), x, P)
        assert abs(g - want) <= REL_TOL * want, f"{r}x{c} P={P}: {g} vs {want}"
        # the same estimate in float64 by the oracle (wide orientation)
        xw = x.reshape(r, c).astype(np.float64)
        exact = ref.power_sigma(xw if r <= c else xw.T, P)
        assert abs(g - exact) <= REL_TOL * exact, f"{r}x{c} P={P}: {g} vs oracle {exact}"


def test_noalloc_allocates_nothing_after_setup():
    r, c = 512, 700
    x = torch.randn(r * c, device="cuda")
    sig = torch.zeros(4, device="cuda")
    smo.signmuon_spectral_norm_noalloc(x, r, c, 2, sig)  # first call: one-time set-up
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(5):
        smo.signmuon_spectral_norm_noalloc(x, r, c, 2, sig)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert np.isfinite(float(sig[0].item())) and float(sig[0].item()) > 0


def test_noalloc_rejects_sizes_beyond_the_scratch():
    x = torch.zeros(16, device="cuda")
    sig = torch.zeros(4, device="cuda")
    with pytest.raises(smo.SignMuonError) as e:
        smo.signmuon_spectral_norm_noalloc(x, 400_000, 400_000, 2, sig)
    assert e.value.status == smo.SIGNMUON_E_INVALID
    assert "static scratch" in smo.signmuon_last_error(None)


@pytest.mark.parametrize("rows,cols,P", [(1, 1048574, 2), (1048574, 1, 1)])
def test_noalloc_accepts_the_largest_size(rows, cols, P):
    """max(rows, cols) + 2 * min(rows, cols) equal to the scratch's 1,048,576
    floats is accepted, in both orientations.  A single row or column has one
    singular value, its 2-norm, which every power iteration returns."""
    n = rows * cols
    x = torch.randn(n, device="cuda", generator=torch.Generator(device="cuda").manual_seed(77))
    sig = torch.zeros(4, device="cuda")
    smo.signmuon_spectral_norm_noalloc(x, rows, cols, P, sig)
    torch.cuda.synchronize()
    got = float(sig[0].item())
    want = float(np.linalg.norm(x.double().cpu().numpy()))
    assert abs(got - want) <= REL_TOL * want, f"{rows}x{cols}: {got} vs {want}"


@pytest.mark.parametrize("rows,cols", [(1, 1048575), (1048575, 1), (349527, 349525)])
def test_noalloc_rejects_one_past_the_largest_size(rows, cols):
    x = torch.zeros(16, device="cuda")
    sig = torch.full((4,), -1.0, device="cuda")
    with pytest.raises(smo.SignMuonError) as e:
        smo.signmuon_spectral_norm_noalloc(x, rows, cols, 1, sig)
    assert e.value.status == smo.SIGNMUON_E_INVALID
    torch.cuda.synchronize()
    assert float(sig[0].item()) == -1.0  # nothing was launched
