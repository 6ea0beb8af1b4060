"""Shared helpers of the GPU parity tests (imported only by tests marked gpu)."""
import numpy as np

from oracle import signmuon_ref as ref

# Tolerances of the parity bar: polar factor max-abs error per precision, and
# the allowed fraction of sign disagreements among entries whose magnitude is
# above 1e-3 of the largest |U|.
POLAR_TOL = {"bf16": 2e-2, "fp32": 1e-4}
SIGN_FRAC = 1e-3
SIGN_MASK = 1e-3


def dev(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def host(t):
    import torch
    torch.cuda.synchronize()
    return t.detach().cpu().numpy()


def oracle_polar_flat(flat, shapes, K, eps, scale, P, order="cubic", coeffs=None):
    out = np.empty(flat.size, np.float64)
    off = 0
    for r, c in shapes:
        out[off: off + r * c] = ref.polar_ns(flat[off: off + r * c].reshape(r, c), K, eps, scale, P, order,
                                             coeffs).ravel()
        off += r * c
    return out


def sign_disagreement(u_gpu, u_ref):
    """(disagreements, counted entries) over entries with |u_ref| above the mask."""
    u_gpu = np.asarray(u_gpu, np.float64)
    u_ref = np.asarray(u_ref, np.float64)
    thr = SIGN_MASK * np.max(np.abs(u_ref)) if u_ref.size else 0.0
    mask = np.abs(u_ref) > thr
    dis = (ref.sign_bits(u_gpu) != ref.sign_bits(u_ref)) & mask
    return int(dis.sum()), int(mask.sum())


def assert_polar_close(u_gpu, u_ref, precision, what=""):
    err = float(np.max(np.abs(np.asarray(u_gpu, np.float64) - u_ref))) if u_ref.size else 0.0
    assert err <= POLAR_TOL[precision], f"{what}: polar max abs error {err:.3e} > {POLAR_TOL[precision]}"
    n_dis, n = sign_disagreement(u_gpu, u_ref)
    assert n_dis <= SIGN_FRAC * n, f"{what}: {n_dis} sign disagreements of {n} entries"
    return err, n_dis, n


def assert_momentum_close(got, mom0, g, w, beta, lam):
    """fp32 momentum against float64: at most a few fp32 roundings of the
    terms beta*|Mom|, (1-beta)*|G|, (1-beta)*lambda*|W| (unit roundoff 2^-24)."""
    mom0 = np.asarray(mom0, np.float64)
    g = np.asarray(g, np.float64)
    w = np.asarray(w, np.float64)
    want = ref.momentum_update(mom0, g, w, beta, lam)
    scale = beta * np.abs(mom0) + (1 - beta) * (np.abs(g) + lam * np.abs(w)) + np.abs(want)
    err = np.abs(np.asarray(got, np.float64) - want)
    bad = err > 4 * 2.0 ** -24 * scale + 1e-30
    assert not bad.any(), f"{bad.sum()} momentum entries off; worst {err[bad].max():.3e}"
