"""GPU parity of the individual stages, through the C ABI, against the oracle.

Bit-exact: one-bit pack, vote sums / majority (int32 and int8), the update.
Tolerance: the momentum pass (fp32 against float64) and PolarNS (2e-2 bf16,
1e-4 fp32 max abs; <= 1e-3 sign disagreements above the 1e-3 mask).
"""
import json
import os

import numpy as np
import pytest

import synth
from oracle import signmuon_ref as ref

from gpu_helpers import assert_momentum_close, assert_polar_close, dev, host, oracle_polar_flat

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import sign_muon_optimizer_b200 as smo  # noqa: E402


def _vote_handle(M, acc8=False):
    flags = smo.SIGNMUON_VOTE_ONLY | (smo.SIGNMUON_ACC_INT8 if acc8 else 0)
    return smo.SignMuon([(1, 1)], M, flags=flags)


@pytest.mark.parametrize("d", [1, 7, 31, 33, 1000, 1024, 1025, 5 * 1024 + 17, 100003])
def test_pack_bit_exact(d):
    u = synth.uniform_values(d, config_id=11, step=d)
    if d > 40:
        u[5] = np.nan
        u[6] = np.float32(-0.0)
        u[7] = np.float32(0.0)
    h = _vote_handle(1)
    U = dev(u)
    out = torch.zeros((d + 7) // 8 + 16, dtype=torch.uint8, device="cuda")
    h.pack(U, d, out)
    got = host(out)
    want = ref.pack_bits(ref.sign_bits(u))
    assert np.array_equal(got[: want.size], want)
    assert not got[want.size:].any()  # nothing written past ceil(d/8)


def test_vote_blog_worked_example():
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "blog_worked_example.json")))
    dirs = np.array(g["directions"], np.float32)
    h = _vote_handle(3)
    signs = [dev(ref.pack_bits(ref.sign_bits(x.ravel()))) for x in dirs]
    signs = [torch.nn.functional.pad(s, (0, 15)) for s in signs]  # 16-byte aligned copies
    sums = torch.zeros(4, dtype=torch.int32, device="cuda")
    maj = torch.zeros(16, dtype=torch.int8, device="cuda")
    h.vote(signs, 4, sums, maj)
    assert host(sums).reshape(2, 2).tolist() == g["sums"]
    assert host(maj)[:4].reshape(2, 2).tolist() == g["majority"]


@pytest.mark.parametrize("M", [1, 2, 3, 16, 127, 200, 256])
@pytest.mark.parametrize("d", [1, 7, 1024, 5000, 8192, 40 * 1024 + 3])
def test_vote_bit_exact(M, d):
    # d = 8192: whole 4096-entry tiles only; 5000 and 40963: tiles plus a
    # ragged rest; M = 256: above the byte-lane counters' range (all entries
    # on the register kernel)
    bits = synth.bernoulli_bits(d, M, config_id=M * 1000 + d % 997)
    packed = [ref.pack_bits(b) for b in bits]
    want_sums = ref.vote_sums_from_bits(packed, d, "int32")
    want_maj = ref.majority(want_sums)
    nb = (d + 7) // 8
    signs = [dev(np.concatenate([p, np.zeros(16, np.uint8)])) for p in packed]
    h = _vote_handle(M)
    sums = torch.zeros(d, dtype=torch.int32, device="cuda")
    maj = torch.zeros(d, dtype=torch.int8, device="cuda")
    h.vote(signs, d, sums, maj)
    assert np.array_equal(host(sums), want_sums)
    assert np.array_equal(host(maj), want_maj)
    if M <= 127:
        h8 = _vote_handle(M, acc8=True)
        sums8 = torch.zeros(d, dtype=torch.int8, device="cuda")
        h8.vote(signs, d, sums8, None)
        assert np.array_equal(host(sums8), ref.vote_sums_from_bits(packed, d, "int8"))
    assert nb == ref.packed_nbytes(d)


def test_int8_guard_rejects_large_M():
    with pytest.raises(smo.SignMuonError) as e:
        _vote_handle(128, acc8=True)
    assert e.value.status == smo.SIGNMUON_E_OVERFLOW


@pytest.mark.parametrize("kind", ["ternary", "real"])
@pytest.mark.parametrize("d", [1, 5, 4096, 100003])
def test_update_bit_exact(kind, d):
    w = synth.weights0([(1, d)], config_id=d)
    if kind == "ternary":
        D = synth.ternary_direction(d, config_id=d)
    else:
        D = synth.uniform_values(d, config_id=d, step=3)
    eta = np.float32(0.02)
    h = _vote_handle(1)
    W = dev(w)
    h.apply_update(W, dev(D), d, eta)
    want = ref.update(w, D, eta)
    assert np.array_equal(host(W).view(np.uint32), want.view(np.uint32))


SHAPES_SMALL = [(3, 5), (5, 3), (130, 70), (64, 147), (200, 200), (96, 300)]


def _polar_case(shapes, M, K, scale, P, precision, order, seed, coeffs=None, extra=0, want_gram_ns=None):
    flags = (smo.SIGNMUON_NS_FP32 if precision == "fp32" else 0) | (smo.SIGNMUON_NS_QUINTIC if order == "quintic" else 0)
    flags |= extra
    if want_gram_ns is not None:
        assert smo.signmuon_plan_tables(shapes, M, K, scale, P, flags)["gram_ns"] == want_gram_ns
    h = smo.SignMuon(shapes, M, beta=0.9, lam=0.0, K=K, eps=1e-7, scale=scale, P=P, flags=flags)
    if coeffs is not None:
        h.set_ns_coeffs(coeffs)
    xs = synth.gaussian_matrices(shapes, M, config_id=seed)
    X = [dev(x) for x in xs]
    U = [torch.zeros_like(x) for x in X]
    h.polar(X, U)
    worst = 0.0
    for m in range(M):
        want = oracle_polar_flat(xs[m].astype(np.float64), shapes, K, 1e-7, scale, P, order, coeffs)
        err, _, _ = assert_polar_close(host(U[m]), want, precision, f"worker {m}")
        worst = max(worst, err)
    return worst


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
@pytest.mark.parametrize("scale,P", [("fro", 1), ("spectral", 2)])
@pytest.mark.parametrize("K", [0, 1, 5])
def test_polar_cubic(precision, scale, P, K):
    _polar_case(SHAPES_SMALL, 2, K, scale, P, precision, "cubic", seed=100 + K)


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_polar_quintic(precision):
    _polar_case(SHAPES_SMALL, 2, 5, "spectral", 2, precision, "quintic", seed=7)


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
@pytest.mark.parametrize("order,coeffs", [("cubic", (1.75, -0.75)), ("quintic", (2.0, -1.5, 0.5))])
def test_polar_custom_coefficients(precision, order, coeffs):
    """signmuon_set_ns_coeffs: generic two- and three-coefficient iterations
    against the oracle run with the same coefficients (both converge to the
    polar factor: p(1) = 1 for each)."""
    _polar_case(SHAPES_SMALL, 2, 4, "fro", 1, precision, order, seed=11, coeffs=coeffs)


@pytest.mark.parametrize("gram", [True, False])
@pytest.mark.parametrize("K", [2, 3, 5])
@pytest.mark.parametrize("scale,P", [("fro", 1), ("spectral", 2)])
def test_polar_gram_space(gram, K, scale, P):
    """bf16 cubic PolarNS in Gram space (SIGNMUON_NS_GRAM, taken for matrices
    with n well above m) and, by default, on X: both against the oracle's
    iteration on X, on multi-tile Grams with ragged edges (m = 300, 768, 520)
    in both orientations."""
    shapes = [(300, 1000), (3072, 768), (520, 1600)]
    _polar_case(shapes, 2, K, scale, P, "bf16", "cubic", seed=300 + K,
                extra=smo.SIGNMUON_NS_GRAM if gram else 0, want_gram_ns=1 if gram else 0)


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_polar_large_tiles(precision):
    # several 128x256 tiles per problem, ragged edges, both orientations
    _polar_case([(768, 2304), (2304, 768), (520, 600)], 2, 5, "spectral", 2, precision, "cubic", seed=21)


def test_momentum_pass():
    shapes = [(256, 128), (3, 5), (64, 147)]
    M = 3
    h = smo.SignMuon(shapes, M, beta=0.9, lam=0.01, K=1, eps=1e-7, scale="fro", flags=smo.SIGNMUON_NS_FP32)
    d = h.d
    w = synth.weights0(shapes, 1)
    mom0 = synth.momentum0(shapes, M, 1)
    for m in range(M):
        h.set_momentum(m, dev(mom0[m]))
    G = synth.gradients(shapes, M, 0.5, step=1, config_id=1)
    h.step(dev(w), [dev(g) for g in G], 0.02)
    for m in range(M):
        got = torch.zeros(d, device="cuda")
        h.get_momentum(m, got)
        assert_momentum_close(host(got), mom0[m], G[m], w, 0.9, 0.01)


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
@pytest.mark.parametrize("shapes", [[(200, 200), (130, 70)], [(600, 900)], [(768, 2304), (300, 64)]])
def test_gram_matches_bf16_product(precision, shapes):
    """The first Newton-Schulz GEMM's output (the Gram of the staged input,
    wide orientation) against numpy on the same staged values: bf16-rounded
    inputs with exact products, fp32-accumulated, then rounded to bf16 (or
    kept fp32).  Covers multi-tile Grams, the mirrored upper-triangle tiles
    and ragged edges of every 64x64 block."""
    flags = smo.SIGNMUON_NS_FP32 if precision == "fp32" else 0
    M = 2
    h = smo.SignMuon(shapes, M, beta=0.9, lam=0.0, K=1, eps=1e-7, scale="fro", flags=flags)
    xs = synth.gaussian_matrices(shapes, M, config_id=77)
    X = [dev(x) for x in xs]
    U = [torch.zeros_like(x) for x in X]
    h.polar(X, U)
    for m in range(M):
        off = 0
        for i, (r, c) in enumerate(shapes):
            mat = xs[m][off: off + r * c].reshape(r, c)
            off += r * c
            if precision == "bf16":
                mat = torch.from_numpy(mat).bfloat16().double().numpy()
            wide = mat.astype(np.float64) if r <= c else mat.astype(np.float64).T
            want = wide @ wide.T
            got = h.get_gram(m, i).astype(np.float64)
            tol = (2.0 ** -7 if precision == "bf16" else 1e-5) * np.abs(want).max()
            bad = np.abs(got - want) > tol
            assert not bad.any(), f"{r}x{c} worker {m}: {bad.sum()} Gram entries off, rows {np.nonzero(bad)[0][:5]}"


@pytest.mark.parametrize("M", [2, 4, 16])
@pytest.mark.parametrize("d", [5000, 8192])
def test_vote_tie_plus_bit_exact(M, d):
    """Named variant: a tie gives +1 ([paper] Algorithm 2's default)."""
    bits = synth.bernoulli_bits(d, M, config_id=7000 + M + d % 97)
    packed = [ref.pack_bits(b) for b in bits]
    want_sums = ref.vote_sums_from_bits(packed, d, "int32")
    assert (want_sums == 0).any()
    signs = [dev(np.concatenate([p, np.zeros(16, np.uint8)])) for p in packed]
    h = smo.SignMuon([(1, d)], M, flags=smo.SIGNMUON_VOTE_ONLY | smo.SIGNMUON_TIE_PLUS)
    sums = torch.zeros(d, dtype=torch.int32, device="cuda")
    maj = torch.zeros(d, dtype=torch.int8, device="cuda")
    h.vote(signs, d, sums, maj)
    assert np.array_equal(host(sums), want_sums)
    assert np.array_equal(host(maj), ref.majority(want_sums, tie=1))


def test_empty_calls_write_nothing():
    """d = 0: vote, pack and update return at once and leave their outputs."""
    h = _vote_handle(3)
    signs = [torch.zeros(16, dtype=torch.uint8, device="cuda") for _ in range(3)]
    sums = torch.full((4,), 7, dtype=torch.int32, device="cuda")
    maj = torch.full((16,), 5, dtype=torch.int8, device="cuda")
    h.vote(signs, 0, sums, maj)
    assert host(sums).tolist() == [7] * 4 and (host(maj) == 5).all()
    U = torch.ones(4, device="cuda")
    out = torch.full((16,), 9, dtype=torch.uint8, device="cuda")
    h.pack(U, 0, out)
    assert (host(out) == 9).all()
    W = torch.full((4,), 2.0, device="cuda")
    h.apply_update(W, torch.ones(4, device="cuda"), 0, 0.5)
    assert (host(W) == 2.0).all()
