"""Pins for the CPU oracle against what the pages and plain mathematics fix.

Each test checks the oracle against something other than itself: a worked
example printed on a page, a closed form, a textbook/library routine
(LAPACK SVD, numpy.packbits), exact rational arithmetic or brute force.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import synth
from oracle import signmuon_ref as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# vote, tie policy, payload
# ---------------------------------------------------------------------------

def test_blog_worked_example_ternary():
    g = _golden("blog_worked_example.json")
    dirs = np.array(g["directions"])
    signs = [ref.sign_ternary(x) for x in dirs]
    sums = ref.vote_sums_ternary(signs)
    assert sums.dtype == np.int32
    assert sums.tolist() == g["sums"]
    assert ref.majority(sums).tolist() == g["majority"]


def test_blog_worked_example_one_bit_path():
    # no direction entry is zero, so the 1-bit path must give the same vote
    g = _golden("blog_worked_example.json")
    dirs = np.array(g["directions"])
    packed = [ref.pack_bits(ref.sign_bits(x.ravel())) for x in dirs]
    assert all(p.size == 1 for p in packed)  # ceil(4/8) bytes
    sums = ref.vote_sums_from_bits(packed, 4)
    assert sums.reshape(2, 2).tolist() == g["sums"]
    assert ref.majority(sums).reshape(2, 2).tolist() == g["majority"]


def test_blog_mean_versus_majority():
    g = _golden("blog_mean_vs_majority.json")
    x = np.array(g["directions"])
    assert int(np.sign(x.mean())) == g["mean_sign"]
    sums = ref.vote_sums_ternary([ref.sign_ternary(v) for v in x])
    assert int(ref.majority(sums)) == g["majority"]


@pytest.mark.parametrize("votes", [[1, -1], [1, 1, -1, -1], [-1, 1, 1, -1, 1, -1]])
def test_ties_map_to_zero(votes):
    packed = [ref.pack_bits(np.array([v > 0])) for v in votes]
    sums = ref.vote_sums_from_bits(packed, 1)
    assert int(sums[0]) == 0 and int(ref.majority(sums)[0]) == 0


@pytest.mark.parametrize("M", list(range(1, 11)))
def test_vote_brute_force_all_patterns(M):
    # every one of the 2^M bit patterns is one entry; count by hand
    patterns = list(itertools.product([0, 1], repeat=M))
    d = len(patterns)
    bits = np.array(patterns, bool).T  # (M, d)
    packed = [ref.pack_bits(bits[m]) for m in range(M)]
    sums = ref.vote_sums_from_bits(packed, d)
    maj = ref.majority(sums)
    for i, pat in enumerate(patterns):
        plus = sum(pat)
        minus = M - plus
        want = plus - minus
        assert int(sums[i]) == want
        assert -M <= int(sums[i]) <= M
        assert (int(sums[i]) - M) % 2 == 0
        assert int(maj[i]) == (1 if plus > minus else (-1 if minus > plus else 0))


def test_int8_accumulator_matches_int32_and_guards_overflow():
    rs = np.random.default_rng(0)
    for M in (1, 2, 16, 127):
        bits = rs.random((M, 1000)) < 0.5
        packed = [ref.pack_bits(b) for b in bits]
        s32 = ref.vote_sums_from_bits(packed, 1000, "int32")
        s8 = ref.vote_sums_from_bits(packed, 1000, "int8")
        assert s8.dtype == np.int8
        assert np.array_equal(s32.astype(np.int64), s8.astype(np.int64))
    bits = rs.random((128, 10)) < 0.5
    with pytest.raises(ref.AccumulatorOverflow):
        ref.vote_sums_from_bits([ref.pack_bits(b) for b in bits], 10, "int8")
    # all 128 workers agreeing would need +128, which int8 cannot hold
    assert np.iinfo(np.int8).max < 128


@pytest.mark.parametrize("d", [1, 7, 8, 9, 31, 32, 33, 100, 4096, 4099])
def test_pack_layout_against_numpy_packbits(d):
    rs = np.random.default_rng(d)
    bits = rs.random(d) < 0.5
    p = ref.pack_bits(bits)
    assert p.dtype == np.uint8 and p.size == (d + 7) // 8 == ref.packed_nbytes(d)
    assert np.array_equal(p, np.packbits(bits, bitorder="little"))
    # pad bits are zero
    if d % 8:
        assert int(p[-1]) >> (d % 8) == 0
    assert np.array_equal(ref.unpack_bits(p, d), bits)
    # bit j of byte b is element 8b+j
    for e in rs.integers(0, d, size=min(d, 20)):
        assert ((int(p[e // 8]) >> (e % 8)) & 1) == int(bits[e])


def test_payload_sizes_for_the_pages_ratios():
    d = 1_000_003
    assert ref.packed_nbytes(d) * 8 >= d > (ref.packed_nbytes(d) - 1) * 8
    # fp32 4d bytes vs packed ~d/8: the 32x ratio of the paper's abstract
    assert abs(4 * d / ref.packed_nbytes(d) - 32) < 1e-3


def test_one_bit_sign_of_zero_and_ternary_sign():
    u = np.array([0.0, -0.0, 1e-30, -1e-30, 2.0, -3.0], np.float32)
    assert ref.sign_bits(u).tolist() == [True, True, True, False, True, False]
    assert ref.sign_ternary(u).tolist() == [0, 0, 1, -1, 1, -1]


# ---------------------------------------------------------------------------
# Newton-Schulz: closed forms and convergence
# ---------------------------------------------------------------------------

def _orthonormal(rs, n, k):
    q, _ = np.linalg.qr(rs.standard_normal((n, k)))
    return q


def _svd_built(rs, rows, cols, svals):
    k = min(rows, cols)
    q1 = _orthonormal(rs, rows, k)
    q2 = _orthonormal(rs, cols, k)
    return q1 @ np.diag(svals) @ q2.T, q1, q2


def _f_cubic(s, K, a=1.5, b=-0.5):
    for _ in range(K):
        s = a * s + b * s ** 3
    return s


def _f_quintic(s, K):
    for _ in range(K):
        s = s * (15 / 8 - 10 / 8 * s ** 2 + 3 / 8 * s ** 4)
    return s


@pytest.mark.parametrize("rows,cols", [(6, 9), (9, 6), (7, 7), (3, 20), (20, 3)])
@pytest.mark.parametrize("K", [0, 1, 5, 10])
def test_ns_iterate_closed_form_cubic(rows, cols, K):
    rs = np.random.default_rng(rows * 100 + cols + K)
    k = min(rows, cols)
    s = rs.uniform(0.05, 1.2, size=k)
    x0, q1, q2 = _svd_built(rs, rows, cols, s)
    wide = x0 if rows <= cols else x0.T
    out = ref.ns_iterate(wide, K)
    if rows > cols:
        out = out.T
    want = q1 @ np.diag(_f_cubic(s, K)) @ q2.T
    assert np.max(np.abs(out - want)) < 1e-12


@pytest.mark.parametrize("rows,cols", [(5, 8), (8, 5)])
@pytest.mark.parametrize("K", [1, 3, 5])
def test_ns_iterate_closed_form_quintic_and_generic(rows, cols, K):
    rs = np.random.default_rng(7 + K)
    k = min(rows, cols)
    s = rs.uniform(0.05, 1.0, size=k)
    x0, q1, q2 = _svd_built(rs, rows, cols, s)
    wide = x0 if rows <= cols else x0.T
    out = ref.ns_iterate(wide, K, "quintic")
    out = out.T if rows > cols else out
    assert np.max(np.abs(out - q1 @ np.diag(_f_quintic(s, K)) @ q2.T)) < 1e-12
    out = ref.ns_iterate(wide, K, "cubic", coeffs=(2.0, -1.25))
    out = out.T if rows > cols else out
    assert np.max(np.abs(out - q1 @ np.diag(_f_cubic(s, K, 2.0, -1.25)) @ q2.T)) < 1e-12


@pytest.mark.parametrize("rows,cols", [(4, 6), (6, 4), (8, 8), (2, 5)])
def test_polar_fro_closed_form(rows, cols):
    rs = np.random.default_rng(rows + 10 * cols)
    k = min(rows, cols)
    s = rs.uniform(0.5, 3.0, size=k)
    mat, q1, q2 = _svd_built(rs, rows, cols, s)
    eps = 1e-7
    fro = math.sqrt(float(np.sum(s ** 2)))
    out = ref.polar_ns(mat, 5, eps, "fro")
    want = q1 @ np.diag(_f_cubic(s / (fro + eps), 5)) @ q2.T
    assert np.max(np.abs(out - want)) < 1e-12


@pytest.mark.parametrize("rows,cols", [(4, 6), (6, 4), (5, 5)])
@pytest.mark.parametrize("P", [1, 2, 3])
def test_polar_spectral_closed_form(rows, cols, P):
    # power iteration on X X^T from u0 = ones/sqrt(m): in the left singular
    # basis the iterate is diag(s^(2P)) a with a = Q1^T u0, so
    # sigma^2 = sum a_i^2 s_i^(4P+2) / sum a_i^2 s_i^(4P)
    rs = np.random.default_rng(3 * rows + cols + P)
    k = min(rows, cols)
    s = rs.uniform(0.5, 3.0, size=k)
    mat, q1, q2 = _svd_built(rs, rows, cols, s)
    left = q1 if rows <= cols else q2
    m = min(rows, cols)
    a = left.T @ np.full(m, 1 / math.sqrt(m))
    sig = math.sqrt(np.sum(a ** 2 * s ** (4 * P + 2)) / np.sum(a ** 2 * s ** (4 * P)))
    eps = 1e-7
    out, got_s = ref.polar_ns(mat, 5, eps, "spectral", P, return_scale=True)
    assert abs(got_s - sig) < 1e-12 * sig
    want = q1 @ np.diag(_f_cubic(s / (sig + eps), 5)) @ q2.T
    assert np.max(np.abs(out - want)) < 1e-11


@pytest.mark.parametrize("rows,cols", [(3, 3), (4, 7), (7, 4), (8, 8), (2, 6)])
def test_cubic_ns_converges_to_svd_polar_factor(rows, cols):
    rs = np.random.default_rng(11 * rows + cols)
    k = min(rows, cols)
    mat, _, _ = _svd_built(rs, rows, cols, rs.uniform(0.6, 1.0, size=k))
    mat = mat * 3.7
    u, _, vt = np.linalg.svd(mat, full_matrices=False)  # LAPACK
    polar = u @ vt
    out = ref.polar_ns(mat, 40, 1e-12, "fro")
    assert np.max(np.abs(out - polar)) < 1e-10
    out = ref.polar_ns(mat, 40, 1e-12, "spectral", 4)
    assert np.max(np.abs(out - polar)) < 1e-10
    out = ref.polar_ns(mat, 30, 1e-12, "fro", order="quintic")
    assert np.max(np.abs(out - polar)) < 1e-10


def test_orthogonal_input_is_a_fixed_point_under_spectral_scaling():
    rs = np.random.default_rng(5)
    q = _orthonormal(rs, 6, 6)
    out = ref.polar_ns(q, 5, 0.0, "spectral", 3)
    assert np.max(np.abs(out - q)) < 1e-12


def test_power_iteration_against_exact_sigma_max():
    rs = np.random.default_rng(9)
    for rows, cols in [(5, 9), (9, 5), (6, 6)]:
        mat = rs.standard_normal((rows, cols))
        smax = np.linalg.svd(mat, compute_uv=False)[0]
        wide = mat if rows <= cols else mat.T
        est = [ref.power_sigma(wide, P) for P in (1, 2, 5, 200)]
        assert all(e <= smax * (1 + 1e-12) for e in est)
        assert est[0] <= est[1] * (1 + 1e-12) and est[1] <= est[2] * (1 + 1e-12)
        assert abs(est[-1] - smax) < 1e-9 * smax


def test_power_iteration_rank_one_and_zero():
    rs = np.random.default_rng(2)
    u = rs.standard_normal(4)
    v = rs.standard_normal(7)
    mat = 3.0 * np.outer(u / np.linalg.norm(u), v / np.linalg.norm(v))
    assert abs(ref.power_sigma(mat, 1) - 3.0) < 1e-12
    assert ref.power_sigma(np.zeros((3, 5)), 2) == 0.0
    # zero matrix: scale 0, X0 = 0, NS keeps 0, the 1-bit sign sends +1
    out = ref.polar_ns(np.zeros((3, 5)), 5, 1e-7, "spectral", 2)
    assert np.all(out == 0) and np.all(ref.sign_bits(out))


# ---------------------------------------------------------------------------
# momentum and update
# ---------------------------------------------------------------------------

def test_momentum_closed_form_constant_gradient():
    rs = np.random.default_rng(4)
    g = rs.standard_normal(50)
    w = rs.standard_normal(50)
    beta, lam = 0.9, 0.01
    mom = np.zeros(50)
    for t in range(1, 8):
        mom = ref.momentum_update(mom, g, w, beta, lam)
        assert np.max(np.abs(mom - (1 - beta ** t) * (g + lam * w))) < 1e-14
    assert np.array_equal(ref.momentum_update(np.ones(50), g, w, 0.0, lam), g + lam * w)


def _exact_round_f32(w, eta, dd):
    # exact rational value rounded to the nearest float32, ties to even
    v = Fraction(float(w)) - Fraction(float(eta)) * Fraction(float(dd))
    f = np.float32(float(v))  # candidate; fix up by comparing neighbours exactly
    best = None
    for c in (np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))):
        err = abs(Fraction(float(c)) - v)
        key = (err, int(np.frombuffer(np.float32(c).tobytes(), np.uint32)[0]) & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return np.float32(best[1])


def test_update_single_rounding_against_exact_rationals():
    rs = np.random.default_rng(6)
    n = 3000
    w = (0.02 * rs.standard_normal(n)).astype(np.float32)
    w[:50] = (rs.standard_normal(50) * 1e6).astype(np.float32)    # large exponent gaps
    w[50:100] = (rs.standard_normal(50) * 1e-12).astype(np.float32)
    w[100] = np.float32(0.0)
    eta = np.float32(0.02)
    d_tern = rs.choice([-1.0, 0.0, 1.0], size=n).astype(np.float32)
    d_real = rs.standard_normal(n).astype(np.float32)
    for dd in (d_tern, d_real):
        got = ref.update(w, dd, eta)
        assert got.dtype == np.float32
        want = np.array([_exact_round_f32(w[i], eta, dd[i]) for i in range(n)], np.float32)
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_update_midpoint_cases():
    # w - eta*d is 1 + 2^-24 + 2^-64: float64 rounds it onto the float32
    # midpoint 1 + 2^-24, where ties-to-even would give 1.0; the exact value
    # lies above the midpoint, so one correct rounding gives 1 + 2^-23
    w = np.array([1.0 + 2.0 ** -23], np.float32)
    eta = np.float32(2.0 ** -24 * (1.0 + 2.0 ** -20))
    dd = np.array([1.0 - 2.0 ** -20], np.float32)
    naive = np.float32(np.float64(w[0]) - np.float64(eta) * np.float64(dd[0]))
    want = _exact_round_f32(w[0], eta, dd[0])
    assert want == np.float32(1.0 + 2.0 ** -23) and naive != want  # the case discriminates
    assert ref.update(w, dd, eta)[0] == want
    # mirrored: below the midpoint by 2^-64 -> rounds down
    w = np.array([1.0], np.float32)
    eta = np.float32(2.0 ** -24 * (1.0 + 2.0 ** -20))
    dd = np.array([-(1.0 - 2.0 ** -20)], np.float32)
    assert ref.update(w, dd, eta)[0] == _exact_round_f32(w[0], eta, dd[0])
    # exact midpoints (err = 0) keep ties-to-even
    w = np.array([1.0, 1.0, 1.0 + 2 ** -23], np.float32)
    eta = np.float32(2 ** -24)
    dd = np.array([-1.0, 1.0, -1.0], np.float32)
    got = ref.update(w, dd, eta)
    want = np.array([_exact_round_f32(w[i], eta, dd[i]) for i in range(3)], np.float32)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


# ---------------------------------------------------------------------------
# the composed step
# ---------------------------------------------------------------------------

def test_step_reduces_to_the_blog_vote_when_polar_is_off():
    # beta=0, lambda=0, K=0: U_m = G_m/(s+eps), so sign(U_m) = sign(G_m) and
    # the step must move W by -eta * (the page's majority)
    g = _golden("blog_worked_example.json")
    dirs = np.array(g["directions"])
    W = np.array([0.5, -0.25, 0.125, 1.0], np.float32)
    out = ref.step(W, [x.ravel() for x in dirs], [np.zeros(4)] * 3, [(2, 2)],
                   beta=0.0, lam=0.0, eta=0.02, K=0, eps=1e-7, scale="fro")
    assert out["majority"].reshape(2, 2).tolist() == g["majority"]
    assert out["sums"].reshape(2, 2).tolist() == g["sums"]
    want = np.array([np.float32(float(W[i]) - float(np.float32(0.02)) * g["majority"][i // 2][i % 2])
                     for i in range(4)], np.float32)
    assert np.array_equal(out["W"], want)


def test_step_polar_of_orthogonal_gradients_and_post_polar():
    # every worker sees the same gradient sqrt(2)*H with H orthogonal, so
    # U_m = H*f^K(sqrt(2)/(2+eps)*...) and the majority is sign(H); the
    # post-vote polar of the +-1 matrix [[1,1],[1,-1]] = sqrt(2)*H' is
    # H' * f^K(sqrt(2)/(2+eps))
    H = np.array([[1.0, 1.0], [1.0, -1.0]]) / math.sqrt(2)
    G = (math.sqrt(2) * H).ravel()
    W = np.zeros(4, np.float32)
    eps = 1e-7
    out = ref.step(W, [G, G, G], [np.zeros(4)] * 3, [(2, 2)], beta=0.0, lam=0.0, eta=0.5,
                   K=3, eps=eps, scale="fro", post_polar=True)
    s1 = _f_cubic(np.array([math.sqrt(2) / (2 + eps)]), 3)[0]
    assert np.max(np.abs(out["U"][0].reshape(2, 2) - H * s1)) < 1e-14
    assert out["majority"].reshape(2, 2).tolist() == [[1, 1], [1, -1]]
    assert np.max(np.abs(out["D"].reshape(2, 2) - H * s1)) < 1e-14
    assert np.array_equal(out["W"], ref.update(W, out["D32"], 0.5))


# ---------------------------------------------------------------------------
# named variants ([paper] Algorithm 2's tie default, after-only polar, Muon)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 6, 7, 8])
def test_tie_plus_brute_force_all_patterns(M):
    # every pattern of M one-bit votes on one entry: the tie-to-+1 majority
    # is +1 exactly when the +1 votes are at least half (counted bit by bit)
    for pattern in range(1 << M):
        plus = bin(pattern).count("1")
        packed = [np.array([(pattern >> m) & 1], np.uint8) for m in range(M)]
        sums = ref.vote_sums_from_bits(packed, 1, "int32")
        want = 1 if 2 * plus >= M else -1
        assert int(ref.majority(sums, tie=1)[0]) == want
        if M % 2 == 1:  # no ties with an odd number of voters
            assert int(ref.majority(sums, tie=1)[0]) == int(ref.majority(sums)[0])


def test_tie_plus_in_the_step_moves_w_by_eta():
    # two workers whose one-bit signs disagree everywhere: every entry ties;
    # tie=0 leaves W alone, tie=+1 moves every entry by -eta
    W = np.array([0.25, -0.5, 1.0, 0.0], np.float32)
    g1 = np.array([1.0, -1.0, 1.0, -1.0])
    out0 = ref.step(W, [g1, -g1], [np.zeros(4)] * 2, [(2, 2)], beta=0.0, lam=0.0, eta=0.125, K=0, eps=1e-7,
                    scale="fro")
    out1 = ref.step(W, [g1, -g1], [np.zeros(4)] * 2, [(2, 2)], beta=0.0, lam=0.0, eta=0.125, K=0, eps=1e-7,
                    scale="fro", tie=1)
    assert out0["sums"].tolist() == [0, 0, 0, 0]
    assert np.array_equal(out0["W"], W)
    assert out1["majority"].tolist() == [1, 1, 1, 1]
    assert np.array_equal(out1["W"], (W - np.float32(0.125)).astype(np.float32))


def test_after_only_polar_signs_the_momentum():
    # pre_polar=False: the signs are those of the momentum itself; all three
    # workers see sqrt(2) H (H orthogonal) so the majority is sign(H) and the
    # post-vote polar of the +-1 matrix sqrt(2) H' is H' f^K(sqrt(2)/(2+eps))
    H = np.array([[1.0, 1.0], [1.0, -1.0]]) / math.sqrt(2)
    G = (math.sqrt(2) * H).ravel()
    W = np.zeros(4, np.float32)
    eps = 1e-7
    out = ref.step(W, [G, G, G], [np.zeros(4)] * 3, [(2, 2)], beta=0.5, lam=0.0, eta=0.5, K=3, eps=eps,
                   scale="fro", post_polar=True, pre_polar=False)
    # momentum = (1 - beta) G: U is the momentum, unorthogonalised
    assert np.max(np.abs(out["U"][0] - 0.5 * G)) < 1e-15
    assert out["majority"].reshape(2, 2).tolist() == [[1, 1], [1, -1]]
    s1 = _f_cubic(np.array([math.sqrt(2) / (2 + eps)]), 3)[0]
    assert np.max(np.abs(out["D"].reshape(2, 2) - H * s1)) < 1e-14
    with pytest.raises(ValueError):
        ref.step(W, [G], [np.zeros(4)], [(2, 2)], beta=0.0, lam=0.0, eta=0.5, K=3, eps=eps, scale="fro",
                 pre_polar=False)


def test_muon_mean_closed_form():
    # the momenta of 3 workers are 0.5*(a_m * H) with mean 0.5*H*mean(a);
    # D = PolarNS(mean) = H f^K(|.|/(||.||_F+eps)) for the orthogonal H
    H = np.array([[1.0, 1.0], [1.0, -1.0]]) / math.sqrt(2)
    a = [1.0, 2.0, 6.0]
    G = [(x * H).ravel() for x in a]
    W = np.array([0.5, -0.25, 0.125, 1.0], np.float32)
    eps = 1e-7
    out = ref.muon_step(W, G, [np.zeros(4)] * 3, [(2, 2)], beta=0.5, lam=0.0, eta=0.25, K=4, eps=eps, scale="fro")
    mean = 0.5 * np.mean(a)
    assert np.max(np.abs(out["mean"] - mean * H.ravel())) < 1e-15
    # ||mean*H||_F = mean*sqrt(2): singular values are mean each
    s = _f_cubic(np.array([mean / (mean * math.sqrt(2) + eps)]), 4)[0]
    assert np.max(np.abs(out["D"].reshape(2, 2) - H * s)) < 1e-14
    assert np.array_equal(out["W"], ref.update(W, out["D32"], 0.25))
    # one worker: Muon's direction is that worker's polar factor
    one = ref.muon_step(W, G[:1], [np.zeros(4)], [(2, 2)], beta=0.5, lam=0.0, eta=0.25, K=4, eps=eps, scale="fro")
    full = ref.step(W, G[:1], [np.zeros(4)], [(2, 2)], beta=0.5, lam=0.0, eta=0.25, K=4, eps=eps, scale="fro")
    assert np.max(np.abs(one["D"] - full["U"][0])) < 1e-15


# ---------------------------------------------------------------------------
# ternary int8 signs ([paper] §3 sign(0) = 0; Algorithm 2's d-byte int8 SUM)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 6])
def test_ternary_vote_brute_force_all_patterns(M):
    # every pattern of M ternary votes on one entry, counted one by one
    for pattern in itertools.product((-1, 0, 1), repeat=M):
        plus = sum(1 for v in pattern if v == 1)
        minus = sum(1 for v in pattern if v == -1)
        signs = [np.array([v], np.int8) for v in pattern]
        s32 = ref.vote_sums_ternary(signs, "int32")
        s8 = ref.vote_sums_ternary(signs, "int8")
        assert s32.dtype == np.int32 and s8.dtype == np.int8
        assert int(s32[0]) == plus - minus == int(s8[0])
        want0 = 1 if plus > minus else (-1 if minus > plus else 0)
        want1 = 1 if plus >= minus else -1
        assert int(ref.majority(s32)[0]) == want0
        assert int(ref.majority(s32, tie=1)[0]) == want1


def test_ternary_vote_guards():
    with pytest.raises(ValueError):
        ref.vote_sums_ternary([np.array([2], np.int8)])
    with pytest.raises(ref.AccumulatorOverflow):
        ref.vote_sums_ternary([np.zeros(3, np.int8)] * 128, "int8")
    # 127 unanimous voters still fit an int8 accumulator
    assert ref.vote_sums_ternary([np.ones(3, np.int8)] * 127, "int8").tolist() == [127] * 3


def test_ternary_step_zero_momentum_closed_form():
    # zero gradients and no weight decay: Mom = 0, so U = 0 (0 / (0 + eps),
    # and NS keeps 0 at 0); the ternary signs are all 0, every sum is 0 and
    # tie=0 leaves W alone, tie=+1 moves it by -eta, while the one-bit wire
    # sends +1 (sign of 0 is +1 there) and moves it by -eta as well
    W = np.array([0.5, -0.25, 2.0, 0.0, 1.0, -1.0], np.float32)
    G = [np.zeros(6)] * 4
    kw = dict(beta=0.9, lam=0.0, eta=0.125, K=3, eps=1e-7, scale="fro")
    t0 = ref.step(W, G, [np.zeros(6)] * 4, [(2, 3)], signs="ternary", **kw)
    t1 = ref.step(W, G, [np.zeros(6)] * 4, [(2, 3)], signs="ternary", tie=1, **kw)
    b0 = ref.step(W, G, [np.zeros(6)] * 4, [(2, 3)], **kw)
    assert all(np.array_equal(p, np.zeros(6, np.int8)) for p in t0["packed"])
    assert t0["sums"].tolist() == [0] * 6 and t0["majority"].tolist() == [0] * 6
    assert np.array_equal(t0["W"], W)
    assert np.array_equal(t1["W"], (W - np.float32(0.125)).astype(np.float32))
    assert b0["sums"].tolist() == [4] * 6
    assert np.array_equal(b0["W"], t1["W"])


def test_ternary_step_equals_one_bit_step_without_zeros():
    # Gaussian gradients leave no exact zero in U: sign(U) in {-1, +1} and the
    # two wires must carry the same vote (ternary sums = 2 popcount - M)
    rng = np.random.default_rng(11)
    shapes = [(4, 6), (5, 3)]
    d = 24 + 15
    W = (0.02 * rng.standard_normal(d)).astype(np.float32)
    G = [rng.standard_normal(d) for _ in range(5)]
    kw = dict(beta=0.9, lam=0.01, eta=0.02, K=3, eps=1e-7, scale="spectral", P=2)
    t = ref.step(W, G, [np.zeros(d)] * 5, shapes, signs="ternary", **kw)
    b = ref.step(W, G, [np.zeros(d)] * 5, shapes, **kw)
    assert all(np.all(u != 0) for u in t["U"])
    assert np.array_equal(t["sums"], b["sums"])
    assert np.array_equal(t["majority"], b["majority"])
    assert np.array_equal(t["W"], b["W"])
    for m in range(5):
        assert np.array_equal(ref.pack_bits(t["packed"][m] > 0), b["packed"][m])
    tp = ref.step(W, G, [np.zeros(d)] * 5, shapes, signs="ternary", post_polar=True, **kw)
    bp = ref.step(W, G, [np.zeros(d)] * 5, shapes, post_polar=True, **kw)
    assert np.array_equal(tp["D32"], bp["D32"]) and np.array_equal(tp["W"], bp["W"])


# ---------------------------------------------------------------------------
# explicitly normalised sign step D / ||D||_2 ([paper] §4, single-worker notes)
# ---------------------------------------------------------------------------

def _sign_pattern_step(pattern, scale, P=2, M=3, eps=1e-7):
    # M identical workers whose gradient is the pattern itself: the majority
    # is the pattern (K = 0, positive scaling keeps every sign; the ternary
    # wire keeps the pattern's zeros, which the one-bit wire would send as +1)
    r, c = pattern.shape
    W = np.zeros(r * c, np.float32)
    G = [pattern.astype(np.float64).ravel()] * M
    return ref.step(W, G, [np.zeros(r * c)] * M, [(r, c)], beta=0.5, lam=0.0, eta=0.25, K=0, eps=eps,
                    scale=scale, P=P, normalize=True, signs="ternary")


@pytest.mark.parametrize("rows,cols", [(3, 5), (5, 3), (4, 4)])
def test_normalize_rank_one_sign_pattern(rows, cols):
    # a = sign pattern with unequal +-1 counts (so ones . a != 0), b any signs:
    # a b^T has the single singular value sqrt(rows*cols), and one power
    # iteration from the all-ones start lands on it exactly
    a = np.array([1, 1, -1, 1, 1][:rows], np.float64)
    b = np.array([1, -1, -1, 1, -1][:cols], np.float64)
    if rows == 4:
        a = np.array([1, 1, 1, -1], np.float64)
    pattern = np.outer(a, b)
    eps = 1e-7
    out = _sign_pattern_step(pattern, "spectral", P=1, eps=eps)
    assert out["majority"].reshape(rows, cols).tolist() == pattern.astype(int).tolist()
    want = pattern / (math.sqrt(rows * cols) + eps)
    assert np.max(np.abs(out["D"].reshape(rows, cols) - want)) < 1e-15
    assert np.array_equal(out["W"], ref.update(np.zeros(rows * cols, np.float32), out["D32"], 0.25))
    # Frobenius: ||a b^T||_F = sqrt(rows*cols) as well
    fro = _sign_pattern_step(pattern, "fro", eps=eps)
    assert np.max(np.abs(fro["D"].reshape(rows, cols) - want)) < 1e-15


@pytest.mark.parametrize("rows,cols", [(4, 4), (3, 6), (6, 3)])
@pytest.mark.parametrize("P", [1, 2, 5])
def test_normalize_signed_permutation(rows, cols, P):
    # one +-1 per row (wide) or per column (tall) at distinct places: every
    # singular value is 1, so D = pattern / (1 + eps) for any P
    k = min(rows, cols)
    perm = [2, 0, 3, 1, 5, 4][:k] if max(rows, cols) >= 6 else [2, 0, 3, 1][:k]
    sgn = [1, -1, -1, 1, 1, -1]
    pattern = np.zeros((rows, cols))
    for i in range(k):
        if rows <= cols:
            pattern[i, perm[i] % cols] = sgn[i]
        else:
            pattern[perm[i] % rows, i] = sgn[i]
    assert np.allclose(np.linalg.svd(pattern, compute_uv=False), 1.0)
    eps = 1e-7
    out = _sign_pattern_step(pattern, "spectral", P=P, eps=eps)
    assert out["majority"].reshape(rows, cols).tolist() == pattern.astype(int).tolist()
    assert np.max(np.abs(out["D"].reshape(rows, cols) - pattern / (1.0 + eps))) < 1e-15


def test_normalize_against_exact_sigma_max():
    # a sign pattern with a dominant rank-one part: many power iterations
    # reach numpy's exact largest singular value of the majority matrix
    rng = np.random.default_rng(5)
    u, v = rng.standard_normal(7), rng.standard_normal(11)
    pattern = np.sign(np.outer(u, v) + 0.3 * rng.standard_normal((7, 11)))
    pattern[pattern == 0] = 1
    out = _sign_pattern_step(pattern, "spectral", P=300, eps=1e-12)
    smax = np.linalg.svd(out["majority"].reshape(7, 11).astype(np.float64), compute_uv=False)[0]
    assert np.max(np.abs(out["D"].reshape(7, 11) * smax - pattern)) < 1e-9
    fro = _sign_pattern_step(pattern, "fro", eps=1e-12)
    assert np.max(np.abs(fro["D"].reshape(7, 11) * math.sqrt(77.0) - pattern)) < 1e-9


def test_normalize_of_an_all_tied_vote_is_zero_and_guards():
    # two workers with opposite signs everywhere: every entry ties, the
    # majority is 0, and eps keeps D at 0 (no 0/0)
    W = np.array([0.25, -0.5, 1.0, 0.0], np.float32)
    g = np.array([1.0, -1.0, 2.0, -3.0])
    out = ref.step(W, [g, -g], [np.zeros(4)] * 2, [(2, 2)], beta=0.0, lam=0.0, eta=0.5, K=2, eps=1e-7,
                   scale="spectral", P=2, normalize=True)
    assert out["majority"].tolist() == [0, 0, 0, 0]
    assert np.array_equal(out["D"], np.zeros(4)) and np.array_equal(out["W"], W)
    with pytest.raises(ValueError):
        ref.step(W, [g], [np.zeros(4)], [(2, 2)], beta=0.0, lam=0.0, eta=0.5, K=2, eps=1e-7, scale="fro",
                 normalize=True, post_polar=True)
    with pytest.raises(ValueError):
        ref.step(W, [g], [np.zeros(4)], [(2, 2)], beta=0.0, lam=0.0, eta=0.5, K=2, eps=1e-7, scale="fro",
                 signs="trits")


# ---------------------------------------------------------------------------
# warm-started power iteration (named variant: the iterate carried across steps)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("P", [1, 2])
def test_warm_power_iteration_composes_with_cold_start(P):
    # power iteration composes: t warm calls of P iterations on one matrix are
    # the same arithmetic as one cold call of P*t iterations (bit for bit)
    rng = np.random.default_rng(3)
    x = rng.standard_normal((6, 9))
    u = None
    for t in range(1, 6):
        s_warm, u = ref.power_sigma(x, P, u, return_u=True)
        s_cold, u_cold = ref.power_sigma(x, P * t, return_u=True)
        assert s_warm == s_cold and np.array_equal(u, u_cold)
    # and it converges to numpy's largest singular value
    s_far, _ = ref.power_sigma(x, 400, return_u=True)
    assert abs(s_far - np.linalg.svd(x, compute_uv=False)[0]) < 1e-12 * s_far


def test_warm_power_iteration_fixed_point_and_restart():
    # diag(5, 2, 1) padded wide: e1 is the top singular vector, so a warm
    # start there gives sigma = 5 after one iteration; a zero or non-finite
    # stored iterate restarts from ones/sqrt(m) exactly like a cold start
    x = np.zeros((3, 5))
    x[0, 0], x[1, 1], x[2, 2] = 5.0, 2.0, 1.0
    s, u = ref.power_sigma(x, 1, np.array([1.0, 0.0, 0.0]), return_u=True)
    assert s == 5.0 and np.array_equal(u, np.array([1.0, 0.0, 0.0]))
    cold = ref.power_sigma(x, 2)
    assert ref.power_sigma(x, 2, np.zeros(3)) == cold
    assert ref.power_sigma(x, 2, np.array([np.nan, 1.0, 0.0])) == cold
    # a zero matrix leaves a zero iterate behind, which the next call restarts
    s0, u0 = ref.power_sigma(np.zeros((3, 5)), 2, return_u=True)
    assert s0 == 0.0 and not u0.any()
    assert ref.power_sigma(x, 2, u0) == cold


@pytest.mark.parametrize("post_polar", [False, True])
def test_warm_step_threads_the_state_per_worker_and_matrix(post_polar):
    # beta = 0, lambda = 0 and one gradient per worker repeated every step:
    # the momentum (so the Gram) is constant, and after t warm steps of P
    # iterations each (worker, matrix) iterate equals a cold start with P*t
    # iterations on that worker's matrix; the post-vote state does the same on
    # the majority matrix, constant too because K = 0 makes the signs those of
    # the momentum (with K > 0 the changing scale moves small entries of U)
    rng = np.random.default_rng(9)
    shapes = [(4, 7), (6, 3)]
    d = 28 + 18
    M, P = 3, 1
    G = [rng.standard_normal(d) for _ in range(M)]
    W = np.zeros(d, np.float32)
    kw = dict(beta=0.0, lam=0.0, eta=0.01, K=0, eps=1e-7, scale="spectral", P=P, post_polar=post_polar)
    warm = {}
    maj0 = None
    for t in range(1, 4):
        out = ref.step(W, G, [np.zeros(d)] * M, shapes, warm=warm, **kw)
        warm = out["warm"]
        maj0 = out["majority"] if maj0 is None else maj0
        assert np.array_equal(out["majority"], maj0)
        for m in range(M):
            for i, x in enumerate(ref.split(G[m], shapes)):
                xw = x.T if x.shape[0] > x.shape[1] else x
                _, u_cold = ref.power_sigma(xw, P * t, return_u=True)
                assert np.array_equal(warm["workers"][m][i], u_cold)
        if post_polar:
            for i, x in enumerate(ref.split(out["majority"].astype(np.float64), shapes)):
                xw = x.T if x.shape[0] > x.shape[1] else x
                _, u_cold = ref.power_sigma(xw, P * t, return_u=True)
                assert np.array_equal(warm["single"][i], u_cold)
        else:
            assert warm["single"] is None
    # without warm the step keeps no state
    assert ref.step(W, G, [np.zeros(d)] * M, shapes, **kw)["warm"] is None


def test_warm_muon_step_uses_the_single_state():
    rng = np.random.default_rng(13)
    shapes = [(5, 8)]
    G = [rng.standard_normal(40) for _ in range(2)]
    W = np.zeros(40, np.float32)
    kw = dict(beta=0.0, lam=0.0, eta=0.01, K=1, eps=1e-7, scale="spectral", P=2)
    warm = {}
    for t in range(1, 3):
        out = ref.muon_step(W, G, [np.zeros(40)] * 2, shapes, warm=warm, **kw)
        warm = out["warm"]
        _, u_cold = ref.power_sigma(out["mean"].reshape(5, 8), 2 * t, return_u=True)
        assert np.array_equal(warm["single"][0], u_cold)


def test_float32_mode_matches_float64_within_the_fp32_tolerance():
    """The oracle's float32 mode (timed as the CPU baseline) against its
    float64 parity mode on the small 256x128 workload and a post-vote step:
    the polar factors within the fp32 polar tolerance (1e-4), the momentum
    within float32 rounding, and the float32 arithmetic really in float32."""
    shapes = [(256, 128), (96, 300)]
    M = 3
    w0 = synth.weights0(shapes, 71)
    G = synth.gradients(shapes, M, 0.5, step=1, config_id=71)
    mom0 = synth.momentum0(shapes, M, 71, scale=0.5)
    kw = dict(beta=0.9, lam=0.01, eta=0.02, K=5, eps=1e-7, scale="spectral", P=2, post_polar=True)
    a = ref.step(w0, G, mom0, shapes, **kw)
    b = ref.step(w0, G, mom0, shapes, dtype=np.float32, **kw)
    for m in range(M):
        assert b["mom"][m].dtype == np.float32 and b["U"][m].dtype == np.float32
        assert np.max(np.abs(b["mom"][m] - a["mom"][m])) <= 4 * 2.0 ** -24 * np.max(np.abs(a["mom"][m])) * 4
        assert np.max(np.abs(b["U"][m] - a["U"][m])) <= 1e-4
    assert np.max(np.abs(b["D"] - a["D"])) <= 1e-4
