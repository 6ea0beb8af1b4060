"""Property-based checks of the oracle (hypothesis): invariants that must hold
for every input, against references other than the oracle itself: numpy's
packbits, exact rational arithmetic, LAPACK's SVD and counting by hand.  Each
property runs a bounded number of small examples, so the file stays fast."""
from fractions import Fraction

import numpy as np
import pytest

hyp = pytest.importorskip("hypothesis")
from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402

from oracle import signmuon_ref as ref  # noqa: E402

# derandomized: the same examples on every run
FAST = settings(max_examples=60, deadline=None, derandomize=True)
SLOW = settings(max_examples=25, deadline=None, derandomize=True)

finite32 = st.floats(min_value=-2.0 ** 100, max_value=2.0 ** 100, allow_nan=False, width=32)


@FAST
@given(st.lists(st.booleans(), min_size=0, max_size=300))
def test_pack_equals_numpy_packbits_and_round_trips(bits):
    b = np.array(bits, bool)
    packed = ref.pack_bits(b)
    assert packed.size == (b.size + 7) // 8
    assert np.array_equal(packed, np.packbits(b, bitorder="little"))
    assert np.array_equal(ref.unpack_bits(packed, b.size), b)


@FAST
@given(st.integers(1, 12), st.integers(1, 40), st.integers(0, 2 ** 31 - 1))
def test_one_bit_vote_invariants(M, d, seed):
    rng = np.random.default_rng(seed)
    bits = rng.random((M, d)) < 0.5
    sums = ref.vote_sums_from_bits([ref.pack_bits(b) for b in bits], d)
    plus = bits.sum(axis=0)
    # sum = 2 popcount - M, in [-M, M], with the parity of M
    assert np.array_equal(sums, 2 * plus - M)
    assert np.all(np.abs(sums) <= M) and np.all((sums - M) % 2 == 0)
    maj = ref.majority(sums)
    assert np.array_equal(maj, np.where(2 * plus > M, 1, np.where(2 * plus < M, -1, 0)))


@FAST
@given(st.integers(1, 12), st.integers(1, 40), st.integers(0, 2 ** 31 - 1))
def test_ternary_vote_is_a_plain_count(M, d, seed):
    rng = np.random.default_rng(seed)
    t = rng.integers(-1, 2, size=(M, d)).astype(np.int8)
    sums = ref.vote_sums_ternary(list(t))
    for i in range(d):  # counted one entry at a time
        assert int(sums[i]) == sum(1 for m in range(M) if t[m, i] == 1) - sum(1 for m in range(M) if t[m, i] == -1)


@FAST
@given(finite32, finite32, st.sampled_from([-1.0, 0.0, 1.0]))
def test_update_is_one_rounding_of_the_exact_value(w, eta, dsign):
    w32, eta32, d32 = np.float32(w), np.float32(eta), np.float32(dsign)
    got = ref.update(np.array([w32]), np.array([d32]), eta32)[0]
    exact = Fraction(float(w32)) - Fraction(float(eta32)) * Fraction(float(d32))
    if not np.isfinite(got):
        return  # overflow: nothing to compare at this magnitude
    # no float32 lies strictly closer to the exact value than the result
    err = abs(Fraction(float(got)) - exact)
    for nb in (np.nextafter(got, np.float32(np.inf)), np.nextafter(got, np.float32(-np.inf))):
        if np.isfinite(nb):
            assert abs(Fraction(float(nb)) - exact) >= err


@SLOW
@given(st.integers(1, 6), st.integers(1, 6), st.integers(0, 2 ** 31 - 1))
def test_power_iteration_never_overestimates_and_converges(r, c, seed):
    x = np.random.default_rng(seed).standard_normal((r, c))
    xw = x if r <= c else x.T
    sv = np.linalg.svd(x, compute_uv=False)
    smax = sv[0]
    prev = 0.0
    for P in (1, 2, 4, 8):
        s = ref.power_sigma(xw, P)
        assert s <= smax * (1 + 1e-12)          # a Rayleigh-quotient estimate from below
        assert s >= prev * (1 - 1e-12)          # and it never decreases with P
        prev = s
    if len(sv) == 1 or sv[1] < 0.99 * sv[0]:   # a gap: the error shrinks like (s2/s1)^(2P)
        assert abs(ref.power_sigma(xw, 2000) - smax) <= 1e-6 * smax


@SLOW
@given(st.integers(1, 5), st.integers(1, 5), st.integers(0, 2 ** 31 - 1))
def test_polar_of_a_well_conditioned_matrix_reaches_the_svd_factor(r, c, seed):
    rng = np.random.default_rng(seed)
    k = min(r, c)
    q1, _ = np.linalg.qr(rng.standard_normal((r, k)))
    q2, _ = np.linalg.qr(rng.standard_normal((c, k)))
    sv = rng.uniform(0.5, 1.0, size=k)          # condition number at most 2
    x = q1 @ np.diag(sv) @ q2.T
    u, _, vt = np.linalg.svd(x, full_matrices=False)
    polar = u @ vt
    got = ref.polar_ns(x, 40, 1e-12, "fro")
    assert np.max(np.abs(got - polar)) < 1e-9
    # the signs of the result are what the one-bit and ternary paths send
    assert np.array_equal(ref.sign_bits(got), got >= 0)


@SLOW
@given(st.integers(2, 5), st.integers(0, 2 ** 31 - 1), st.booleans(), st.sampled_from(["bits", "ternary"]))
def test_step_is_symmetric_in_the_workers(M, seed, post_polar, signs):
    # the vote is a sum: any order of the workers gives the same W and D
    rng = np.random.default_rng(seed)
    shapes = [(3, 5), (4, 2)]
    d = 15 + 8
    W = (0.02 * rng.standard_normal(d)).astype(np.float32)
    G = [rng.standard_normal(d) for _ in range(M)]
    mom = [0.3 * rng.standard_normal(d) for _ in range(M)]
    kw = dict(beta=0.9, lam=0.01, eta=0.02, K=3, eps=1e-7, scale="spectral", P=2, post_polar=post_polar,
              signs=signs)
    a = ref.step(W, G, mom, shapes, **kw)
    perm = rng.permutation(M)
    b = ref.step(W, [G[i] for i in perm], [mom[i] for i in perm], shapes, **kw)
    assert np.array_equal(a["sums"], b["sums"]) and np.array_equal(a["W"], b["W"])
    assert np.array_equal(a["D32"], b["D32"])


@SLOW
@given(st.integers(1, 6), st.integers(0, 2 ** 31 - 1), st.sampled_from([0, 1]))
def test_identical_workers_vote_like_one(M, seed, tie):
    # M copies of one worker: every sum is +-M (or 0 only where its ternary
    # sign is 0), so the majority, D and W are the one-worker step's
    rng = np.random.default_rng(seed)
    shapes = [(5, 3)]
    W = (0.02 * rng.standard_normal(15)).astype(np.float32)
    g = rng.standard_normal(15)
    kw = dict(beta=0.5, lam=0.01, eta=0.05, K=2, eps=1e-7, scale="fro", tie=tie)
    one = ref.step(W, [g], [np.zeros(15)], shapes, **kw)
    many = ref.step(W, [g] * M, [np.zeros(15)] * M, shapes, **kw)
    assert np.array_equal(many["sums"], M * one["sums"])
    assert np.array_equal(many["majority"], one["majority"]) and np.array_equal(many["W"], one["W"])


@SLOW
@given(st.integers(1, 7), st.integers(1, 7), st.integers(1, 4), st.integers(0, 2 ** 31 - 1))
def test_normalised_sign_step_norm_bounds(r, c, P, seed):
    # D = maj / (s + eps): the power-iteration estimate never exceeds sigma_max,
    # so the spectral-normalised D has ||D||_2 >= 1 - eps/sigma (any P); the
    # Frobenius norm bounds sigma_max from above, so that D has ||D||_2 < 1
    rng = np.random.default_rng(seed)
    maj = rng.integers(-1, 2, size=(r, c)).astype(np.float64)
    if not maj.any():
        maj[0, 0] = 1.0
    eps = 1e-9
    for scale in ("spectral", "fro"):
        D = ref.normalize_flat(maj.ravel(), [(r, c)], eps, scale, P).reshape(r, c)
        n2 = np.linalg.svd(D, compute_uv=False)[0]
        if scale == "spectral":
            assert n2 >= 1.0 - 1e-6
        else:
            assert n2 <= 1.0
        assert np.array_equal(np.sign(D), maj)      # a positive rescaling only
