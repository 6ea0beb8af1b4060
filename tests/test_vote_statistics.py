"""The vote's reliability against probability theory (the 1/sqrt(M) trend in
the convergence bound of [paper] "SignMuon: 通信高效的分布式Muon优化" §5,
Theorem 5.4, and the noise-averaging argument of its §3): for gradients
G_m = S + sigma N_m with the N_m i.i.d. standard normal, worker m's one-bit
sign of an entry is wrong with probability p = Phi(-|S| / sigma),
independently across workers, so the majority of M workers is wrong, or for
even M tied at 0, with the binomial tail probability
    t_M(p) = P(Bin(M, p) > M/2) + P(Bin(M, p) = M/2).
The measured mismatch fraction against sign(S) must equal the mean of t_M over
the entries to within a few standard deviations of its sampling error, and
fall as M grows.  A statistical check of the vote's counting and tie rule
(the oracle's on the CPU; the library's pack and vote kernels on the GPU), not
a parity check."""
import math

import numpy as np
import pytest

from oracle import signmuon_ref as ref

SIGMA = 2.0          # the nanoGPT workload's noise level
D = 200_000
M_ODD = [1, 3, 5, 9, 17]


def _phi_neg(x):
    """Phi(-x) for x >= 0, elementwise."""
    return 0.5 * np.vectorize(math.erfc)(np.asarray(x, np.float64) / math.sqrt(2.0))


def _tail(M, p):
    """P(Bin(M, p) > M/2) + P(Bin(M, p) = M/2), elementwise in p."""
    k = np.arange(M + 1)
    comb = np.array([math.comb(M, int(i)) for i in k], np.float64)
    pk = comb[None, :] * p[:, None] ** k[None, :] * (1.0 - p[:, None]) ** (M - k)[None, :]
    return pk[:, 2 * k > M].sum(axis=1) + pk[:, 2 * k == M].sum(axis=1)


def _inputs(M, seed):
    rng = np.random.default_rng(seed)
    S = rng.standard_normal(D)
    G = [(S + SIGMA * rng.standard_normal(D)).astype(np.float32) for _ in range(M)]
    return S, G


def _expected(M, S):
    t = _tail(M, _phi_neg(np.abs(S) / SIGMA))
    return t.mean(), math.sqrt(float((t * (1.0 - t)).sum())) / S.size


def _oracle_mismatch(M, S, G):
    packed = [ref.pack_bits(ref.sign_bits(g)) for g in G]
    maj = ref.majority(ref.vote_sums_from_bits(packed, D))
    return float((maj != np.sign(S)).mean())


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 9, 17])
def test_oracle_vote_error_is_the_binomial_tail(M):
    S, G = _inputs(M, 1000 + M)
    want, sd = _expected(M, S)
    got = _oracle_mismatch(M, S, G)
    assert abs(got - want) <= 5.0 * sd, (M, got, want, sd)


def test_vote_error_falls_with_more_workers():
    """Odd M (no ties): both the tail and the measured mismatch decrease; from
    M = 1 to M = 17 the error drops by more than half."""
    got, want = [], []
    for M in M_ODD:
        S, G = _inputs(M, 2000 + M)
        want.append(_expected(M, S)[0])
        got.append(_oracle_mismatch(M, S, G))
    assert all(a > b for a, b in zip(want, want[1:]))
    assert all(a > b for a, b in zip(got, got[1:]))
    assert got[-1] < 0.5 * got[0]


@pytest.mark.gpu
@pytest.mark.parametrize("M", [2, 5, 17])
def test_library_vote_error_is_the_binomial_tail(M):
    """The same through the library: signmuon_pack of each worker's gradient,
    then signmuon_vote; its majority must equal the oracle's bit for bit and
    meet the same statistical bound."""
    torch = pytest.importorskip("torch")
    import sign_muon_optimizer_b200 as smo
    S, G = _inputs(M, 3000 + M)
    h = smo.SignMuon([(1, D)], M, flags=smo.SIGNMUON_VOTE_ONLY)
    nb = ref.packed_nbytes(D)
    bufs = []
    for g in G:
        b = torch.zeros(nb + 16, dtype=torch.uint8, device="cuda")
        h.pack(torch.from_numpy(g).cuda(), D, b)
        bufs.append(b)
    maj = torch.zeros(D, dtype=torch.int8, device="cuda")
    h.vote(bufs, D, None, maj)
    got_maj = maj.cpu().numpy()
    packed = [ref.pack_bits(ref.sign_bits(g)) for g in G]
    assert np.array_equal(got_maj, ref.majority(ref.vote_sums_from_bits(packed, D)))
    want, sd = _expected(M, S)
    assert abs(float((got_maj != np.sign(S)).mean()) - want) <= 5.0 * sd
