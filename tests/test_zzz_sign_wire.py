"""GPU parity of the sign-wire variants: the int8 ternary signs (SIGNMUON_TERNARY,
signmuon_sign_ternary, signmuon_vote_ternary) and the explicitly normalised
sign step (SIGNMUON_NORMALIZED_SIGN).

Sources, by page title: [paper] "SignMuon: 通信高效的分布式Muon优化" §3 (sign(0) = 0),
§4 (the analysis normalises the sign matrix by its spectral norm), Algorithm 2
(an int8 SUM all-reduce of d bytes per worker); [blog] "SignMuon: Matrix
Directions, Majority Votes, and the Actual Bytes Sent" (ternary vote, ties to 0).

Integer results (signs, sums, majorities) are compared bit for bit with the
oracle; the normalised direction against the oracle's D / (s + eps) on the
GPU's own majority, and against closed forms (rank-one sign patterns and
signed permutations, whose spectral norms are sqrt(rows*cols) and 1).  The
file name sorts it after the other GPU suites.
"""
import numpy as np
import pytest

import synth
from oracle import signmuon_ref as ref

from gpu_helpers import assert_momentum_close, assert_polar_close, dev, host, oracle_polar_flat

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import sign_muon_optimizer_b200 as smo  # noqa: E402

HP = dict(beta=0.9, lam=0.01, eta=0.02, eps=1e-7)
# relative error of the normalised direction: bf16 rounds the majority's Gram
# matrix before the power iteration (2^-9 relative per entry), fp32 does not
NORM_RTOL = {"bf16": 1e-2, "fp32": 1e-4}


# ---------------------------------------------------------------------------
# kernels through the C ABI
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d", [0, 1, 15, 16, 17, 4096 + 5, 100003])
def test_sign_ternary_bit_exact(d):
    u = synth.uniform_values(d, config_id=21, step=d)
    if d > 40:
        u[3], u[4], u[5], u[6] = np.nan, np.inf, -np.inf, np.float32(1e-45)
        u[7], u[8] = np.float32(-0.0), np.float32(0.0)
    h = smo.SignMuon([(1, 1)], 1, flags=smo.SIGNMUON_VOTE_ONLY)
    out = torch.full((max(d, 1),), 7, dtype=torch.int8, device="cuda")
    h.sign_ternary(dev(u) if d else torch.zeros(1, device="cuda"), d, out)
    got = host(out)
    assert np.array_equal(got[:d], ref.sign_ternary(u).astype(np.int8))
    if d == 0:
        assert got[0] == 7  # nothing written


@pytest.mark.parametrize("M,d", [(1, 1000), (3, 17), (4, 65536 + 7), (8, 100003), (127, 4099), (200, 5000),
                                 (256, 1000)])
@pytest.mark.parametrize("tie", [0, 1])
def test_vote_ternary_bit_exact(M, d, tie):
    # M = 200, 256: more workers than the byte lanes hold (flushed every 120)
    t = synth.ternary_signs(d, M, config_id=M * 100 + d % 89)
    want = ref.vote_sums_ternary(list(t), "int32")
    flags = smo.SIGNMUON_VOTE_ONLY | (smo.SIGNMUON_TIE_PLUS if tie else 0)
    h = smo.SignMuon([(1, 1)], M, flags=flags)
    signs = [dev(t[m]) for m in range(M)]
    sums = torch.zeros(d, dtype=torch.int32, device="cuda")
    maj = torch.zeros(d, dtype=torch.int8, device="cuda")
    h.vote_ternary(signs, d, sums, maj)
    assert np.array_equal(host(sums), want)
    assert np.array_equal(host(maj), ref.majority(want, tie=tie))
    if M <= 127:
        h8 = smo.SignMuon([(1, 1)], M, flags=flags | smo.SIGNMUON_ACC_INT8)
        s8 = torch.zeros(d, dtype=torch.int8, device="cuda")
        h8.vote_ternary(signs, d, s8, None)
        assert np.array_equal(host(s8), ref.vote_sums_ternary(list(t), "int8"))


def test_vote_ternary_blog_worked_example_and_empty():
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "blog_worked_example.json")))
    dirs = np.array(g["directions"], np.float32)
    h = smo.SignMuon([(1, 1)], len(dirs), flags=smo.SIGNMUON_VOTE_ONLY)
    signs = []
    for x in dirs:
        s = torch.zeros(4, dtype=torch.int8, device="cuda")
        h.sign_ternary(dev(x.ravel()), 4, s)
        signs.append(s)
    sums = torch.zeros(4, dtype=torch.int32, device="cuda")
    maj = torch.zeros(4, dtype=torch.int8, device="cuda")
    h.vote_ternary(signs, 4, sums, maj)
    assert host(sums).reshape(2, 2).tolist() == g["sums"]
    assert host(maj).reshape(2, 2).tolist() == g["majority"]
    before = smo.signmuon_kernel_launches()
    h.vote_ternary(signs, 0, sums, maj)  # empty: no launch, no write
    assert smo.signmuon_kernel_launches() == before
    assert host(sums).reshape(2, 2).tolist() == g["sums"]


# ---------------------------------------------------------------------------
# the step with the ternary wire
# ---------------------------------------------------------------------------

def _ternary_step(shapes, M, K, scale, P, precision, extra, seed, tie=0):
    flags = smo.SIGNMUON_TERNARY | (smo.SIGNMUON_NS_FP32 if precision == "fp32" else 0) | extra
    if not extra & smo.SIGNMUON_POLAR_AFTER_ONLY:
        flags |= smo.SIGNMUON_KEEP_POLAR   # U is read back below
    if tie:
        flags |= smo.SIGNMUON_TIE_PLUS
    h = smo.SignMuon(shapes, M, beta=HP["beta"], lam=HP["lam"], K=K, eps=HP["eps"], scale=scale, P=P, flags=flags)
    d = h.d
    w0 = synth.weights0(shapes, seed)
    mom0 = synth.momentum0(shapes, M, seed, scale=0.5)
    G = synth.gradients(shapes, M, 1.0, step=1, config_id=seed)
    for m in range(M):
        h.set_momentum(m, dev(mom0[m]))
    W = dev(w0)
    h.step(W, [dev(g) for g in G], HP["eta"])
    gpu = dict(mom=[], U=[], t=[])
    for m in range(M):
        x = torch.zeros(d, device="cuda")
        h.get_momentum(m, x)
        gpu["mom"].append(host(x))
        if not extra & smo.SIGNMUON_POLAR_AFTER_ONLY:
            x = torch.zeros(d, device="cuda")
            h.get_polar(m, x)
            gpu["U"].append(host(x))
        s = torch.full((d,), 5, dtype=torch.int8, device="cuda")
        h.get_ternary_signs(m, s)
        gpu["t"].append(host(s))
    D = torch.zeros(d, device="cuda")
    h.get_direction(D)
    gpu["D"], gpu["W"] = host(D), host(W)
    with pytest.raises(smo.SignMuonError) as ei:
        h.get_signs(0, torch.zeros(ref.packed_nbytes(d) + 16, dtype=torch.uint8, device="cuda"))
    assert ei.value.status == smo.SIGNMUON_E_UNSUPPORTED
    return h, gpu, dict(w0=w0, mom0=mom0, G=G)


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
@pytest.mark.parametrize("post_polar", [False, True])
def test_step_ternary(precision, post_polar):
    shapes = [(3, 5), (130, 70), (64, 147), (96, 300)]
    M, K, scale, P = 4, 5, "spectral", 2  # even M: ties occur
    h, gpu, inp = _ternary_step(shapes, M, K, scale, P, precision,
                                smo.SIGNMUON_POST_POLAR if post_polar else 0, seed=61)
    want = ref.step(inp["w0"], inp["G"], inp["mom0"], shapes, beta=HP["beta"], lam=HP["lam"], eta=HP["eta"], K=K,
                    eps=HP["eps"], scale=scale, P=P, post_polar=post_polar, signs="ternary")
    d = synth.numel(shapes)
    agree = np.ones(d, bool)
    for m in range(M):
        assert_momentum_close(gpu["mom"][m], inp["mom0"][m], inp["G"][m], inp["w0"], HP["beta"], HP["lam"])
        assert_polar_close(gpu["U"][m], want["U"][m], precision, f"U worker {m}")
        # the int8 signs are exactly the ternary signs of the GPU's own U
        assert np.array_equal(gpu["t"][m], ref.sign_ternary(gpu["U"][m]).astype(np.int8))
        agree &= gpu["t"][m] == want["packed"][m]
    # the vote on the GPU's own signs, bit for bit
    maj = ref.majority(ref.vote_sums_ternary(gpu["t"]))
    assert np.array_equal(maj[agree], want["majority"][agree])
    assert (~agree).mean() <= M * 1e-3
    if post_polar:
        D_ref = oracle_polar_flat(maj.astype(np.float64), shapes, K, HP["eps"], scale, P)
        assert_polar_close(gpu["D"], D_ref, precision, "post-vote polar of the ternary majority")
    else:
        assert np.array_equal(gpu["D"], maj.astype(np.float32))
    assert np.array_equal(gpu["W"].view(np.uint32), ref.update(inp["w0"], gpu["D"], HP["eta"]).view(np.uint32))


def test_step_ternary_after_only_tie_plus():
    """The ternary signs of the momentum itself, orthogonalised only after
    the vote, ties to +1."""
    shapes = [(64, 96), (130, 70)]
    M, K, scale, P = 4, 5, "fro", 1
    h, gpu, inp = _ternary_step(shapes, M, K, scale, P, "fp32",
                                smo.SIGNMUON_POST_POLAR | smo.SIGNMUON_POLAR_AFTER_ONLY, seed=67, tie=1)
    for m in range(M):
        assert np.array_equal(gpu["t"][m], ref.sign_ternary(gpu["mom"][m]).astype(np.int8))
    maj = ref.majority(ref.vote_sums_ternary(gpu["t"]), tie=1)
    D_ref = oracle_polar_flat(maj.astype(np.float64), shapes, K, HP["eps"], scale, P)
    assert_polar_close(gpu["D"], D_ref, "fp32", "post-vote polar, after-only placement")
    assert np.array_equal(gpu["W"].view(np.uint32), ref.update(inp["w0"], gpu["D"], HP["eta"]).view(np.uint32))


@pytest.mark.parametrize("tie", [0, 1])
def test_step_ternary_zero_gradients(tie):
    """Closed form: zero gradients and momentum with no weight decay give U = 0,
    every ternary sign 0 and every sum 0: W stays bit for bit (tie to 0) or
    moves by exactly -eta (tie to +1)."""
    shapes = [(64, 96), (96, 64)]
    M = 3
    d = synth.numel(shapes)
    flags = smo.SIGNMUON_TERNARY | (smo.SIGNMUON_TIE_PLUS if tie else 0)
    h = smo.SignMuon(shapes, M, beta=HP["beta"], lam=0.0, K=5, eps=HP["eps"], scale="spectral", P=2, flags=flags)
    w0 = synth.weights0(shapes, 71)
    W = dev(w0)
    h.step(W, [torch.zeros(d, device="cuda") for _ in range(M)], HP["eta"])
    for m in range(M):
        s = torch.full((d,), 9, dtype=torch.int8, device="cuda")
        h.get_ternary_signs(m, s)
        assert not host(s).any()
    want = ref.step(w0, [np.zeros(d)] * M, [np.zeros(d)] * M, shapes, beta=HP["beta"], lam=0.0, eta=HP["eta"], K=5,
                    eps=HP["eps"], scale="spectral", P=2, signs="ternary", tie=tie)
    assert np.array_equal(host(W).view(np.uint32), want["W"].view(np.uint32))
    if tie == 0:
        assert np.array_equal(want["W"], w0)


# ---------------------------------------------------------------------------
# the explicitly normalised sign step
# ---------------------------------------------------------------------------

def _norm_compare(gpu_D, maj, shapes, eps, scale, P, precision):
    want = ref.normalize_flat(maj.astype(np.float64), shapes, eps, scale, P)
    off = 0
    for r, c in shapes:
        sl = slice(off, off + r * c)
        Dg, Dw = gpu_D[sl].astype(np.float64), want[sl]
        # zeros exactly where the majority is 0; one magnitude per matrix
        assert np.array_equal(Dg == 0, maj[sl] == 0)
        nz = Dg[Dg != 0]
        if nz.size:
            assert np.all(np.abs(nz) == np.abs(nz[0]))
            assert np.array_equal(np.sign(nz), np.sign(Dw[Dw != 0]))
            rel = abs(abs(nz[0]) - abs(Dw[Dw != 0][0])) / abs(Dw[Dw != 0][0])
            assert rel <= NORM_RTOL[precision], f"{r}x{c}: relative error {rel:.3e}"
        off += r * c


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
@pytest.mark.parametrize("scale,P", [("spectral", 2), ("fro", 1)])
@pytest.mark.parametrize("ternary", [False, True])
def test_step_normalized_sign(precision, scale, P, ternary):
    shapes = [(3, 5), (130, 70), (64, 147), (96, 300)]
    M, K, seed = 4, 5, 73
    d = synth.numel(shapes)
    flags = smo.SIGNMUON_NORMALIZED_SIGN | smo.SIGNMUON_KEEP_POLAR
    flags |= smo.SIGNMUON_NS_FP32 if precision == "fp32" else 0
    flags |= smo.SIGNMUON_TERNARY if ternary else 0
    h = smo.SignMuon(shapes, M, beta=HP["beta"], lam=HP["lam"], K=K, eps=HP["eps"], scale=scale, P=P, flags=flags)
    w0 = synth.weights0(shapes, seed)
    mom0 = synth.momentum0(shapes, M, seed, scale=0.5)
    G = synth.gradients(shapes, M, 1.0, step=1, config_id=seed)
    for m in range(M):
        h.set_momentum(m, dev(mom0[m]))
    W = dev(w0)
    h.step(W, [dev(g) for g in G], HP["eta"])
    sums = np.zeros(d, np.int64)
    for m in range(M):
        if ternary:
            s = torch.zeros(d, dtype=torch.int8, device="cuda")
            h.get_ternary_signs(m, s)
            sums += host(s).astype(np.int64)
        else:
            b = torch.zeros(ref.packed_nbytes(d) + 16, dtype=torch.uint8, device="cuda")
            h.get_signs(m, b)
            sums += 2 * ref.unpack_bits(host(b), d).astype(np.int64) - 1
    maj = ref.majority(sums)
    Dg = torch.zeros(d, device="cuda")
    h.get_direction(Dg)
    D = host(Dg)
    _norm_compare(D, maj, shapes, HP["eps"], scale, P, precision)
    assert np.array_equal(host(W).view(np.uint32), ref.update(w0, D, HP["eta"]).view(np.uint32))


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_step_normalized_sign_closed_forms(precision):
    """Independent of the oracle.  (a) Every worker's gradient is a rank-one
    sign pattern a b^T: the polar factor keeps its signs, the majority is the
    pattern and its spectral norm is sqrt(rows*cols).  (b) With the ternary
    wire, a signed partial permutation keeps its zeros through PolarNS; its
    singular values are all 1, so D = pattern / (1 + eps)."""
    M, eps = 3, HP["eps"]
    shapes = [(64, 96), (96, 64), (32, 128)]
    rng = np.random.default_rng(7)
    patterns = []
    for r, c in shapes:
        # unequal +-1 counts on both sides, so that the all-ones start of the
        # power iteration is not orthogonal to the pattern on either side
        a = np.where(rng.random(r) < 0.7, 1.0, -1.0)
        b = np.where(rng.random(c) < 0.3, 1.0, -1.0)
        assert a.sum() != 0 and b.sum() != 0
        patterns.append(np.outer(a, b))
    g = np.concatenate([p.ravel() for p in patterns]).astype(np.float32)
    d = g.size
    flags = smo.SIGNMUON_NORMALIZED_SIGN | (smo.SIGNMUON_NS_FP32 if precision == "fp32" else 0)
    h = smo.SignMuon(shapes, M, beta=0.5, lam=0.0, K=5, eps=eps, scale="spectral", P=1, flags=flags)
    W = torch.zeros(d, device="cuda")
    h.step(W, [dev(g) for _ in range(M)], 0.25)
    Dg = torch.zeros(d, device="cuda")
    h.get_direction(Dg)
    D = host(Dg).astype(np.float64)
    off = 0
    for (r, c), p in zip(shapes, patterns):
        want = p / (np.sqrt(r * c) + eps)
        got = D[off: off + r * c].reshape(r, c)
        assert np.max(np.abs(got - want)) <= 1e-5 * np.max(np.abs(want)), f"rank-one {r}x{c}"
        off += r * c

    shapes = [(48, 48), (32, 80), (80, 32)]
    perms = []
    for r, c in shapes:
        k = min(r, c)
        p = np.zeros((r, c))
        idx = rng.permutation(max(r, c))[:k]
        sg = np.where(rng.random(k) < 0.5, 1.0, -1.0)
        for i in range(k):
            if r <= c:
                p[i, idx[i]] = sg[i]
            else:
                p[idx[i], i] = sg[i]
        perms.append(p)
    g = np.concatenate([p.ravel() for p in perms]).astype(np.float32)
    d = g.size
    h = smo.SignMuon(shapes, M, beta=0.5, lam=0.0, K=5, eps=eps, scale="spectral", P=2,
                     flags=flags | smo.SIGNMUON_TERNARY)
    W = torch.zeros(d, device="cuda")
    h.step(W, [dev(g) for _ in range(M)], 0.25)
    Dg = torch.zeros(d, device="cuda")
    h.get_direction(Dg)
    D = host(Dg).astype(np.float64)
    off = 0
    for (r, c), p in zip(shapes, perms):
        got = D[off: off + r * c].reshape(r, c)
        assert np.array_equal(got == 0, p == 0), f"permutation {r}x{c}: zeros moved"
        assert np.max(np.abs(got - p / (1.0 + eps))) <= 1e-5, f"permutation {r}x{c}"
        off += r * c


@pytest.mark.parametrize("post_polar", [False, True])
def test_ternary_signs_in_gemm_match_kept_polar(post_polar):
    """On the bf16 path the int8 ternary signs come out of the last
    Newton-Schulz GEMM's epilogue, and U is written only with
    SIGNMUON_KEEP_POLAR.  Two handles, one keeping U, run the same step:
    their signs, directions and W must be identical, the signs must be
    sign(U) of the kept U (0 for an exact zero), and get_polar of the handle
    that kept nothing must refuse.  Ragged shapes: rows whose 32-column
    chunks start at unaligned flat offsets take the bytewise stores."""
    shapes = [(3, 5), (130, 70), (64, 147), (96, 300), (256, 512)]
    M, seed = 4, 83
    base = smo.SIGNMUON_TERNARY | (smo.SIGNMUON_POST_POLAR if post_polar else 0)
    d = synth.numel(shapes)
    w0 = synth.weights0(shapes, seed)
    mom0 = synth.momentum0(shapes, M, seed, scale=0.5)
    G = synth.gradients(shapes, M, 1.0, step=1, config_id=seed)
    out = {}
    for keep in (True, False):
        h = smo.SignMuon(shapes, M, beta=HP["beta"], lam=HP["lam"], K=5, eps=HP["eps"], scale="spectral", P=2,
                         flags=base | (smo.SIGNMUON_KEEP_POLAR if keep else 0))
        for m in range(M):
            h.set_momentum(m, dev(mom0[m]))
        W = dev(w0)
        h.step(W, [dev(g) for g in G], HP["eta"])
        t = []
        for m in range(M):
            s = torch.full((d,), 7, dtype=torch.int8, device="cuda")
            h.get_ternary_signs(m, s)
            t.append(host(s))
        D = torch.zeros(d, device="cuda")
        h.get_direction(D)
        U = []
        if keep:
            for m in range(M):
                x = torch.zeros(d, device="cuda")
                h.get_polar(m, x)
                U.append(host(x))
        else:
            with pytest.raises(smo.SignMuonError):
                h.get_polar(0, torch.zeros(d, device="cuda"))
        out[keep] = dict(t=t, D=host(D), W=host(W), U=U)
    for m in range(M):
        assert np.array_equal(out[True]["t"][m], out[False]["t"][m])
        assert np.array_equal(out[True]["t"][m], np.sign(out[True]["U"][m]).astype(np.int8))
    assert np.array_equal(out[True]["D"].view(np.uint32), out[False]["D"].view(np.uint32))
    assert np.array_equal(out[True]["W"].view(np.uint32), out[False]["W"].view(np.uint32))


@pytest.mark.parametrize("case", ["quintic-ternary", "quintic-ragged", "gram-ternary", "tieplus-ternary-post"])
def test_epilogue_signs_across_flag_combinations(case):
    """The signs written by the last GEMM's epilogue under flag combinations:
    quintic with the ternary wire, quintic with one-bit signs of ragged
    column counts, the Gram-space iteration with the ternary wire, and tie to
    +1 with the ternary wire and the post-vote polar step.  A handle that
    keeps U and one that does not run the same step: their signs, directions
    and W must be identical, and the signs must be those of the kept U (the
    one-bit bit = U >= 0, the ternary sign(U)); the kept U must be the
    oracle's polar factor within the bf16 tolerance."""
    flags = {"quintic-ternary": smo.SIGNMUON_NS_QUINTIC | smo.SIGNMUON_TERNARY,
             "quintic-ragged": smo.SIGNMUON_NS_QUINTIC,
             "gram-ternary": smo.SIGNMUON_NS_GRAM | smo.SIGNMUON_TERNARY,
             "tieplus-ternary-post": smo.SIGNMUON_TIE_PLUS | smo.SIGNMUON_TERNARY | smo.SIGNMUON_POST_POLAR}[case]
    shapes = ([(300, 1000), (3072, 768), (520, 1600)] if case.startswith("gram")
              else [(3, 5), (130, 70), (64, 147), (96, 300), (256, 512)])
    order = "quintic" if case.startswith("quintic") else "cubic"
    ternary = bool(flags & smo.SIGNMUON_TERNARY)
    M, seed = 4, 97
    if case.startswith("gram"):
        assert smo.signmuon_plan_tables(shapes, M, 5, "spectral", 2, flags)["gram_ns"] == 1
    d = synth.numel(shapes)
    w0 = synth.weights0(shapes, seed)
    mom0 = synth.momentum0(shapes, M, seed, scale=0.5)
    G = synth.gradients(shapes, M, 1.0, step=1, config_id=seed)
    out = {}
    for keep in (True, False):
        h = smo.SignMuon(shapes, M, beta=HP["beta"], lam=HP["lam"], K=5, eps=HP["eps"], scale="spectral", P=2,
                         flags=flags | (smo.SIGNMUON_KEEP_POLAR if keep else 0))
        for m in range(M):
            h.set_momentum(m, dev(mom0[m]))
        W = dev(w0)
        h.step(W, [dev(g) for g in G], HP["eta"])
        sg, U, mom = [], [], []
        for m in range(M):
            if ternary:
                s = torch.full((d,), 7, dtype=torch.int8, device="cuda")
                h.get_ternary_signs(m, s)
            else:
                s = torch.zeros(ref.packed_nbytes(d), dtype=torch.uint8, device="cuda")
                h.get_signs(m, s)
            sg.append(host(s))
            if keep:
                x = torch.zeros(d, device="cuda")
                h.get_polar(m, x)
                U.append(host(x))
                y = torch.zeros(d, device="cuda")
                h.get_momentum(m, y)
                mom.append(host(y))
        D = torch.zeros(d, device="cuda")
        h.get_direction(D)
        out[keep] = dict(s=sg, U=U, mom=mom, D=host(D), W=host(W))
    for m in range(M):
        assert np.array_equal(out[True]["s"][m], out[False]["s"][m])
        u = out[True]["U"][m]
        if ternary:
            assert np.array_equal(out[True]["s"][m], np.sign(u).astype(np.int8))
        else:
            want = np.packbits(u >= 0, bitorder="little")
            assert np.array_equal(out[True]["s"][m][: want.size], want)
        teacher = oracle_polar_flat(out[True]["mom"][m].astype(np.float64), shapes, 5, HP["eps"], "spectral", 2,
                                    order)
        assert_polar_close(u, teacher, "bf16", f"{case} worker {m}")
    assert np.array_equal(out[True]["D"].view(np.uint32), out[False]["D"].view(np.uint32))
    assert np.array_equal(out[True]["W"].view(np.uint32), out[False]["W"].view(np.uint32))
