"""GPU parity of the whole Sign-Muon step (signmuon_step through the C ABI).

The oracle runs the same step independently from the same seeded state (W0,
momentum, gradients).  Momentum and U are compared with tolerances; the packed
signs may differ only on entries whose |U| is within the precision's noise
(counted by the 1e-3 sign-disagreement bar); wherever every worker's sign
agrees the majority must be identical, and wherever D agrees W must be
bit-exact.
"""
import numpy as np
import pytest

import synth
from oracle import signmuon_ref as ref

from gpu_helpers import assert_momentum_close, assert_polar_close, dev, host

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import sign_muon_optimizer_b200 as smo  # noqa: E402

HP = dict(beta=0.9, lam=0.01, eta=0.02, eps=1e-7)


def _flags(precision, post_polar=False, order="cubic"):
    # these tests read U back, so the step keeps it
    f = (smo.SIGNMUON_NS_FP32 if precision == "fp32" else 0) | smo.SIGNMUON_KEEP_POLAR
    if post_polar:
        f |= smo.SIGNMUON_POST_POLAR
    if order == "quintic":
        f |= smo.SIGNMUON_NS_QUINTIC
    return f


def _run_one_step(shapes, M, sigma, K, scale, P, precision, post_polar, seed, order="cubic", extra_flags=0,
                  tie=0):
    h = smo.SignMuon(shapes, M, beta=HP["beta"], lam=HP["lam"], K=K, eps=HP["eps"], scale=scale, P=P,
                     flags=_flags(precision, post_polar, order) | extra_flags)
    d = h.d
    w0 = synth.weights0(shapes, seed)
    mom0 = synth.momentum0(shapes, M, seed, scale=0.5)
    G = synth.gradients(shapes, M, sigma, step=1, config_id=seed)
    for m in range(M):
        h.set_momentum(m, dev(mom0[m]))
    W = dev(w0)
    h.step(W, [dev(g) for g in G], HP["eta"])
    gpu = dict(W=host(W), mom=[], U=[], bits=[])
    for m in range(M):
        t = torch.zeros(d, device="cuda")
        h.get_momentum(m, t)
        gpu["mom"].append(host(t))
        t = torch.zeros(d, device="cuda")
        h.get_polar(m, t)
        gpu["U"].append(host(t))
        b = torch.zeros(ref.packed_nbytes(d), dtype=torch.uint8, device="cuda")
        h.get_signs(m, b)
        gpu["bits"].append(host(b))
    D = torch.zeros(d, device="cuda")
    h.get_direction(D)
    gpu["D"] = host(D)
    gpu["scales"] = h.get_scales()
    want = ref.step(w0, G, mom0, shapes, beta=HP["beta"], lam=HP["lam"], eta=HP["eta"], K=K, eps=HP["eps"],
                    scale=scale, P=P, order=order, post_polar=post_polar, tie=tie)
    want.update(mom0=mom0, G=G, w0=w0, K=K, scale=scale, P=P, order=order)
    return h, gpu, want


def _np_bits(packed, d):
    return np.unpackbits(np.asarray(packed, np.uint8), bitorder="little")[:d].astype(bool)


def _np_majority(packed_list, d, tie=0):
    s = np.zeros(d, np.int64)
    for p in packed_list:
        s += 2 * _np_bits(p, d).astype(np.int64) - 1
    maj = np.sign(s).astype(np.int8)
    if tie == 1:
        maj[s == 0] = 1
    return maj


def _compare_step(shapes, M, gpu, want, precision, post_polar, tie=0):
    d = synth.numel(shapes)
    for m in range(M):
        assert_momentum_close(gpu["mom"][m], want["mom0"][m], want["G"][m], want["w0"], HP["beta"], HP["lam"])
        assert_polar_close(gpu["U"][m], want["U"][m], precision, f"U worker {m}")
    # the GPU's packed signs are exactly the signs of its own U (numpy check)
    for m in range(M):
        assert np.array_equal(gpu["bits"][m], np.packbits(gpu["U"][m] >= 0, bitorder="little"))
    # wherever every worker's sign agrees with the oracle's, the vote agrees exactly
    agree = np.ones(d, bool)
    for m in range(M):
        agree &= _np_bits(gpu["bits"][m], d) == _np_bits(want["packed"][m], d)
    gpu_maj = _np_majority(gpu["bits"], d, tie)
    assert np.array_equal(gpu_maj[agree], want["majority"][agree])
    assert (~agree).mean() <= M * 1e-3
    if not post_polar:
        assert np.array_equal(gpu["D"], gpu_maj.astype(np.float32))
        same = gpu["D"] == want["D32"]
        assert np.array_equal(gpu["W"][same].view(np.uint32), want["W"][same].view(np.uint32))
        assert (~same).mean() <= M * 1e-3
    else:
        off = 0
        compared = 0
        for r, c in shapes:
            sl = slice(off, off + r * c)
            # every matrix: D is the PolarNS of the GPU's own majority
            teacher = ref.polar_ns(gpu_maj[sl].reshape(r, c).astype(np.float64), want["K"], HP["eps"],
                                   want["scale"], want["P"], want["order"]).ravel()
            assert_polar_close(gpu["D"][sl], teacher, precision, f"post-polar D of the GPU majority {r}x{c}")
            if np.array_equal(gpu_maj[sl], want["majority"][sl]):
                assert_polar_close(gpu["D"][sl], want["D"][sl], precision, f"post-polar D {r}x{c}")
                tol = HP["eta"] * (2e-2 if precision == "bf16" else 1e-4) + 1e-6
                assert np.max(np.abs(gpu["W"][sl] - want["W"][sl])) <= tol
                compared += 1
            off += r * c
        assert compared >= 1


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_step_small_256x128_single(precision):
    shapes = synth.SMALL_256x128_SHAPES
    h, gpu, want = _run_one_step(shapes, 3, 0.5, 5, "fro", 1, precision, False, seed=1)
    _compare_step(shapes, 3, gpu, want, precision, False)


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
@pytest.mark.parametrize("scale,P", [("fro", 1), ("spectral", 2)])
def test_step_ragged_post_polar(precision, scale, P):
    shapes = [(3, 5), (130, 70), (64, 147), (96, 300)]
    M = 4  # even: ties occur and must map to zero
    h, gpu, want = _run_one_step(shapes, M, 1.0, 5, scale, P, precision, True, seed=3)
    _compare_step(shapes, M, gpu, want, precision, True)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 9, 15, 16])
def test_step_post_polar_streamed_stage(M):
    """Shapes whose matrices start at multiples of 128 entries and have a
    multiple of 8 columns: the majority is staged into the post-vote input by
    the streaming vote kernels, one warp per chunk -- bit-sliced counters up
    to 15 workers (M = 15 the largest), byte counters from 16.  Ragged chunks
    (512 and 64 entries, the last below one lane's 128), odd and even M, and
    a second batch of workers (M >= 9)."""
    shapes = [(136, 64), (64, 200), (128, 128), (96, 136), (8, 8)]
    h, gpu, want = _run_one_step(shapes, M, 1.0, 5, "spectral", 2, "bf16", True, seed=37)
    _compare_step(shapes, M, gpu, want, "bf16", True)


@pytest.mark.parametrize("M", [1, 2])
@pytest.mark.parametrize("post_polar", [False, True])
def test_step_one_and_two_workers(M, post_polar):
    """The vote's two smallest cases: one worker (the majority is its own
    sign, no tie possible) and two (every disagreement is a tie and maps to
    zero), with and without the post-vote polar step.  With so few workers
    no other vote hides a sign that rounding flipped, so the comparison runs
    on the fp32 path, where the majority of a whole matrix can match the
    oracle's exactly (the post-vote check needs one such matrix)."""
    shapes = [(130, 70), (64, 147), (96, 300), (8, 8)]
    h, gpu, want = _run_one_step(shapes, M, 1.0, 5, "spectral", 2, "fp32", post_polar, seed=61 + M)
    _compare_step(shapes, M, gpu, want, "fp32", post_polar)


@pytest.mark.parametrize("M", [4, 7])
def test_step_post_polar_streamed_stage_tie_plus(M):
    """The bit-sliced staging with ties to +1 (its threshold moves from
    floor(M/2) + 1 to ceil(M/2)): even M, where ties occur, and odd M."""
    shapes = [(136, 64), (64, 200), (128, 128), (8, 8)]
    h, gpu, want = _run_one_step(shapes, M, 1.0, 5, "spectral", 2, "bf16", True, seed=43,
                                 extra_flags=smo.SIGNMUON_TIE_PLUS, tie=1)
    _compare_step(shapes, M, gpu, want, "bf16", True, tie=1)


def test_step_quintic_fp32():
    shapes = [(64, 96), (96, 64)]
    h, gpu, want = _run_one_step(shapes, 2, 1.0, 3, "spectral", 2, "fp32", False, seed=5, order="quintic")
    _compare_step(shapes, 2, gpu, want, "fp32", False)


def test_step_small_256x128_ten_steps_drift():
    """The small 256x128 workload end to end: 10 steps on the GPU (fp32 NS) and in the oracle,
    each from its own state; the trajectories may part only where a sign was
    within rounding of zero."""
    shapes = synth.SMALL_256x128_SHAPES
    M = 3
    h = smo.SignMuon(shapes, M, beta=HP["beta"], lam=HP["lam"], K=5, eps=HP["eps"], scale="fro",
                     flags=smo.SIGNMUON_NS_FP32)
    w0 = synth.weights0(shapes, 0)
    W = dev(w0)
    w_ref = w0.copy()
    mom_ref = [np.zeros(h.d)] * M
    for t in range(10):
        G = synth.gradients(shapes, M, 0.5, step=t, config_id=0)
        h.step(W, [dev(g) for g in G], HP["eta"])
        out = ref.step(w_ref, G, mom_ref, shapes, beta=HP["beta"], lam=HP["lam"], eta=HP["eta"], K=5,
                       eps=HP["eps"], scale="fro")
        w_ref, mom_ref = out["W"], out["mom"]
    w_gpu = host(W)
    differ = w_gpu != w_ref
    assert differ.mean() <= 1e-2, f"{differ.sum()} of {w_gpu.size} weights differ after 10 steps"
    assert np.max(np.abs(w_gpu - w_ref)) <= 2 * HP["eta"] * 10 + 1e-6


def test_nonfinite_gradient_keeps_w():
    shapes = [(64, 96)]
    h = smo.SignMuon(shapes, 2, K=2, scale="fro")
    w0 = synth.weights0(shapes, 9)
    G = synth.gradients(shapes, 2, 1.0, step=0, config_id=9)
    G[1][17] = np.nan
    W = dev(w0)
    with pytest.raises(smo.SignMuonError) as e:
        h.step(W, [dev(g) for g in G], 0.02)
    assert e.value.status == smo.SIGNMUON_E_NONFINITE
    assert np.array_equal(host(W).view(np.uint32), w0.view(np.uint32))


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_checkpoint_resume_bit_exact(precision):
    shapes = [(128, 256), (300, 64)]
    M = 3
    kw = dict(beta=0.9, lam=0.01, K=5, eps=1e-7, scale="spectral", P=2, flags=_flags(precision))
    w0 = synth.weights0(shapes, 4)
    grads = [synth.gradients(shapes, M, 1.0, step=t, config_id=4) for t in range(10)]
    a = smo.SignMuon(shapes, M, **kw)
    Wa = dev(w0)
    for t in range(10):
        a.step(Wa, [dev(g) for g in grads[t]], 0.02)
    b = smo.SignMuon(shapes, M, **kw)
    Wb = dev(w0)
    for t in range(5):
        b.step(Wb, [dev(g) for g in grads[t]], 0.02)
    saved = []
    for m in range(M):
        s = torch.zeros(b.d, device="cuda")
        b.get_momentum(m, s)
        saved.append(s)
    b.close()
    c = smo.SignMuon(shapes, M, **kw)
    for m in range(M):
        c.set_momentum(m, saved[m])
    for t in range(5, 10):
        c.step(Wb, [dev(g) for g in grads[t]], 0.02)
    assert np.array_equal(host(Wa).view(np.uint32), host(Wb).view(np.uint32))
    for m in range(M):
        x = torch.zeros(a.d, device="cuda")
        y = torch.zeros(a.d, device="cuda")
        a.get_momentum(m, x)
        c.get_momentum(m, y)
        assert torch.equal(x, y)


def test_step_host_matches_device_step():
    shapes = [(128, 256)]
    M = 2
    w0 = synth.weights0(shapes, 6)
    G = synth.gradients(shapes, M, 1.0, step=0, config_id=6)
    a = smo.SignMuon(shapes, M, K=3, scale="fro")
    W = dev(w0)
    a.step(W, [dev(g) for g in G], 0.02)
    b = smo.SignMuon(shapes, M, K=3, scale="fro")
    wh = w0.copy()
    b.step_host(wh, G, 0.02)
    assert np.array_equal(wh.view(np.uint32), host(W).view(np.uint32))


@pytest.mark.parametrize("pinned", [True, False])
def test_step_host_async_pipeline_matches_device_steps(pinned):
    """SIGNMUON_ASYNC step_host calls queued back to back (each call's
    gradients come in on the copy stream, alternating between two device
    sets, while the step before runs): after one sync, W and the momenta are
    bit-identical to the same steps on device buffers, for gradients that
    differ from call to call and one W host buffer shared by all calls."""
    shapes = [(256, 512), (96, 160), (130, 70)]
    M, T = 3, 5
    w0 = synth.weights0(shapes, 41)
    grads = [synth.gradients(shapes, M, 1.0, step=t, config_id=41) for t in range(T)]
    kw = dict(beta=HP["beta"], lam=HP["lam"], K=3, eps=HP["eps"], scale="spectral", P=2,
              flags=smo.SIGNMUON_POST_POLAR)
    a = smo.SignMuon(shapes, M, **kw)
    W = dev(w0)
    for t in range(T):
        a.step(W, [dev(g) for g in grads[t]], 0.02)
    b = smo.SignMuon(shapes, M, **dict(kw, flags=kw["flags"] | smo.SIGNMUON_ASYNC))
    if pinned:
        wt = torch.from_numpy(w0.copy()).pin_memory()
        gts = [[torch.from_numpy(g).pin_memory() for g in grads[t]] for t in range(T)]
        wh, gh = wt.numpy(), [[g.numpy() for g in gt] for gt in gts]
    else:
        wh, gh = w0.copy(), [[g.copy() for g in grads[t]] for t in range(T)]
    for t in range(T):
        b.step_host(wh, gh[t], 0.02)
    b.sync()
    assert np.array_equal(wh.view(np.uint32), host(W).view(np.uint32))
    for m in range(M):
        x = torch.zeros(a.d, device="cuda")
        y = torch.zeros(a.d, device="cuda")
        a.get_momentum(m, x)
        b.get_momentum(m, y)
        assert torch.equal(x, y)


@pytest.mark.parametrize("ragged", [False, True, "gram"])
@pytest.mark.parametrize("post_polar", [False, True])
def test_signs_packed_in_gemm_match_kept_polar(post_polar, ragged):
    """The bf16 step packs the one-bit signs in the last Newton-Schulz GEMM;
    without SIGNMUON_KEEP_POLAR it writes no U.  With every column count a
    multiple of 32 each 32-column chunk is one word of the bit stream; with
    ragged column counts chunks straddle words and OR their bits into both.
    Both handles run the same step: the packed signs, the direction and W
    must be identical, the signs must be U >= 0 of the kept U, and get_polar
    of the handle that kept nothing must refuse."""
    if ragged == "gram":
        # SIGNMUON_NS_GRAM: the final product X_K = Q_K X0 packs the signs
        # (1000 columns: ragged chunks)
        shapes = [(300, 1000), (3072, 768), (520, 1600)]
    elif ragged:
        shapes = [(3, 5), (130, 70), (64, 147), (96, 300), (256, 512), (33, 31)]
    else:
        shapes = [(256, 512), (512, 256), (96, 160), (384, 384)]
    M, seed = 4, 23
    base = (smo.SIGNMUON_POST_POLAR if post_polar else 0) | (smo.SIGNMUON_NS_GRAM if ragged == "gram" else 0)
    if ragged == "gram":
        assert smo.signmuon_plan_tables(shapes, M, 5, "spectral", 2, base)["gram_ns"] == 1
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
        bits = []
        for m in range(M):
            b = torch.zeros(ref.packed_nbytes(d), dtype=torch.uint8, device="cuda")
            h.get_signs(m, b)
            bits.append(host(b))
        Dg = torch.zeros(d, device="cuda")
        h.get_direction(Dg)
        U = []
        if keep:
            for m in range(M):
                t = torch.zeros(d, device="cuda")
                h.get_polar(m, t)
                U.append(host(t))
        else:
            t = torch.zeros(d, device="cuda")
            with pytest.raises(smo.SignMuonError) as ei:
                h.get_polar(0, t)
            assert ei.value.status == 7
        out[keep] = dict(W=host(W), bits=bits, D=host(Dg), U=U)
        h.close()
    for m in range(M):
        assert np.array_equal(out[True]["bits"][m], out[False]["bits"][m])
        want = np.packbits(out[True]["U"][m] >= 0, bitorder="little")
        assert np.array_equal(out[True]["bits"][m][: want.size], want)
    assert np.array_equal(out[True]["D"], out[False]["D"])
    assert np.array_equal(out[True]["W"].view(np.uint32), out[False]["W"].view(np.uint32))


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
@pytest.mark.parametrize("post_polar", [False, True])
def test_step_tie_plus(precision, post_polar):
    """Named variant: a tied vote gives +1 ([paper] Algorithm 2's default);
    M = 4 so that ties occur.  With ties this frequent a sign within rounding
    of zero flips a large matrix's majority somewhere, so the post-vote polar
    factor is compared on the small matrices, whose majorities match."""
    shapes = [(3, 5), (8, 16), (64, 96), (130, 70)]
    M = 4
    h, gpu, want = _run_one_step(shapes, M, 1.0, 5, "spectral", 2, precision, post_polar, seed=31,
                                 extra_flags=smo.SIGNMUON_TIE_PLUS, tie=1)
    assert (want["sums"] == 0).any()
    _compare_step(shapes, M, gpu, want, precision, post_polar, tie=1)


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_step_polar_after_only(precision):
    """Named variant: the signs of the momentum itself, orthogonalised only
    after the vote ([paper] §4 placement)."""
    shapes = [(64, 96), (130, 70), (96, 64)]
    M, seed = 3, 37
    d = synth.numel(shapes)
    w0 = synth.weights0(shapes, seed)
    mom0 = synth.momentum0(shapes, M, seed, scale=0.5)
    G = synth.gradients(shapes, M, 1.0, step=1, config_id=seed)
    h = smo.SignMuon(shapes, M, beta=HP["beta"], lam=HP["lam"], K=5, eps=HP["eps"], scale="spectral", P=2,
                     flags=_flags(precision, True) | smo.SIGNMUON_POLAR_AFTER_ONLY)
    for m in range(M):
        h.set_momentum(m, dev(mom0[m]))
    W = dev(w0)
    h.step(W, [dev(g) for g in G], HP["eta"])
    want = ref.step(w0, G, mom0, shapes, beta=HP["beta"], lam=HP["lam"], eta=HP["eta"], K=5, eps=HP["eps"],
                    scale="spectral", P=2, post_polar=True, pre_polar=False)
    agree = np.ones(d, bool)
    bits = []
    for m in range(M):
        t = torch.zeros(d, device="cuda")
        h.get_momentum(m, t)
        mom = host(t)
        assert_momentum_close(mom, mom0[m], G[m], w0, HP["beta"], HP["lam"])
        b = torch.zeros(ref.packed_nbytes(d), dtype=torch.uint8, device="cuda")
        h.get_signs(m, b)
        bits.append(host(b))
        # the packed signs are exactly those of the GPU's own momentum
        assert np.array_equal(bits[m], np.packbits(mom >= 0, bitorder="little"))
        agree &= _np_bits(bits[m], d) == _np_bits(want["packed"][m], d)
    with pytest.raises(smo.SignMuonError) as ei:
        h.get_polar(0, torch.zeros(d, device="cuda"))
    assert ei.value.status == smo.SIGNMUON_E_UNSUPPORTED
    assert (~agree).mean() <= M * 1e-4
    gpu_maj = _np_majority(bits, d)
    assert np.array_equal(gpu_maj[agree], want["majority"][agree])
    Dg = torch.zeros(d, device="cuda")
    h.get_direction(Dg)
    D, Wn = host(Dg), host(W)
    off = 0
    compared = 0
    for r, c in shapes:
        sl = slice(off, off + r * c)
        if np.array_equal(gpu_maj[sl], want["majority"][sl]):
            assert_polar_close(D[sl], want["D"][sl], precision, f"after-only D {r}x{c}")
            compared += 1
        off += r * c
    assert compared >= 1
    # W is the single-rounding update with the GPU's own D
    assert np.array_equal(Wn.view(np.uint32), ref.update(w0, D, HP["eta"]).view(np.uint32))


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
@pytest.mark.parametrize("K", [0, 5])
def test_step_muon_mean(precision, K):
    """Muon baseline on the same kernels: D = PolarNS(mean momentum)."""
    shapes = [(64, 96), (130, 70), (96, 64)]
    M, seed = 3, 41
    d = synth.numel(shapes)
    w0 = synth.weights0(shapes, seed)
    mom0 = synth.momentum0(shapes, M, seed, scale=0.5)
    G = synth.gradients(shapes, M, 1.0, step=1, config_id=seed)
    h = smo.SignMuon(shapes, M, beta=HP["beta"], lam=HP["lam"], K=K, eps=HP["eps"], scale="spectral", P=2,
                     flags=_flags(precision) | smo.SIGNMUON_MUON_MEAN)
    for m in range(M):
        h.set_momentum(m, dev(mom0[m]))
    W = dev(w0)
    h.step(W, [dev(g) for g in G], HP["eta"])
    want = ref.muon_step(w0, G, mom0, shapes, beta=HP["beta"], lam=HP["lam"], eta=HP["eta"], K=K, eps=HP["eps"],
                         scale="spectral", P=2)
    Dg = torch.zeros(d, device="cuda")
    h.get_direction(Dg)
    D = host(Dg)
    assert_polar_close(D, want["D"], precision, "Muon D")
    assert np.array_equal(host(W).view(np.uint32), ref.update(w0, D, HP["eta"]).view(np.uint32))
    with pytest.raises(smo.SignMuonError) as ei:
        h.get_signs(0, torch.zeros(ref.packed_nbytes(d), dtype=torch.uint8, device="cuda"))
    assert ei.value.status == smo.SIGNMUON_E_UNSUPPORTED


def test_async_step_matches_sync_and_defers_errors():
    """SIGNMUON_ASYNC: the step returns without waiting and gives the same W
    bit for bit; a non-finite gradient is reported by signmuon_sync (and
    cleared by it), with W left untouched."""
    shapes = [(64, 96), (96, 64)]
    M, seed = 2, 51
    w0 = synth.weights0(shapes, seed)
    mom0 = synth.momentum0(shapes, M, seed, scale=0.5)
    G = synth.gradients(shapes, M, 1.0, step=1, config_id=seed)
    out = []
    for flags in (0, smo.SIGNMUON_ASYNC):
        h = smo.SignMuon(shapes, M, beta=HP["beta"], lam=HP["lam"], K=5, eps=HP["eps"], scale="spectral", P=2,
                         flags=flags)
        for m in range(M):
            h.set_momentum(m, dev(mom0[m]))
        W = dev(w0)
        h.step(W, [dev(g) for g in G], HP["eta"])
        h.sync()
        out.append((h, host(W)))
    assert np.array_equal(out[0][1].view(np.uint32), out[1][1].view(np.uint32))
    ha = out[1][0]
    bad = [g.copy() for g in G]
    bad[0][5] = np.nan
    W2 = dev(w0)
    ha.step(W2, [dev(g) for g in bad], HP["eta"])   # no wait, no error yet
    with pytest.raises(smo.SignMuonError) as ei:
        ha.sync()
    assert ei.value.status == smo.SIGNMUON_E_NONFINITE
    assert np.array_equal(host(W2).view(np.uint32), w0.view(np.uint32))
    ha.sync()  # the deferred error was cleared


def test_profile_info_and_launch_counter():
    """signmuon_profile / profile_read time every kernel kind of a step;
    signmuon_kernel_launches counts the launches; signmuon_info reports the
    handle's sizes."""
    shapes = [(64, 96), (96, 64), (130, 70)]
    M = 3
    h = smo.SignMuon(shapes, M, beta=HP["beta"], lam=HP["lam"], K=5, eps=HP["eps"], scale="spectral", P=2,
                     flags=smo.SIGNMUON_POST_POLAR)
    d = h.d
    info = smo.signmuon_info(h.h)
    assert info["d"] == d == synth.numel(shapes)
    assert info["packed_bytes"] == ref.packed_nbytes(d)
    assert info["M"] == M and info["n_mats"] == len(shapes) and info["groups"] == 3
    assert info["device_bytes"] > 0
    W = dev(synth.weights0(shapes, 3))
    G = [dev(g) for g in synth.gradients(shapes, M, 1.0, step=1, config_id=3)]
    h.step(W, G, HP["eta"])
    h.profile(True)
    h.profile_read()
    n0 = smo.signmuon_kernel_launches()
    h.step(W, G, HP["eta"])
    prof = h.profile_read()
    h.profile(False)
    n1 = smo.signmuon_kernel_launches()
    want = dict(momentum=1, norm_finalize=2, ns_gram=5, ns_apply=5, power_iter=2, vote=1, post_gram=5,
                post_apply=5, update=1)
    for kind, n in want.items():
        ms, cnt = prof[kind]
        assert cnt == n, (kind, cnt)
        assert ms > 0.0, kind
    assert n1 - n0 >= sum(want.values())


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
@pytest.mark.parametrize("post_polar", [False, True])
def test_step_zero_gradients_degenerate(precision, post_polar):
    """The degenerate case: zero weights, gradients and momentum.  The scale
    is 0, X0 = 0/(0 + eps) = 0, so U = 0 exactly, every one-bit sign is +1
    (reading R5), the majority is +1 and, without the post-vote polar step,
    W moves to -eta exactly; with it D is the polar factor of the all-ones
    matrix (its own rank-one direction)."""
    shapes = [(64, 96), (96, 64)]
    M = 3
    d = synth.numel(shapes)
    h = smo.SignMuon(shapes, M, beta=HP["beta"], lam=HP["lam"], K=5, eps=HP["eps"], scale="spectral", P=2,
                     flags=_flags(precision, post_polar))
    W = torch.zeros(d, device="cuda")
    h.step(W, [torch.zeros(d, device="cuda") for _ in range(M)], HP["eta"])
    z = np.zeros(d, np.float32)
    want = ref.step(z, [z] * M, [z] * M, shapes, beta=HP["beta"], lam=HP["lam"], eta=HP["eta"], K=5, eps=HP["eps"],
                    scale="spectral", P=2, post_polar=post_polar)
    for m in range(M):
        t = torch.ones(d, device="cuda")
        h.get_polar(m, t)
        assert not host(t).any()
        b = torch.zeros(ref.packed_nbytes(d), dtype=torch.uint8, device="cuda")
        h.get_signs(m, b)
        assert np.array_equal(host(b), want["packed"][m])
    Dg = torch.zeros(d, device="cuda")
    h.get_direction(Dg)
    D = host(Dg)
    if post_polar:
        assert_polar_close(D, want["D"], precision, "polar factor of the all-ones majority")
        assert np.array_equal(host(W).view(np.uint32), ref.update(z, D, HP["eta"]).view(np.uint32))
    else:
        assert np.array_equal(D, np.ones(d, np.float32))
        assert np.array_equal(host(W).view(np.uint32), want["W"].view(np.uint32))


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
@pytest.mark.parametrize("scale,P", [("fro", 1), ("spectral", 2)])
def test_step_signsgd_k0(precision, scale, P):
    """The signSGD baseline of the comparison family ([paper] Table 1's
    SignSGD row, §3's sign vote): K = 0 Newton-Schulz iterations, so U is the
    scaled momentum and the vote runs on sign(Mom); no post-vote step.  An
    even M makes ties occur; they must map to 0.  Momentum, U, bits, the vote
    on agreed entries and W where D agrees, as for the other steps."""
    shapes = [(3, 5), (130, 70), (64, 147), (96, 300)]
    M = 4
    h, gpu, want = _run_one_step(shapes, M, 1.0, 0, scale, P, precision, False, seed=31)
    _compare_step(shapes, M, gpu, want, precision, False)
    d = synth.numel(shapes)
    # with K = 0 the signs are those of the momentum itself (U = Mom / (s + eps))
    for m in range(M):
        mom = np.asarray(gpu["mom"][m])
        assert np.array_equal(_np_bits(gpu["bits"][m], d), mom >= 0)
    # ties occurred and went to 0
    assert (_np_majority(gpu["bits"], d) == 0).any()


def test_step_signsgd_k0_without_kept_polar():
    """K = 0 with the flags a caller of the baseline would use (no
    SIGNMUON_KEEP_POLAR): the packed signs come from the pack kernel of the
    scaled momentum and must equal the signs of the GPU's own momentum bit for
    bit; W moves by the vote of those signs."""
    shapes = [(130, 70), (96, 300), (256, 128)]
    M = 6
    h = smo.SignMuon(shapes, M, beta=HP["beta"], lam=HP["lam"], K=0, eps=HP["eps"], scale="fro", P=1, flags=0)
    d = h.d
    w0 = synth.weights0(shapes, 33)
    mom0 = synth.momentum0(shapes, M, 33, scale=0.5)
    G = synth.gradients(shapes, M, 1.0, step=1, config_id=33)
    for m in range(M):
        h.set_momentum(m, dev(mom0[m]))
    W = dev(w0)
    h.step(W, [dev(g) for g in G], HP["eta"])
    bits, moms = [], []
    for m in range(M):
        t = torch.zeros(d, device="cuda")
        h.get_momentum(m, t)
        moms.append(host(t))
        b = torch.zeros(ref.packed_nbytes(d), dtype=torch.uint8, device="cuda")
        h.get_signs(m, b)
        bits.append(host(b))
        assert np.array_equal(bits[m], ref.pack_bits(ref.sign_bits(moms[m])))
    maj = ref.majority(ref.vote_sums_from_bits(bits, d))
    assert (maj == 0).any()
    want_w = ref.update(w0, maj.astype(np.float32), HP["eta"])
    assert np.array_equal(host(W).view(np.uint32), want_w.view(np.uint32))
    # and the oracle's own step agrees wherever every worker's sign agrees
    want = ref.step(w0, G, mom0, shapes, beta=HP["beta"], lam=HP["lam"], eta=HP["eta"], K=0, eps=HP["eps"],
                    scale="fro", P=1)
    agree = np.ones(d, bool)
    for m in range(M):
        agree &= _np_bits(bits[m], d) == _np_bits(want["packed"][m], d)
    assert np.array_equal(maj[agree], want["majority"][agree])
    assert (~agree).mean() <= M * 1e-3


@pytest.mark.parametrize("post_polar", [True, False])
def test_step_replays_from_a_cuda_graph(post_polar):
    """With SIGNMUON_ASYNC the step makes no host synchronisation and no
    allocation, so it can be captured into a CUDA graph on the handle's
    stream (torch.cuda.graph) and replayed: T replays over static gradient
    buffers refilled before each give W and momenta bit-identical to T eager
    steps."""
    shapes = [(256, 512), (96, 160), (130, 70)]
    M, T = 3, 4
    w0 = synth.weights0(shapes, 47)
    grads = [synth.gradients(shapes, M, 1.0, step=t, config_id=47) for t in range(T)]
    flags = (smo.SIGNMUON_POST_POLAR if post_polar else 0) | smo.SIGNMUON_ASYNC
    kw = dict(beta=HP["beta"], lam=HP["lam"], K=3, eps=HP["eps"], scale="spectral", P=2, flags=flags)
    a = smo.SignMuon(shapes, M, **kw)
    Wa = dev(w0)
    for t in range(T):
        a.step(Wa, [dev(g) for g in grads[t]], 0.02)
    a.sync()
    s = torch.cuda.Stream()
    b = smo.SignMuon(shapes, M, stream=s.cuda_stream, **kw)
    Wb = dev(w0)
    Gs = [torch.zeros(b.d, device="cuda") for _ in range(M)]
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        b.step(Wb, Gs, 0.02)
    for t in range(T):
        with torch.cuda.stream(s):
            for m in range(M):
                Gs[m].copy_(dev(grads[t][m]))
            g.replay()
    s.synchronize()
    b.sync()
    assert np.array_equal(host(Wb).view(np.uint32), host(Wa).view(np.uint32))
    for m in range(M):
        x = torch.zeros(a.d, device="cuda")
        y = torch.zeros(a.d, device="cuda")
        a.get_momentum(m, x)
        b.get_momentum(m, y)
        assert torch.equal(x, y)
    del g
