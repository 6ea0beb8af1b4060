"""Parity at the full workload sizes, in the benchmark's launch configuration.

The oracle cannot run whole steps at these sizes, so each test checks sampled
outputs that the oracle computes one matrix (or one entry) at a time, plus
invariants over the whole output:

* nanoGPT-124M shapes, M=8, bf16, K=5 cubic, spectral P=2, post-vote polar:
  one matrix of every shape (first and last layer): U of every worker, the
  vote where every worker's sign agrees with the oracle's, the post-vote
  polar D and the updated W.
* ResNet-50 shapes, M=4, bf16, spectral P=2: the stem, a 3x3 conv, a
  projection shortcut and the classifier.
* LLaMA-layer vote, d = 717,225,984, M=16: sampled entries bit-exact
  (int32 and int8 sums, majority); range, parity and sign invariants over
  every entry.
* nanoGPT in the benchmark's exact configuration (signs packed inside the
  last GEMM, no U written): packed bits, vote, post-vote D and W on sampled
  matrices of three layers; and the signSGD baseline (K = 0) at full size.
* NS sweep shapes: sampled problems of 64 x 1024^2 and 256 x 512x2048
  against the oracle over the whole grid (K in {5, 10}, cubic and quintic,
  bf16 and fp32), and the M = 8 vote on the sweep's results; one 8192^2
  matrix with a known polar factor (a normalised Sylvester-Hadamard matrix
  times a diagonal times a signed permutation), compared entry by entry over
  the same grid.
Inputs are seeded synthetic data; large ones are drawn on the device by the
synth module (torch Philox) and the sampled parts read back for the oracle.
"""
import math

import numpy as np
import pytest

import synth
from oracle import signmuon_ref as ref

from gpu_helpers import assert_polar_close

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import sign_muon_optimizer_b200 as smo  # noqa: E402

HP = synth.HYPER


def _mat(flat_dev, shapes, i):
    off = synth.flat_offsets(shapes)[i]
    r, c = shapes[i]
    return flat_dev[off: off + r * c].double().cpu().numpy().reshape(r, c)


def _step_sampled(name, sample, post_polar):
    wl = synth.WORKLOADS[name]
    shapes, M = wl["shapes"], wl["M"]
    flags = (smo.SIGNMUON_POST_POLAR if post_polar else 0) | smo.SIGNMUON_KEEP_POLAR
    opt = smo.SignMuon(shapes, M, beta=HP["beta"], lam=HP["lam"], K=wl["K"], eps=HP["eps"], scale=wl["scale"],
                       P=wl["P"], flags=flags)
    W = synth.device_weights0(shapes, config_id=41)
    W0 = W.clone()
    G = synth.device_gradients(shapes, M, wl["sigma"], step=0, config_id=41)
    opt.step(W, [G[m] for m in range(M)], HP["eta"])
    d = opt.d
    U = torch.empty(d, device="cuda")
    Dg = torch.empty(d, device="cuda")
    opt.get_direction(Dg)
    us = []
    for m in range(M):
        opt.get_polar(m, U)
        us.append(U.clone())
    for i in sample:
        r, c = shapes[i]
        w0 = _mat(W0, shapes, i).astype(np.float32)
        u_ref = []
        for m in range(M):
            g = _mat(G[m], shapes, i)
            mom = ref.momentum_update(np.zeros_like(g), g, w0, HP["beta"], HP["lam"])
            u = ref.polar_ns(mom, wl["K"], HP["eps"], wl["scale"], wl["P"])
            u_ref.append(u)
            assert_polar_close(_mat(us[m], shapes, i), u, "bf16", f"{name} matrix {i} ({r}x{c}) worker {m}")
        # the vote: wherever every worker's sign agrees with the oracle's
        ref_bits = [ref.sign_bits(u) for u in u_ref]
        gpu_bits = [_mat(us[m], shapes, i) >= 0 for m in range(M)]
        agree = np.logical_and.reduce([a == b for a, b in zip(ref_bits, gpu_bits)])
        ref_maj = np.sign(sum(2 * b.astype(np.int64) - 1 for b in ref_bits))
        gpu_D = _mat(Dg, shapes, i)
        if not post_polar:
            assert np.array_equal(gpu_D[agree], ref_maj[agree].astype(np.float64))
            w_ref = ref.update(w0.ravel(), ref_maj.ravel().astype(np.float32), HP["eta"]).reshape(r, c)
            w_gpu = _mat(W, shapes, i).astype(np.float32)
            assert np.array_equal(w_gpu[agree].view(np.uint32), w_ref[agree].view(np.uint32))
        else:
            gpu_maj = np.sign(sum(2 * b.astype(np.int64) - 1 for b in gpu_bits))
            assert np.array_equal(gpu_maj[agree], ref_maj[agree])
            # D is a global function of the majority, which legitimately differs
            # on the entries where a worker's sign sat within rounding of zero;
            # the post-vote polar itself is compared in isolation below.  Here:
            # W moved by -eta*D of the GPU's own D (one rounding, numpy bound)
            w_gpu = _mat(W, shapes, i)
            expect = w0.astype(np.float64) - np.float64(np.float32(HP["eta"])) * gpu_D
            assert np.all(np.abs(w_gpu - expect) <= np.spacing(np.abs(expect).astype(np.float32)))
        assert (~agree).mean() <= M * 1e-3


def test_nanogpt_step_full_size_sampled():
    shapes = synth.NANOGPT_SHAPES
    _step_sampled("nanogpt", [0, 1, 2, 3, len(shapes) - 1], post_polar=True)


def _unpack_range(packed_dev, off, n):
    """Bits off .. off+n of a device bit stream (off and n multiples of 8)."""
    assert off % 8 == 0 and n % 8 == 0
    b = packed_dev[off // 8: (off + n) // 8].cpu().numpy()
    return np.unpackbits(b, bitorder="little").astype(bool)


def test_nanogpt_bench_configuration_full_size():
    """The exact configuration the benchmark times: SIGNMUON_POST_POLAR only,
    so the last Newton-Schulz GEMM writes the one-bit signs of its epilogue
    straight into the packed buffers and no U at all (384 problems, M = 8).
    Checked on sampled matrices of three layers against the oracle: every
    worker's packed bits (sign disagreement <= 1e-3 of the entries above the
    magnitude mask), the vote (exact wherever every worker's sign agrees), the
    post-vote polar D against the oracle's PolarNS of the GPU's own majority
    (the teacher-forced global step), and W bit-exact given the GPU's D."""
    wl = synth.WORKLOADS["nanogpt"]
    shapes, M = wl["shapes"], wl["M"]
    opt = smo.SignMuon(shapes, M, beta=HP["beta"], lam=HP["lam"], K=wl["K"], eps=HP["eps"], scale=wl["scale"],
                       P=wl["P"], flags=smo.SIGNMUON_POST_POLAR)
    W = synth.device_weights0(shapes, config_id=43)
    W0 = W.clone()
    G = synth.device_gradients(shapes, M, wl["sigma"], step=0, config_id=43)
    opt.step(W, [G[m] for m in range(M)], HP["eta"])
    d = opt.d
    # no U is kept in this configuration
    with pytest.raises(smo.SignMuonError):
        opt.get_polar(0, torch.empty(d, device="cuda"))
    nb = (d + 7) // 8
    bits = []
    for m in range(M):
        b = torch.zeros(nb, dtype=torch.uint8, device="cuda")
        opt.get_signs(m, b)
        bits.append(b)
    Dg = torch.empty(d, device="cuda")
    opt.get_direction(Dg)
    offs = synth.flat_offsets(shapes)
    sample = [0, 1, 2, 3, 24, 25, 26, 27, len(shapes) - 4, len(shapes) - 3, len(shapes) - 2, len(shapes) - 1]
    for i in sample:
        r, c = shapes[i]
        w0 = _mat(W0, shapes, i).astype(np.float32)
        agree = np.ones(r * c, bool)
        ref_bits, gpu_bits = [], []
        for m in range(M):
            g = _mat(G[m], shapes, i)
            mom = ref.momentum_update(np.zeros_like(g), g, w0, HP["beta"], HP["lam"])
            u = ref.polar_ns(mom, wl["K"], HP["eps"], wl["scale"], wl["P"]).ravel()
            rb = ref.sign_bits(u)
            gb = _unpack_range(bits[m], offs[i], r * c)
            thr = 1e-3 * np.max(np.abs(u))
            dis = int(((rb != gb) & (np.abs(u) > thr)).sum())
            assert dis <= 1e-3 * int((np.abs(u) > thr).sum()), f"matrix {i} worker {m}: {dis} sign disagreements"
            agree &= rb == gb
            ref_bits.append(rb)
            gpu_bits.append(gb)
        ref_maj = np.sign(sum(2 * b.astype(np.int64) - 1 for b in ref_bits))
        gpu_maj = np.sign(sum(2 * b.astype(np.int64) - 1 for b in gpu_bits))
        assert np.array_equal(gpu_maj[agree], ref_maj[agree]), f"matrix {i}: vote differs on agreed entries"
        assert (~agree).mean() <= M * 1e-3
        # the post-vote polar step of the GPU's own majority
        d_ref = ref.polar_ns(gpu_maj.reshape(r, c).astype(np.float64), wl["K"], HP["eps"], wl["scale"], wl["P"])
        d_gpu = _mat(Dg, shapes, i)
        assert_polar_close(d_gpu, d_ref, "bf16", f"post-vote D of matrix {i} ({r}x{c})")
        # W moved by exactly one rounding of -eta * D
        w_ref = ref.update(w0.ravel(), d_gpu.ravel().astype(np.float32), HP["eta"])
        w_gpu = _mat(W, shapes, i).astype(np.float32).ravel()
        assert np.array_equal(w_gpu.view(np.uint32), w_ref.view(np.uint32)), f"matrix {i}: W not bit-exact"
    # over every entry: W = W0 - eta * D to within one float32 rounding
    expect = W0.double() - float(np.float32(HP["eta"])) * Dg.double()
    ulp = torch.abs(expect.float()).double() * 2.0 ** -23
    assert bool((torch.abs(W.double() - expect) <= ulp).all())


def test_nanogpt_signsgd_k0_full_size():
    """The signSGD member of the comparison family at the headline size: K = 0
    (no Newton-Schulz, the one-bit signs of the scaled momentum), no post-vote
    step, M = 8.  Sampled matrices against the oracle: bits where |Mom| is
    above the mask, the vote wherever every worker agrees, and W bit-exact
    wherever the direction agrees."""
    wl = synth.WORKLOADS["nanogpt"]
    shapes, M = wl["shapes"], wl["M"]
    opt = smo.SignMuon(shapes, M, beta=HP["beta"], lam=HP["lam"], K=0, eps=HP["eps"], scale="fro", flags=0)
    W = synth.device_weights0(shapes, config_id=44)
    W0 = W.clone()
    G = synth.device_gradients(shapes, M, wl["sigma"], step=0, config_id=44)
    opt.step(W, [G[m] for m in range(M)], HP["eta"])
    d = opt.d
    nb = (d + 7) // 8
    bits = []
    for m in range(M):
        b = torch.zeros(nb, dtype=torch.uint8, device="cuda")
        opt.get_signs(m, b)
        bits.append(b)
    Dg = torch.empty(d, device="cuda")
    opt.get_direction(Dg)
    offs = synth.flat_offsets(shapes)
    for i in [0, 1, 2, 3, len(shapes) - 1]:
        r, c = shapes[i]
        w0 = _mat(W0, shapes, i).astype(np.float32)
        agree = np.ones(r * c, bool)
        ref_bits, gpu_bits = [], []
        for m in range(M):
            g = _mat(G[m], shapes, i)
            mom = ref.momentum_update(np.zeros_like(g), g, w0, HP["beta"], HP["lam"])
            u = ref.polar_ns(mom, 0, HP["eps"], "fro").ravel()
            rb = ref.sign_bits(u)
            gb = _unpack_range(bits[m], offs[i], r * c)
            thr = 1e-3 * np.max(np.abs(u))
            dis = int(((rb != gb) & (np.abs(u) > thr)).sum())
            assert dis == 0, f"matrix {i} worker {m}: {dis} sign disagreements above the mask"
            agree &= rb == gb
            ref_bits.append(rb)
            gpu_bits.append(gb)
        ref_maj = np.sign(sum(2 * b.astype(np.int64) - 1 for b in ref_bits))
        gpu_maj = np.sign(sum(2 * b.astype(np.int64) - 1 for b in gpu_bits))
        assert np.array_equal(gpu_maj[agree], ref_maj[agree])
        d_gpu = _mat(Dg, shapes, i).ravel()
        assert np.array_equal(d_gpu, gpu_maj.astype(np.float64)), "D is the GPU's own majority"
        w_ref = ref.update(w0.ravel(), ref_maj.astype(np.float32), HP["eta"])
        w_gpu = _mat(W, shapes, i).astype(np.float32).ravel()
        assert np.array_equal(w_gpu[agree].view(np.uint32), w_ref[agree].view(np.uint32))
        assert (~agree).mean() <= M * 1e-3


@pytest.mark.parametrize("i", [0, 1, 2, 3])
def test_nanogpt_post_vote_polar_full_size(i):
    """The post-vote polar step on its own: PolarNS (bf16, K=5, spectral P=2)
    of a synthetic {-1, 0, +1} matrix of a nanoGPT shape, as the step computes
    it on the majority."""
    shapes = [synth.NANOGPT_SHAPES[i]]
    r, c = shapes[0]
    wl = synth.WORKLOADS["nanogpt"]
    h = smo.SignMuon(shapes, 1, beta=0.9, lam=0.0, K=wl["K"], eps=HP["eps"], scale=wl["scale"], P=wl["P"])
    maj = synth.ternary_direction(r * c, config_id=60 + i, p_zero=0.02)
    X = torch.from_numpy(maj).cuda()
    U = torch.empty_like(X)
    h.polar([X], [U])
    want = ref.polar_ns(maj.astype(np.float64).reshape(r, c), wl["K"], HP["eps"], wl["scale"], wl["P"])
    assert_polar_close(U.double().cpu().numpy().reshape(r, c), want, "bf16", f"post-vote polar {r}x{c}")


def test_resnet50_step_full_size_sampled():
    shapes = synth.RESNET50_SHAPES
    pick = [0, shapes.index((64, 576)), shapes.index((2048, 1024)), len(shapes) - 1]
    _step_sampled("resnet50", pick, post_polar=False)


def _device_bernoulli_packed(d, M, seed):
    """M packed buffers of Bernoulli(p_i) bits, p_i ~ U(0.3, 0.7), drawn on the
    device in chunks (the vote stress input); returns the list of uint8
    tensors (ceil(d/8) bytes each, +16 bytes of zero padding)."""
    g = torch.Generator(device="cuda")
    nb = (d + 7) // 8
    out = [torch.zeros(nb + 16, dtype=torch.uint8, device="cuda") for _ in range(M)]
    weights = torch.tensor([1, 2, 4, 8, 16, 32, 64, 128], dtype=torch.int32, device="cuda")
    chunk = 1 << 26
    for c0 in range(0, d, chunk):
        n = min(chunk, d - c0)
        g.manual_seed(seed * 1000003 + c0)
        p = torch.rand(n, generator=g, device="cuda") * 0.4 + 0.3
        for m in range(M):
            bits = (torch.rand(n, generator=g, device="cuda") < p).to(torch.int32)
            pad = (-n) % 8
            if pad:
                bits = torch.cat([bits, torch.zeros(pad, dtype=torch.int32, device="cuda")])
            byt = (bits.view(-1, 8) * weights).sum(1).to(torch.uint8)
            out[m][c0 // 8: c0 // 8 + byt.numel()] = byt
    return out


@pytest.mark.parametrize("acc8", [False, True])
def test_llama_layer_vote_full_size(acc8):
    shapes = synth.LLAMA_LAYER_SHAPES
    M = 16
    d = synth.numel(shapes)
    signs = _device_bernoulli_packed(d, M, seed=5)
    flags = smo.SIGNMUON_VOTE_ONLY | (smo.SIGNMUON_ACC_INT8 if acc8 else 0)
    h = smo.SignMuon(shapes, M, flags=flags)
    sums = torch.empty(d, dtype=torch.int8 if acc8 else torch.int32, device="cuda")
    maj = torch.empty(d, dtype=torch.int8, device="cuda")
    h.vote(signs, d, sums, maj)
    torch.cuda.synchronize()
    # invariants over every entry
    s32 = sums.to(torch.int32)
    assert int(s32.min()) >= -M and int(s32.max()) <= M
    assert bool(((s32 + M) % 2 == 0).all())
    assert torch.equal(torch.sign(s32).to(torch.int8), maj)
    # sampled entries against the oracle, bit-exact
    rs = np.random.default_rng(3)
    idx = np.unique(np.concatenate([rs.integers(0, d, 4096), np.arange(d - 2048, d)]))
    words = np.unique(idx // 8)
    packed = [s[torch.from_numpy(words).cuda()].cpu().numpy() for s in signs]
    # re-index the sampled bytes as a compact packed vector for the oracle
    local = {w: k for k, w in enumerate(words)}
    sub_idx = np.array([local[i // 8] * 8 + (i % 8) for i in idx])
    want = ref.vote_sums_from_bits(packed, len(words) * 8, "int8" if acc8 else "int32")[sub_idx]
    got = sums[torch.from_numpy(idx).cuda()].cpu().numpy()
    assert np.array_equal(got.astype(np.int64), want.astype(np.int64))
    assert np.array_equal(maj[torch.from_numpy(idx).cuda()].cpu().numpy(), ref.majority(want))


@pytest.mark.parametrize("name,sample", [("batch64_1024", [0, 63]), ("batch256_512x2048", [0, 255])])
@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_ns_sweep_sampled(name, sample, precision):
    _ns_sweep_case(name, sample, precision, "cubic", 5, "spectral")


# the rest of the sweep's grid: K in {5, 10}, cubic and quintic, bf16 and
# fp32, on both batched shapes (the quintic with the Frobenius scale, which
# keeps every singular value of X0 inside the quintic's basin of convergence)
@pytest.mark.parametrize("name,sample", [("batch64_1024", [0, 63]), ("batch256_512x2048", [0, 255])])
@pytest.mark.parametrize("order,K,scale,precision", [
    ("quintic", 5, "fro", "bf16"), ("quintic", 5, "fro", "fp32"), ("cubic", 10, "spectral", "bf16"),
    ("cubic", 10, "spectral", "fp32"), ("quintic", 10, "fro", "bf16"), ("quintic", 10, "fro", "fp32")])
def test_ns_sweep_sampled_grid(name, sample, order, K, scale, precision):
    _ns_sweep_case(name, sample[:1] if precision == "fp32" else sample, precision, order, K, scale)


@pytest.mark.parametrize("name,sample", [("batch64_1024", [0, 63]), ("batch256_512x2048", [0, 255])])
def test_ns_sweep_m8_vote_on_the_results(name, sample):
    """The sweep's M = 8 vote on its results: every worker's PolarNS output
    (bf16, K = 5 cubic, spectral P = 2) packed to one bit per entry and voted
    on the device.  The packed bits equal the signs of the GPU's U (bit for
    bit, sampled matrices); the sums and majority equal the oracle's vote on
    those bits at sampled entries over the whole vector (bit-exact); the
    range, parity and sign invariants hold for every entry; and against the
    oracle's own polar factors the majority agrees wherever every worker's
    sign does."""
    shapes = synth.SWEEP_SHAPES[name]
    M = 8
    h = smo.SignMuon(shapes, M, beta=0.9, lam=0.0, K=5, eps=1e-7, scale="spectral", P=2)
    d = h.d
    X = list(synth.device_gaussian(d, M, seed=2025))
    U = [torch.empty_like(x) for x in X]
    h.polar(X, U)
    nb = (d + 7) // 8
    bits = [torch.zeros(nb + 16, dtype=torch.uint8, device="cuda") for _ in range(M)]
    for m in range(M):
        h.pack(U[m], d, bits[m])
    sums = torch.empty(d, dtype=torch.int32, device="cuda")
    maj = torch.empty(d, dtype=torch.int8, device="cuda")
    h.vote(bits, d, sums, maj)
    torch.cuda.synchronize()
    assert int(sums.min()) >= -M and int(sums.max()) <= M
    assert bool(((sums + M) % 2 == 0).all())
    assert torch.equal(torch.sign(sums).to(torch.int8), maj)
    offs = synth.flat_offsets(shapes)
    for i in sample:
        r, c = shapes[i]
        agree = np.ones(r * c, bool)
        ref_bits, gpu_bits = [], []
        for m in range(M):
            gb = _unpack_range(bits[m], offs[i], r * c)
            assert np.array_equal(gb, _mat(U[m], shapes, i).ravel() >= 0), f"matrix {i} worker {m}: pack"
            u = ref.polar_ns(_mat(X[m], shapes, i), 5, 1e-7, "spectral", 2).ravel()
            rb = ref.sign_bits(u)
            agree &= rb == gb
            ref_bits.append(rb)
            gpu_bits.append(gb)
        ref_maj = np.sign(sum(2 * b.astype(np.int64) - 1 for b in ref_bits))
        got = maj[offs[i]: offs[i] + r * c].cpu().numpy()
        assert np.array_equal(got[agree], ref_maj[agree]), f"matrix {i}: majority differs on agreed entries"
        assert (~agree).mean() <= M * 1e-3
    # sampled entries over the whole vector against the oracle's vote on the GPU's bits
    rs = np.random.default_rng(11)
    idx = np.unique(np.concatenate([rs.integers(0, d, 8192), np.arange(d - 1024, d)]))
    words = np.unique(idx // 8)
    wdev = torch.from_numpy(words).cuda()
    packed = [b[wdev].cpu().numpy() for b in bits]
    local = {w: k for k, w in enumerate(words)}
    sub = np.array([local[i // 8] * 8 + (i % 8) for i in idx])
    want = ref.vote_sums_from_bits(packed, len(words) * 8, "int32")[sub]
    idev = torch.from_numpy(idx).cuda()
    assert np.array_equal(sums[idev].cpu().numpy().astype(np.int64), want.astype(np.int64))
    assert np.array_equal(maj[idev].cpu().numpy(), ref.majority(want))


def _ns_sweep_case(name, sample, precision, order, K, scale):
    shapes = synth.SWEEP_SHAPES[name]
    M = 8
    flags = (smo.SIGNMUON_NS_FP32 if precision == "fp32" else 0) | (smo.SIGNMUON_NS_QUINTIC if order == "quintic" else 0)
    h = smo.SignMuon(shapes, M, beta=0.9, lam=0.0, K=K, eps=1e-7, scale=scale, P=2, flags=flags)
    d = h.d
    X = list(synth.device_gaussian(d, M, seed=2024))
    U = [torch.empty_like(x) for x in X]
    h.polar(X, U)
    for m in (0, M - 1):
        for i in sample:
            want = ref.polar_ns(_mat(X[m], shapes, i), K, 1e-7, scale, 2, order)
            assert_polar_close(_mat(U[m], shapes, i), want, precision, f"{name} {order} K={K} worker {m} matrix {i}")


def _hadamard_entry(i, j):
    """Entry (i, j) of the Sylvester-Hadamard matrix: (-1)^popcount(i & j)."""
    return 1 - 2 * (np.bitwise_count(np.asarray(i) & np.asarray(j)).astype(np.int64) & 1)


@pytest.mark.parametrize("order,K,precision", [
    ("cubic", 5, "fp32"), ("quintic", 5, "fp32"), ("cubic", 10, "fp32"), ("quintic", 10, "fp32"),
    ("cubic", 5, "bf16"), ("quintic", 5, "bf16"), ("cubic", 10, "bf16"), ("quintic", 10, "bf16")])
def test_ns_sweep_8192_known_polar_factor(order, K, precision):
    n = 8192
    rs = np.random.default_rng(8192)
    s = rs.uniform(0.2, 1.0, n)
    perm = rs.permutation(n)
    sgn = rs.choice([-1.0, 1.0], n)
    # X[i, k] = H[i, perm[k]] * s[perm[k]] * sgn[k] / sqrt(n): X = H diag(s) Q^T
    # with Q the signed permutation Q[k, j] = sgn[k] [perm[k] = j]
    i = torch.arange(n, device="cuda", dtype=torch.int64).view(n, 1)
    pk = torch.from_numpy(perm).cuda().view(1, n)
    hbits = (i & pk)
    pop = torch.zeros_like(hbits)
    for b in range(13):
        pop += (hbits >> b) & 1
    Hsign = (1 - 2 * (pop & 1)).to(torch.float32)
    col = torch.from_numpy((s[perm] * sgn / math.sqrt(n)).astype(np.float32)).cuda().view(1, n)
    X = (Hsign * col).reshape(-1).contiguous()
    del Hsign, hbits, pop
    flags = (smo.SIGNMUON_NS_FP32 if precision == "fp32" else 0) | (smo.SIGNMUON_NS_QUINTIC if order == "quintic" else 0)
    h = smo.SignMuon([(n, n)], 1, beta=0.9, lam=0.0, K=K, eps=1e-7, scale="fro", flags=flags)
    U = torch.empty_like(X)
    h.polar([X], [U])
    torch.cuda.synchronize()
    # closed form: U = H diag(f^K(s / (||s|| + eps))) Q^T, entry by entry
    x0 = s / (math.sqrt(float(np.sum(s * s))) + 1e-7)
    fk = x0.copy()
    for _ in range(K):
        fk = 1.5 * fk - 0.5 * fk ** 3 if order == "cubic" else fk * (15 / 8 - 10 / 8 * fk ** 2 + 3 / 8 * fk ** 4)
    ri = rs.integers(0, n, 3000)
    ci = rs.integers(0, n, 3000)
    want = _hadamard_entry(ri, perm[ci]) * fk[perm[ci]] * sgn[ci] / math.sqrt(n)
    got = U.view(n, n)[torch.from_numpy(ri).cuda(), torch.from_numpy(ci).cuda()].double().cpu().numpy()
    err = np.max(np.abs(got - want))
    tol = {"fp32": 1e-4, "bf16": 2e-2}[precision]
    assert err <= tol, f"max abs error {err:.3e}"
    # a sharper bound than the absolute tolerance at this entry scale (|U| ~ 1e-2)
    rel = {"fp32": 0.02, "bf16": 0.1}[precision]
    assert err <= rel * np.max(np.abs(want)), f"relative error {err / np.max(np.abs(want)):.3e}"


@pytest.mark.parametrize("name,steps,flags", [("resnet50", 12, 0), ("nanogpt", 4, "post")])
def test_full_size_steps_are_deterministic(name, steps, flags):
    """Two handles run the same sequence of full-size steps (fresh gradients
    every step, the asynchronous mode the bench times): W and every worker's
    momentum must come out bit-identical.  Nothing in a step depends on
    scheduling -- the GEMM tiles, the power iteration's slot sums in a fixed
    order, the vote's integer counts, and the one-bit signs OR-ed into words
    for ResNet-50's ragged 147-column stem -- so any race would show here."""
    wl = synth.WORKLOADS[name]
    shapes, M = wl["shapes"], wl["M"]
    f = smo.SIGNMUON_ASYNC | (smo.SIGNMUON_POST_POLAR if flags == "post" else 0)
    outs = []
    for _ in range(2):
        opt = smo.SignMuon(shapes, M, beta=HP["beta"], lam=HP["lam"], K=wl["K"], eps=HP["eps"], scale=wl["scale"],
                           P=wl["P"], flags=f)
        W = synth.device_weights0(shapes, config_id=61)
        for t in range(steps):
            G = synth.device_gradients(shapes, M, wl["sigma"], step=t, config_id=61)
            opt.step(W, [G[m] for m in range(M)], HP["eta"])
            del G
        opt.sync()
        moms = []
        for m in range(M):
            x = torch.empty(opt.d, device="cuda")
            opt.get_momentum(m, x)
            moms.append(x)
        outs.append((W, moms))
        opt.close()
    assert torch.equal(outs[0][0].view(torch.int32), outs[1][0].view(torch.int32))
    for m in range(M):
        assert torch.equal(outs[0][1][m].view(torch.int32), outs[1][1][m].view(torch.int32))
