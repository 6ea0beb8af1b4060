"""CPU oracle for the Sign-Muon optimizer step.  TEST INFRASTRUCTURE ONLY.

Only the tests, the package's smoke check and the benchmark's CPU-baseline leg
may import this module.  It is plain numpy in float64 (the update is rounded
once to float32 at the end), slow, and shares no code with the CUDA path.

Sources, by page title:

* [paper]  "SignMuon: 通信高效的分布式Muon优化" -- a rendering of the arXiv paper
  (Mishra, Trivedi & Kumar, arXiv 2605.16311).
* [blog]   "SignMuon: Matrix Directions, Majority Votes, and the Actual Bytes
  Sent" (the authors' methodology post).
* [radio]  "SignMuon: Communication-Efficient Distributed Muon Optimization"
  (AI Radio episode, a paraphrase of the paper).

What one step computes, for M workers that share the weights W:

1. coupled weight decay and momentum per worker       [paper] Algorithm 1, Algorithm 2
2. a polar direction U_m = PolarNS(Mom_m) per matrix  [paper] §3 (Muon update rule), §4
3. entrywise signs of U_m, one bit each               [paper] §3, Algorithm 2; [blog] bytes
4. majority vote sign(sum of signs), ties to 0        [blog] "A tiny aggregation calculation"
5. optional post-vote local polar step                [paper] §4 (where to orthogonalise)
6. W <- W - eta * D                                    [paper] Algorithm 1, Algorithm 2

Readings taken where the pages are silent or disagree (each is listed with its
reason in the design notes):

R1  Non-square NS: iterate on the orientation X (m x n, m <= n) whose Gram
    X X^T is the small one; transpose back at the end.
R2  Power iteration: start u0 = ones(m)/sqrt(m) on the small side (m = min dim
    of the wide orientation), each iteration u <- X(X^T u)/||X(X^T u)||, and
    sigma = ||X^T u|| after P iterations.  A zero iterate stays zero.
R3  Scale: X0 = Mom / (s + eps).
R4  Quintic NS: X <- X (15/8 I - 10/8 X^T X + 3/8 (X^T X)^2), the second-order
    expansion of (X^T X)^(-1/2); cubic is X <- X (3/2 I - 1/2 X^T X).
R5  One-bit sign: bit = (U >= 0), so 0 and -0 send +1.  The ternary sign keeps
    sign(0) = 0 as in [paper] §3.
R6  Packing: one flat bit stream over all matrices (shapes order, row-major),
    bit j of byte b is element 8b+j; ceil(d/8) bytes; pad bits 0.
R7  Ties map to 0 ([blog]) by default; the +1 policy of [paper] Algorithm 2 is
    the named variant majority(..., tie=1).
R8  Post-vote polar: D = PolarNS(majority as floats) with the same K, eps,
    scale and P; no second sign, no rescale.  The pages fix neither where this
    step sits nor its scale, so beyond the PolarNS arithmetic (pinned by the
    closed forms) its parity is unpinned.
R9  Update: W_new = float32 nearest to (W - eta*D), one rounding.
R19 Ternary wire (named variant): sign(U) in {-1, 0, +1}, one int8 per entry.
R20 Normalised sign step (named variant): D = majority / (s + eps) per matrix,
    s the scale PolarNS would use (R2 for spectral, the Frobenius norm for fro).
R21 Warm-started power iteration (named variant): each problem's power
    iteration starts from the iterate it ended with in the previous step;
    a zero or non-finite stored iterate starts from ones/sqrt(m) as in R2.

Named variants (each a flag of the CUDA path, pinned in the tests):

* majority(sums, tie=1): a tie gives +1, [paper] Algorithm 2's default on the
  {-1, +1} wire (pinned by brute force over all vote patterns).
* step(..., pre_polar=False): the signs of the momentum itself, orthogonalised
  only after the vote ([paper] §4, where to orthogonalise; closed-form pin).
* muon_step: the Muon baseline the paper compares against (its §3 Muon update
  applied to the workers' mean momentum; closed-form pin, and equal to a
  worker's polar factor when M = 1).
* step(..., signs="ternary"): int8 signs in {-1, 0, +1}, d bytes per worker
  ([paper] §3 sign(0) = 0; Algorithm 2's int8 all-reduce of d bytes), summed
  as integers (pinned by brute force over all 3^M patterns, by the zero
  momentum closed form, and by equality with the one-bit step when U has no
  zeros).
* step(..., warm={...}): warm-started power iterations (R21; [paper]
  Algorithm 1's P with the iterate carried across steps).  On a constant
  matrix, t warm steps of P iterations equal one cold start with P*t
  iterations exactly (pinned), and a zero state restarts cold.
* step(..., normalize=True): D = majority / ||majority||_2 per matrix
  ([paper] §4, the explicitly normalised sign step of the analysis), with the
  norm estimated as PolarNS estimates its scale (pinned by exact singular
  values of ternary matrices: rank-one sign patterns, signed permutations).
"""
from __future__ import annotations

import math

import numpy as np

# Newton-Schulz polynomials: X <- X * p(X^T X)
CUBIC = (1.5, -0.5)                 # [paper] §4: X(3/2 I - 1/2 X^T X)
QUINTIC = (15.0 / 8.0, -10.0 / 8.0, 3.0 / 8.0)  # reading R4


# ---------------------------------------------------------------------------
# 1. weight decay + momentum
# ---------------------------------------------------------------------------

def momentum_update(mom, g, w, beta, lam, dtype=np.float64):
    """Coupled weight decay then an exponential moving average.

    [paper] Algorithm 1 and Algorithm 2: the decayed gradient is
    G~ = G + lambda*W, and the new momentum is beta*Mom + (1-beta)*G~
    (momentum starts at zero).  dtype: the arithmetic (float64 for parity;
    float32 only for the timed CPU baseline).
    """
    g_tilde = np.asarray(g, dtype) + float(lam) * np.asarray(w, dtype)
    return float(beta) * np.asarray(mom, dtype) + (1.0 - float(beta)) * g_tilde


# ---------------------------------------------------------------------------
# 2. PolarNS
# ---------------------------------------------------------------------------

def frobenius_norm(x):
    """||X||_F = sqrt(sum of squared entries) ([paper] §3 notation)."""
    x = np.asarray(x, np.float64)
    return math.sqrt(float(np.sum(x * x)))


def power_sigma(x, P, u0=None, return_u=False, dtype=np.float64):
    """Estimate of the largest singular value of a wide X (m <= n) by P power
    iterations on X X^T (reading R2; [paper] Algorithm 1 input P, §4).

    u0 is a warm start on the small side (reading R21): the iterate a previous
    call ended with.  None, an all-zero or a non-finite u0 starts from
    ones(m)/sqrt(m).  With return_u the final iterate comes back as well.
    """
    x = np.asarray(x, dtype)
    m = x.shape[0]
    if u0 is not None and np.all(np.isfinite(u0)) and np.any(np.asarray(u0) != 0):
        u = np.array(u0, dtype)
    else:
        u = np.full(m, 1.0 / math.sqrt(m), dtype)
    for _ in range(int(P)):
        y = x @ (x.T @ u)
        nrm = math.sqrt(float(y @ y))
        u = y / nrm if nrm > 0.0 else np.zeros(m, dtype)
    z = x.T @ u
    sigma = math.sqrt(float(z @ z))
    return (sigma, u) if return_u else sigma


def ns_iterate(x0, K, order="cubic", coeffs=None, dtype=np.float64):
    """K Newton-Schulz steps on a wide X (m <= n).

    With A = X X^T, the step X(aI + b X^T X) equals aX + b A X ([paper] §3,
    two-coefficient form; §4, cubic a=3/2, b=-1/2).  The quintic step (reading
    R4) is aX + (bA + cA^2) X.
    """
    x = np.asarray(x0, dtype)
    if order == "cubic":
        a, b = coeffs if coeffs is not None else CUBIC
        for _ in range(int(K)):
            gram = x @ x.T
            x = a * x + b * (gram @ x)
    elif order == "quintic":
        a, b, c = coeffs if coeffs is not None else QUINTIC
        for _ in range(int(K)):
            gram = x @ x.T
            x = a * x + (b * gram + c * (gram @ gram)) @ x
    else:
        raise ValueError(order)
    return x


def polar_ns(mat, K, eps, scale, P=1, order="cubic", coeffs=None, return_scale=False, u0=None,
             return_u=False, dtype=np.float64):
    """PolarNS(Mat; K, eps, scale, P) of one matrix ([paper] Algorithm 1, §4).

    Works on the wide orientation (R1), divides by s + eps where s is the
    Frobenius norm or the power-iteration estimate of the spectral norm
    (R2, R3), runs K Newton-Schulz steps and returns the result in the
    matrix's own orientation.  u0 warm-starts the power iteration (R21);
    return_u returns (result, s, final iterate or None for fro).
    """
    mat = np.asarray(mat, dtype)
    tall = mat.shape[0] > mat.shape[1]
    x = mat.T if tall else mat
    u = None
    if scale == "fro":
        s = frobenius_norm(x)
    elif scale == "spectral":
        s, u = power_sigma(x, P, u0, return_u=True, dtype=dtype)
    else:
        raise ValueError(scale)
    x = x / (s + float(eps))
    x = ns_iterate(x, K, order, coeffs, dtype=dtype)
    out = x.T if tall else x
    if return_u:
        return out, s, u
    return (out, s) if return_scale else out


# ---------------------------------------------------------------------------
# 3. signs and 1-bit packing
# ---------------------------------------------------------------------------

def sign_ternary(u):
    """Entrywise sign with sign(0) = 0 ([paper] §3 notation; [blog] example)."""
    u = np.asarray(u)
    return (u > 0).astype(np.int32) - (u < 0).astype(np.int32)


def sign_bits(u):
    """One-bit sign: True means +1.  0 and -0 send +1 (reading R5)."""
    return np.asarray(u) >= 0


def packed_nbytes(d):
    """Payload of d one-bit signs: ceil(d/8) bytes ([blog] "d/8 bytes")."""
    return (int(d) + 7) // 8


def pack_bits(bits):
    """Flat bool vector -> uint8 bytes, bit j of byte b is element 8b+j (R6)."""
    bits = np.asarray(bits, bool).ravel()
    d = bits.size
    padded = np.zeros(packed_nbytes(d) * 8, np.uint8)
    padded[:d] = bits
    out = np.zeros(packed_nbytes(d), np.uint8)
    for j in range(8):
        out |= (padded[j::8] << j).astype(np.uint8)
    return out


def unpack_bits(packed, d):
    """Inverse of pack_bits: first d bits as a bool vector."""
    packed = np.asarray(packed, np.uint8)
    out = np.zeros(packed.size * 8, bool)
    for j in range(8):
        out[j::8] = (packed >> j) & 1
    return out[: int(d)]


# ---------------------------------------------------------------------------
# 4. majority vote
# ---------------------------------------------------------------------------

class AccumulatorOverflow(ValueError):
    """An int8 accumulator cannot hold sums in [-M, M] for M > 127."""


def vote_sums_from_bits(packed_list, d, acc="int32"):
    """sum_i = sum over workers of (+1 if bit else -1) ([paper] Algorithm 2:
    an integer SUM of the workers' signs; [blog] on the [-P, P] range and
    int8 overflow)."""
    M = len(packed_list)
    if acc == "int8" and M > 127:
        raise AccumulatorOverflow(f"int8 sums overflow for M={M} > 127")
    total = np.zeros(int(d), np.int64)
    for p in packed_list:
        b = unpack_bits(p, d).astype(np.int64)
        total += 2 * b - 1
    return total.astype(np.int8 if acc == "int8" else np.int32)


def vote_sums_ternary(sign_list, acc="int32"):
    """Integer sum of ternary sign arrays: the [blog] worked example, and the
    int8 SUM all-reduce of [paper] Algorithm 2 whose payload is one byte per
    entry and worker.  Entries must be -1, 0 or +1, so sums lie in [-M, M]."""
    M = len(sign_list)
    if acc == "int8" and M > 127:
        raise AccumulatorOverflow(f"int8 sums overflow for M={M} > 127")
    total = np.zeros(np.shape(sign_list[0]), np.int64)
    for s in sign_list:
        s = np.asarray(s, np.int64)
        if np.any(np.abs(s) > 1):
            raise ValueError("ternary signs must be -1, 0 or +1")
        total += s
    return total.astype(np.int8 if acc == "int8" else np.int32)


def majority(sums, tie=0):
    """sign(sum) with a tie (sum 0) mapped to 0 (R7, [blog]); with tie=+1 a
    tie gives +1 instead, [paper] Algorithm 2's default for sign(0) on the
    {-1, +1} wire (a named variant)."""
    maj = sign_ternary(sums).astype(np.int8)
    if tie == 1:
        maj[np.asarray(sums) == 0] = 1
    elif tie != 0:
        raise ValueError("tie must be 0 or 1")
    return maj


# ---------------------------------------------------------------------------
# 6. update
# ---------------------------------------------------------------------------

def _round_f32(s, err):
    """float32 nearest to the exact value s + err (s float64, |err| at most half
    an ulp of s, err the exact residual), ties to even.

    float32(s) is already right unless s sits exactly on a float32 midpoint
    and err != 0; then the exact value lies to err's side of the midpoint.
    """
    r = s.astype(np.float32)
    toward = np.nextafter(r, np.where(s > r.astype(np.float64), np.float32(np.inf),
                                      np.float32(-np.inf)).astype(np.float32))
    mid = (r.astype(np.float64) + toward.astype(np.float64)) * 0.5
    on_mid = (r.astype(np.float64) != s) & (mid == s) & (err != 0)
    hi = np.maximum(r, toward)
    lo = np.minimum(r, toward)
    return np.where(on_mid, np.where(err > 0, hi, lo), r).astype(np.float32)


def update(w, direction, eta):
    """W_new = W - eta*D, rounded once to float32 ([paper] Algorithm 1, 2;
    reading R9).  W, D and eta are float32 values; eta*D is exact in float64
    and the subtraction's rounding error is recovered exactly (two-sum)."""
    w64 = np.asarray(w, np.float32).astype(np.float64)
    p = np.float64(np.float32(eta)) * np.asarray(direction, np.float32).astype(np.float64)
    a, b = w64, -p
    s = a + b
    bb = s - a
    err = (a - (s - bb)) + (b - bb)
    return _round_f32(s, err)


# ---------------------------------------------------------------------------
# the whole step
# ---------------------------------------------------------------------------

def split(flat, shapes, offsets=None):
    """Views of a flat vector as the matrices of ``shapes`` (row-major)."""
    out, off = [], 0
    for r, c in shapes:
        out.append(np.asarray(flat)[off: off + r * c].reshape(r, c))
        off += r * c
    return out


def polar_flat(flat, shapes, K, eps, scale, P=1, order="cubic", u0=None, return_u=False, dtype=np.float64):
    """PolarNS of every matrix of a flat vector, returned flat (in dtype,
    float64 unless asked otherwise).  u0: None or one warm start (or None)
    per matrix (R21); with return_u the per-matrix final iterates come back
    too."""
    out = np.empty(int(np.asarray(flat).size), dtype)
    us = []
    off = 0
    for i, ((r, c), mat) in enumerate(zip(shapes, split(np.asarray(flat, dtype), shapes))):
        res, _, u = polar_ns(mat, K, eps, scale, P, order, u0=None if u0 is None else u0[i], return_u=True,
                             dtype=dtype)
        us.append(u)
        out[off: off + r * c] = res.ravel()
        off += r * c
    return (out, us) if return_u else out


def normalize_flat(flat, shapes, eps, scale, P=1, u0=None, return_u=False):
    """Each matrix of a flat vector divided by its norm: D_i / (s_i + eps).

    [paper] §4 (single-worker variant) notes that the theory normalises the
    sign matrix explicitly by its spectral norm, D / ||D||_2.  s_i is the same
    scale estimate PolarNS uses for its input (reading R2 for spectral: P power
    iterations on the wide orientation; the Frobenius norm for fro), and eps
    keeps an all-zero majority at zero.  This is PolarNS with K = 0.  u0 and
    return_u: per-matrix warm starts and final iterates, as in polar_flat.
    """
    if scale not in ("fro", "spectral"):
        raise ValueError(scale)
    out = np.empty(int(np.asarray(flat).size), np.float64)
    us = []
    off = 0
    for i, ((r, c), mat) in enumerate(zip(shapes, split(np.asarray(flat, np.float64), shapes))):
        x = mat.T if r > c else mat
        u = None
        if scale == "fro":
            s = frobenius_norm(x)
        else:
            s, u = power_sigma(x, P, None if u0 is None else u0[i], return_u=True)
        us.append(u)
        out[off: off + r * c] = (mat / (s + float(eps))).ravel()
        off += r * c
    return (out, us) if return_u else out


def step(W, G_list, mom_list, shapes, *, beta, lam, eta, K, eps, scale, P=1,
         order="cubic", post_polar=False, acc="int32", tie=0, pre_polar=True,
         signs="bits", normalize=False, warm=None, dtype=np.float64):
    """One distributed Sign-Muon step ([paper] Algorithm 2, with the vote of
    [blog] and the optional post-vote polar step of [paper] §4).

    Named variants: tie=1 sends a tied vote to +1 ([paper] Algorithm 2's
    default); pre_polar=False signs the momentum itself and orthogonalises
    only after the vote ([paper] §4 "where to orthogonalise", the
    after-only placement; needs post_polar=True); signs="ternary" sends
    sign(U) in {-1, 0, +1}, one int8 per entry ([paper] §3 sign with
    sign(0) = 0, and Algorithm 2's d-byte int8 all-reduce) instead of one bit;
    normalize=True takes D = majority / ||majority||_2 per matrix ([paper] §4,
    the explicitly normalised sign step of the analysis; cannot be combined
    with post_polar); warm (a dict, {} on the first step) warm-starts every
    power iteration from the previous step's final iterates (reading R21):
    warm["workers"][m][i] for worker m's matrix i, warm["single"][i] for the
    post-vote or normalised step's matrix i; the new state is returned as
    out["warm"].  dtype: the arithmetic of the momentum and both PolarNS
    steps (float64, the parity mode; float32 only for the timed CPU
    baseline); the vote and the update are exact either way.

    Returns a dict with the new momentum (float64), the polar factors U_m
    (the momentum itself when pre_polar is False), the packed bits (the int8
    ternary signs when signs="ternary"), the vote sums, the majority, the
    direction D and the new W (float32).  Inputs are flat vectors; momentum
    is float64 or float32.
    """
    if not pre_polar and not post_polar:
        raise ValueError("pre_polar=False needs post_polar=True")
    if normalize and post_polar:
        raise ValueError("normalize=True replaces the post-vote polar step")
    if signs not in ("bits", "ternary"):
        raise ValueError(signs)
    M = len(G_list)
    d = int(np.asarray(W).size)
    wk = None if warm is None else warm.get("workers")
    new_warm = None if warm is None else dict(workers=[None] * M, single=warm.get("single"))
    new_mom, U_list, packed = [], [], []
    for m in range(M):
        mom = momentum_update(mom_list[m], G_list[m], W, beta, lam, dtype=dtype)
        new_mom.append(mom)
        if pre_polar:
            u, us = polar_flat(mom, shapes, K, eps, scale, P, order, u0=None if wk is None else wk[m],
                               return_u=True, dtype=dtype)
            if new_warm is not None:
                new_warm["workers"][m] = us
        else:
            u = np.asarray(mom, np.float64)
        U_list.append(u)
        if signs == "ternary":
            packed.append(sign_ternary(u).astype(np.int8))
        else:
            packed.append(pack_bits(sign_bits(u)))
    if signs == "ternary":
        sums = vote_sums_ternary(packed, acc)
    else:
        sums = vote_sums_from_bits(packed, d, acc)
    maj = majority(sums, tie)
    single = None if warm is None else warm.get("single")
    if post_polar:
        D, us = polar_flat(maj.astype(dtype), shapes, K, eps, scale, P, order, u0=single, return_u=True,
                           dtype=dtype)
        D32 = D.astype(np.float32)
        if new_warm is not None:
            new_warm["single"] = us
    elif normalize:
        D, us = normalize_flat(maj.astype(np.float64), shapes, eps, scale, P, u0=single, return_u=True)
        D32 = D.astype(np.float32)
        if new_warm is not None:
            new_warm["single"] = us
    else:
        D = maj.astype(np.float64)
        D32 = maj.astype(np.float32)
    W_new = update(W, D32, eta)
    return dict(mom=new_mom, U=U_list, packed=packed, sums=sums, majority=maj,
                D=D, D32=D32, W=W_new, warm=new_warm)


def muon_step(W, G_list, mom_list, shapes, *, beta, lam, eta, K, eps, scale, P=1, order="cubic", warm=None):
    """The Muon baseline the pages compare against ([paper] §4 Muon update,
    Table 1's "Muon" row): the workers' momenta are averaged (the all-reduce
    of full-precision momentum) and the mean goes through one PolarNS per
    matrix; W_new = fl32(W - eta * D) with D = PolarNS(mean Mom).  warm as in
    step (the mean's power iterations use warm["single"])."""
    M = len(G_list)
    new_mom = [momentum_update(mom_list[m], G_list[m], W, beta, lam) for m in range(M)]
    mean = np.sum(np.stack([np.asarray(x, np.float64) for x in new_mom]), axis=0) / M
    D, us = polar_flat(mean, shapes, K, eps, scale, P, order, u0=None if warm is None else warm.get("single"),
                       return_u=True)
    D32 = D.astype(np.float32)
    new_warm = None if warm is None else dict(workers=warm.get("workers"), single=us)
    return dict(mom=new_mom, mean=mean, D=D, D32=D32, W=update(W, D32, eta), warm=new_warm)
