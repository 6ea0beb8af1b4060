"""Seeded synthetic inputs for the Sign-Muon optimizer step.

This module is shared by the CPU oracle's tests, the GPU tests and the
benchmark. It holds only weight-matrix shapes and random-number recipes; it
contains none of the optimizer's arithmetic (no momentum, scaling,
Newton-Schulz, sign, vote or update), so that the oracle and the CUDA path
stay independent of one another.

Workload shapes are stand-ins for the pages' models (the datasets and trained
weights are not used; only the weight shapes are):

* ``small_256x128``: one 256x128 matrix, 3 workers, noise scale 0.5.
* ``resnet50``: the 54 conv/fc weights of ResNet-50, each conv flattened to
  out x (in*kh*kw), in torchvision module order (25,502,912 weights).
* ``nanogpt``: 12 transformer layers x {qkv 2304x768, attn proj 768x768,
  mlp fc 3072x768, mlp proj 768x3072} (84,934,656 weights).
* ``llama_layer``: 32 x 4096x4096 plus 4 x 11008x4096 (717,225,984 weights),
  used for the vote stress test only.
* NS sweep sets: one 8192x8192, 64 x 1024x1024, 256 x 512x2048.

Gradient model (a fresh draw every step): ``G_m = S + sigma * N_m`` with S and
every N_m i.i.d. standard normal; ``W0 ~ N(0, 0.02^2)`` (0.02 is the standard
deviation).
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# shapes
# ---------------------------------------------------------------------------


def _resnet50_shapes():
    shapes = [(64, 3 * 7 * 7)]  # stem conv 7x7, 3 -> 64
    in_ch = 64
    for width, blocks in ((64, 3), (128, 4), (256, 6), (512, 3)):
        out_ch = width * 4
        for b in range(blocks):
            shapes.append((width, in_ch * 1 * 1))      # 1x1 reduce
            shapes.append((width, width * 3 * 3))      # 3x3
            shapes.append((out_ch, width * 1 * 1))     # 1x1 expand
            if b == 0:
                shapes.append((out_ch, in_ch * 1 * 1))  # projection shortcut
            in_ch = out_ch
    shapes.append((1000, 2048))  # classifier
    return shapes


RESNET50_SHAPES = _resnet50_shapes()
NANOGPT_SHAPES = [(2304, 768), (768, 768), (3072, 768), (768, 3072)] * 12
LLAMA_LAYER_SHAPES = [(4096, 4096)] * 32 + [(11008, 4096)] * 4
SMALL_256x128_SHAPES = [(256, 128)]
SWEEP_SHAPES = {
    "single_8192": [(8192, 8192)],
    "batch64_1024": [(1024, 1024)] * 64,
    "batch256_512x2048": [(512, 2048)] * 256,
}

# Per-workload run parameters (hyper-parameters not given for a workload take
# the small 256x128 workload's values: beta=0.9, lambda=0.01, eta=0.02,
# eps=1e-7).
WORKLOADS = {
    "small_256x128": dict(shapes=SMALL_256x128_SHAPES, M=3, sigma=0.5, K=5, scale="fro", P=1,
                          order="cubic", precision="fp32", post_polar=False, steps=10),
    "resnet50": dict(shapes=RESNET50_SHAPES, M=4, sigma=1.0, K=5, scale="spectral", P=2,
                     order="cubic", precision="bf16", post_polar=False, steps=20),
    "nanogpt": dict(shapes=NANOGPT_SHAPES, M=8, sigma=2.0, K=5, scale="spectral", P=2,
                    order="cubic", precision="bf16", post_polar=True, steps=50),
    "llama_vote": dict(shapes=LLAMA_LAYER_SHAPES, M=16),
}
HYPER = dict(beta=0.9, lam=0.01, eta=0.02, eps=1e-7)


def numel(shapes) -> int:
    return int(sum(int(r) * int(c) for r, c in shapes))


def flat_offsets(shapes):
    """Start of each matrix in the flat parameter vector (row-major, shapes order)."""
    off, out = 0, []
    for r, c in shapes:
        out.append(off)
        off += int(r) * int(c)
    return out


# ---------------------------------------------------------------------------
# seeded generators (host, numpy)
# ---------------------------------------------------------------------------

_TAGS = {"w0": 1, "signal": 2, "noise": 3, "mom0": 4, "bits": 5, "p": 6, "u": 7, "dir": 8,
         "mat": 9}


def rng(config_id: int, step: int, tag: str, m: int = 0) -> np.random.Generator:
    """A PCG64 stream keyed by (workload id, step, stream tag, worker)."""
    return np.random.Generator(np.random.PCG64(
        np.random.SeedSequence([int(config_id), int(step), _TAGS[tag], int(m)])))


def weights0(shapes, config_id=0) -> np.ndarray:
    """W0 ~ N(0, 0.02^2), float32, flat."""
    d = numel(shapes)
    return (0.02 * rng(config_id, 0, "w0").standard_normal(d, dtype=np.float32)).astype(np.float32)


def gradients(shapes, M, sigma, step, config_id=0):
    """List of M float32 flat gradients G_m = S + sigma*N_m for this step."""
    d = numel(shapes)
    s = rng(config_id, step, "signal").standard_normal(d, dtype=np.float32)
    out = []
    for m in range(M):
        n = rng(config_id, step, "noise", m).standard_normal(d, dtype=np.float32)
        out.append((s + np.float32(sigma) * n).astype(np.float32))
    return out


def momentum0(shapes, M, config_id=0, scale=1.0):
    """A synthetic non-zero momentum state (float32), for single-step tests."""
    d = numel(shapes)
    return [(np.float32(scale) * rng(config_id, 0, "mom0", m).standard_normal(d, dtype=np.float32))
            .astype(np.float32) for m in range(M)]


def gaussian_matrices(shapes, M, config_id=0, step=0):
    """M flat float32 vectors of i.i.d. N(0,1) entries (NS sweep momentum)."""
    d = numel(shapes)
    return [rng(config_id, step, "mat", m).standard_normal(d, dtype=np.float32) for m in range(M)]


def bernoulli_bits(d, M, config_id=0, lo=0.3, hi=0.7):
    """Vote stress input: p_i ~ U(lo, hi) per entry, then M independent
    Bernoulli(p_i) bits per entry.  Returns a (M, d) bool array."""
    p = rng(config_id, 0, "p").uniform(lo, hi, size=d)
    return np.stack([rng(config_id, 0, "bits", m).random(d) < p for m in range(M)])


def ternary_signs(d, M, config_id=0, p_zero=0.2, lo=0.3, hi=0.7):
    """Ternary vote stress input: per entry p_i ~ U(lo, hi); each of M workers
    independently sends 0 with probability p_zero, else +1 with probability
    p_i and -1 otherwise.  Returns a (M, d) int8 array."""
    p = rng(config_id, 0, "p").uniform(lo, hi, size=d)
    out = np.empty((M, d), np.int8)
    for m in range(M):
        g = rng(config_id, 0, "bits", m)
        z = g.random(d) < p_zero
        plus = g.random(d) < p
        out[m] = np.where(z, 0, np.where(plus, 1, -1)).astype(np.int8)
    return out


def ternary_direction(d, config_id=0, p_zero=0.1):
    """A direction with entries in {-1, 0, +1} (float32)."""
    g = rng(config_id, 0, "dir")
    v = g.choice(np.array([-1.0, 0.0, 1.0], np.float32), size=d,
                 p=[(1 - p_zero) / 2, p_zero, (1 - p_zero) / 2])
    return v.astype(np.float32)


def uniform_values(d, config_id=0, step=0, lo=-1.0, hi=1.0):
    """float32 values U(lo, hi), with a sprinkling of exact zeros and -0.0."""
    g = rng(config_id, step, "u")
    v = g.uniform(lo, hi, size=d).astype(np.float32)
    if d >= 8:
        idx = g.choice(d, size=max(1, d // 64), replace=False)
        v[idx[: len(idx) // 2]] = np.float32(0.0)
        v[idx[len(idx) // 2:]] = np.float32(-0.0)
    return v


# ---------------------------------------------------------------------------
# seeded generators (device, torch) for full-size benchmark inputs
# ---------------------------------------------------------------------------

def device_gradients(shapes, M, sigma, step, config_id=0, device="cuda", out=None):
    """G_m = S + sigma*N_m drawn on the device with torch's Philox generator
    (seeded from the same key); used where host generation of hundreds of
    millions of normals would dominate a run.  ``out`` may be a preallocated
    (M, d) float32 tensor."""
    import torch
    d = numel(shapes)
    key = int(np.random.SeedSequence([int(config_id), int(step), 2]).generate_state(1)[0])
    g = torch.Generator(device=device)
    g.manual_seed(key)
    if out is None:
        out = torch.empty((M, d), dtype=torch.float32, device=device)
    s = torch.randn(d, generator=g, device=device, dtype=torch.float32)
    for m in range(M):
        torch.randn(d, generator=g, device=device, dtype=torch.float32, out=out[m])
        out[m].mul_(float(sigma)).add_(s)
    del s
    return out


def device_gaussian(d, M, seed=0, device="cuda"):
    """(M, d) float32 i.i.d. N(0,1) on the device (NS sweep momentum)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(np.random.SeedSequence([int(seed), 9]).generate_state(1)[0]))
    return torch.randn((M, d), generator=g, device=device, dtype=torch.float32)


def device_weights0(shapes, config_id=0, device="cuda"):
    import torch
    d = numel(shapes)
    key = int(np.random.SeedSequence([int(config_id), 0, 1]).generate_state(1)[0])
    g = torch.Generator(device=device)
    g.manual_seed(key)
    return torch.randn(d, generator=g, device=device, dtype=torch.float32).mul_(0.02)
