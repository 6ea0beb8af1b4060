"""Benchmark of the Sign-Muon optimizer step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = the whole hot path through the C ABI (signmuon_step): momentum
pass, power iteration, 5 cubic Newton-Schulz iterations on the tensor cores
for each of M=8 simulated workers, one-bit pack, majority vote, post-vote
polar step and the update, on nanoGPT-124M-shaped weights (48 matrices,
d = 84,934,656).  Inputs are seeded synthetic gradients resident in HBM (two
alternating 2.7 GB sets, larger than L2).  With N > 1 (torchrun) every rank
runs an independent replica of the same workload; the path has no data
exchange between GPUs.

Rank 0 prints one JSON line.  ``--impl reference`` times the CPU oracle on
the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "Sign-Muon steps/s (nanoGPT-124M, M=8); NS TFLOP/s and vote GB/s % of peak"
WL = synth.WORKLOADS["nanogpt"]
HP = synth.HYPER
SHAPES = WL["shapes"]
M = WL["M"]
K_NS = WL["K"]
D = synth.numel(SHAPES)
WORKLOAD_DESC = ("nanoGPT-124M weight shapes: 12 x {2304x768, 768x768, 3072x768, 768x3072} "
                 f"(d={D:,}); M={M} simulated workers; G_m = S + 2.0 N_m; K={K_NS} cubic Newton-Schulz "
                 "in bf16 on tcgen05 with fp32 accumulation; spectral scale with P=2 power iterations; "
                 "post-vote polar step; beta=0.9 lambda=0.01 eta=0.02 eps=1e-7")

# per-(GPU) fallback peaks, used only when MEASURED_PEAKS.json is absent
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# fp32 FMA peak of the CUDA cores (the fp32 Newton-Schulz path runs there):
# 148 SMs x 128 fp32 lanes x 2 flops x 1.965 GHz
FP32_SIMT_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return j, "measured"
    return FALLBACK, "fallback"


def gemm_traffic_from_profile():
    """DRAM bytes per Newton-Schulz GEMM launch from the committed ncu summary
    (a 2-layer capture scaled to the full workload), or None."""
    p = os.path.join(ROOT, "profiles", "k_gemm_tc_nanogpt_2layers.md")
    try:
        for line in open(p):
            if line.startswith("traffic per full-size launch (bytes):"):
                return float(line.split(":", 1)[1])
    except OSError:
        pass
    return None


def ns_flops_per_step(shapes, M, K, post_polar):
    """Algorithmic Newton-Schulz flops: per matrix and cubic iteration two
    GEMMs, X X^T (2 m^2 n) and A X (2 m^2 n), m = min dim, n = max dim."""
    per_worker = sum(4.0 * min(r, c) ** 2 * max(r, c) for r, c in shapes) * K
    return per_worker * (M + (1 if post_polar else 0))


def ns_kind_flops(shapes, nw, K, gram_ns):
    """Algorithmic flops of each Newton-Schulz GEMM kind for nw problem sets
    (cubic), as the handle runs them.  On X: K x (Gram X X^T, 2 m^2 n;
    apply A X, 2 m^2 n).  In Gram space: one Gram, 3K - 3 products of m x m
    matrices (2 m^3 each) and one apply (2 m^2 n)."""
    mn = sum(2.0 * min(r, c) ** 2 * max(r, c) for r, c in shapes) * nw
    mmm = sum(2.0 * min(r, c) ** 3 for r, c in shapes) * nw
    if gram_ns:
        return {"gram": mn, "square": (3 * K - 3) * mmm, "apply": mn}
    return {"gram": K * mn, "square": 0.0, "apply": K * mn}


def gram_sym_bytes(shapes):
    """bf16 bytes of the entries on and above each Gram's diagonal: what a
    pass of the power iteration must read of the symmetric Gram."""
    return sum(2.0 * min(r, c) * (min(r, c) + 1) / 2 for r, c in shapes)


def hbm_bytes_per_step(shapes, M, P, post_polar):
    """Algorithmic HBM bytes of each streaming kernel per step."""
    d = synth.numel(shapes)
    b = {
        "momentum": d * (14.0 * M + 4.0),          # G r, Mom r+w, X w (bf16) per worker; W r once
        "pack": d * M * (4.0 + 1.0 / 8.0),          # U r (fp32), bits w
        "power_iter": (P + 1) * M * gram_sym_bytes(shapes),
        # bits r; with the post-vote polar the majority goes straight to the
        # bf16 X of the polar step (2 B), else the update of W (8 B) is fused
        "vote": M * d / 8.0 + (2.0 * d if post_polar else 8.0 * d),
        "update": 12.0 * d,                         # W r+w, D r
    }
    if post_polar:
        b["power_iter"] += (P + 1) * gram_sym_bytes(shapes)
    return b


def max_over_ranks(x, device="cpu"):
    """The maximum of a per-rank float over all ranks of the process group
    (the slowest rank's time); the value itself on a single process."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, steps, ms):
    """Whole-job steps/s: every rank runs ``steps`` steps; ``ms`` is the max over ranks."""
    return world * steps / (ms / 1e3)


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
REASON_FIELDS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


class ClockSampler:
    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             + ",".join("clocks_event_reasons." + r for r in REASON_FIELDS))
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                          "-lms", "50", "-i", str(self.gpu_id)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], None, set()
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 5 + len(REASON_FIELDS):
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(REASON_FIELDS, parts[5:]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_smi_id(dev_index):
    import torch
    try:
        u = torch.cuda.get_device_properties(dev_index).uuid
        s = str(u)
        return s if s.startswith("GPU-") else "GPU-" + s
    except Exception:
        return str(dev_index)


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and --impl reference)
# ---------------------------------------------------------------------------
def cpu_oracle_sample(step_idx=0, precision="float32"):
    """One oracle step on the 768x768 attention projection of one layer for
    all 8 workers, including power iteration and the post-vote polar step;
    returns seconds.  Every nanoGPT matrix has 768 as its small side, so both
    the Newton-Schulz flops and the elementwise work of a matrix scale with
    its element count: this sample is exactly 1/144 of one whole step.
    precision: the oracle's arithmetic, float32 (the baseline) or float64
    (its parity mode)."""
    import numpy as np

    from oracle import signmuon_ref as ref
    shapes = [SHAPES[1]]
    w = synth.weights0(shapes, 3)
    G = synth.gradients(shapes, M, WL["sigma"], step=step_idx, config_id=3)
    mom = synth.momentum0(shapes, M, 3, scale=0.5)
    t0 = time.perf_counter()
    ref.step(w, G, mom, shapes, beta=HP["beta"], lam=HP["lam"], eta=HP["eta"], K=K_NS, eps=HP["eps"],
             scale=WL["scale"], P=WL["P"], post_polar=WL["post_polar"], dtype=getattr(np, precision))
    return time.perf_counter() - t0


CPU_SCALE = float(D) / (SHAPES[1][0] * SHAPES[1][1])  # 144


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


_SAMPLE = ("the 768x768 attention projection of one layer (589,824 weights, 1/144 of the model's "
           "weights and Newton-Schulz flops) x 8 workers, full oracle step incl. power iteration and "
           "post-vote polar, numpy float32{}; steps/s scaled by 1/144 to the whole model")
CPU_SAMPLE = _SAMPLE.format(" (float64 beside it)")
REF_SAMPLE = _SAMPLE.format("")


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    for i in range(args.warmup):
        cpu_oracle_sample(i)
    times = [cpu_oracle_sample(args.warmup + i) for i in range(args.steps)]
    sample_s = sum(times) / len(times)
    # each timed step is the 1/144 sample; the value is the whole workload's
    # rate, extrapolated by that factor (ms_per_step is what was timed)
    value = 1.0 / (CPU_SCALE * sample_s)
    cores = cpu_threads()
    extrap = f"x{CPU_SCALE:.0f}: value = 1 / ({CPU_SCALE:.0f} x the timed sample's mean seconds)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sample_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC, "sample": REF_SAMPLE},
        "sample": {"ms_per_sample_step": sample_s * 1e3, "fraction_of_step": 1.0 / CPU_SCALE,
                   "extrapolated": extrap},
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": cores, "kind": "oracle",
                         "sample": REF_SAMPLE, "precision": "float32", "extrapolated": extrap},
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the other configurations: short timed passes, each with its roofline
# fraction (folded into the headline line, and printed by --workload)
# ---------------------------------------------------------------------------
SWEEP_GRID = [(5, "cubic", "bf16"), (10, "cubic", "bf16"), (5, "quintic", "bf16"), (10, "quintic", "bf16"),
              (5, "cubic", "fp32"), (10, "cubic", "fp32"), (5, "quintic", "fp32"), (10, "quintic", "fp32")]


def _events_time(fn, reps, stream, warm=3):
    """Mean ms of fn() over reps calls, CUDA events on the given stream,
    after `warm` warm-up calls."""
    import torch
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def measure_resnet50(smo, stream, pk, steps=20):
    """The ResNet-50 step (M=4, K=5 cubic bf16, spectral P=2): steps/s, and
    its Newton-Schulz GEMMs' TFLOP/s from the library's per-kernel events."""
    import torch
    wl = synth.WORKLOADS["resnet50"]
    shp, Mr = wl["shapes"], wl["M"]
    h = smo.SignMuon(shp, Mr, beta=HP["beta"], lam=HP["lam"], K=wl["K"], eps=HP["eps"], scale=wl["scale"],
                     P=wl["P"], flags=0, stream=stream.cuda_stream)
    W = synth.device_weights0(shp, config_id=2)
    G = synth.device_gradients(shp, Mr, wl["sigma"], step=0, config_id=2)
    gl = [G[m] for m in range(Mr)]
    ms = _events_time(lambda: h.step(W, gl, HP["eta"]), steps, stream)
    h.profile(True)
    h.profile_read()
    for _ in range(steps):
        h.step(W, gl, HP["eta"])
    prof = h.profile_read()
    h.profile(False)
    gram_ns = bool(smo.signmuon_plan_tables(shp, Mr, wl["K"], wl["scale"], wl["P"], 0)["gram_ns"])
    fl = sum(ns_kind_flops(shp, Mr, wl["K"], gram_ns).values())
    gemm_ms = sum(prof[k][0] for k in ("ns_gram", "ns_square", "ns_apply")) / steps
    tf = fl / (gemm_ms / 1e3) / 1e12 if gemm_ms > 0 else None
    h.close()
    del W, G, gl
    torch.cuda.empty_cache()
    return {"metric": "Sign-Muon steps/s (ResNet-50 shapes, M=4, K=5 cubic bf16, spectral P=2)",
            "value": 1e3 / ms, "unit": "steps/s", "ms_per_step": ms, "d": synth.numel(shp),
            "ns_tflops_per_step": fl / 1e12, "ns_ms_per_step": gemm_ms, "ns_form": "gram space" if gram_ns else "x space",
            "ns_TFLOP/s": tf, "ns_frac_of_bf16_burst": (tf / pk["bf16_tflops"]) if tf else None,
            "ns_share_of_step": gemm_ms / ms}


def measure_llama_vote(smo, stream, pk, shapes=None, reps=5):
    """The LLaMA-layer vote stress (M=16 packed one-bit buffers, d =
    717,225,984): int32 and int8 sums + int8 majority, GB/s of algorithmic
    bytes (M d/8 read, 4d or d sums and d majority written)."""
    import torch
    shapes = shapes or synth.LLAMA_LAYER_SHAPES
    Mv = synth.WORKLOADS["llama_vote"]["M"]
    d = synth.numel(shapes)
    nb = (d + 7) // 8
    g = torch.Generator(device="cuda")
    g.manual_seed(4)
    signs = [torch.randint(0, 256, (nb + 16,), generator=g, device="cuda", dtype=torch.uint8) for _ in range(Mv)]
    out = []
    for acc8 in (False, True):
        h = smo.SignMuon(shapes, Mv, flags=smo.SIGNMUON_VOTE_ONLY | (smo.SIGNMUON_ACC_INT8 if acc8 else 0),
                         stream=stream.cuda_stream)
        sums = torch.empty(d, device="cuda", dtype=torch.int8 if acc8 else torch.int32)
        maj = torch.empty(d, device="cuda", dtype=torch.int8)
        ms = _events_time(lambda: h.vote(signs, d, sums, maj), reps, stream)
        nbytes = Mv * d / 8.0 + (1.0 if acc8 else 4.0) * d + d
        gbs = nbytes / (ms / 1e3) / 1e9
        out.append({"acc_dtype": "int8" if acc8 else "int32", "GB/s": gbs, "frac_of_hbm": gbs / pk["hbm_gbs"],
                    "ms": ms, "bytes": nbytes, "d": d, "M": Mv, "payload_bytes_per_worker": nb})
        h.close()
        del sums, maj
    del signs
    torch.cuda.empty_cache()
    return out


def measure_cublas_same_shapes(stream, pk, shapes=None, M=8, reps=20, settle_s=1.0):
    """cuBLAS (torch.bmm, bf16 in, fp32 accumulation, bf16 out) on the
    bench step's own Newton-Schulz GEMM shapes, for comparison with the
    library's tcgen05 kernel: per shape group, the Gram X X^T and the apply
    A X of all M workers' matrices as one batched call each.  TFLOP/s counts
    2 m^2 n per matrix for both (the algorithmic figure the library's own
    per-kernel numbers use; cuBLAS computes the whole Gram).  Each call runs
    for settle_s seconds before it is timed, so that the clock has settled
    under the power cap as it has in the library's step."""
    import time

    import torch
    shapes = shapes or SHAPES
    groups = {}
    for r, c in shapes:
        key = (min(r, c), max(r, c))
        groups[key] = groups.get(key, 0) + 1
    g = torch.Generator(device="cuda")
    g.manual_seed(6)
    res = {"gram_ms": 0.0, "apply_ms": 0.0, "flops": 0.0, "groups": []}
    for (m, n), cnt in sorted(groups.items()):
        b = cnt * M
        X = torch.randn(b, m, n, generator=g, device="cuda", dtype=torch.float32).to(torch.bfloat16)
        A = torch.empty(b, m, m, device="cuda", dtype=torch.bfloat16)
        Y = torch.empty_like(X)
        XT = X.transpose(1, 2)

        def settled(fn):
            t0 = time.perf_counter()
            while time.perf_counter() - t0 < settle_s:
                for _ in range(10):
                    fn()
                torch.cuda.synchronize()
            return _events_time(fn, reps, stream, warm=0)
        cs = ClockSampler(gpu_smi_id(torch.cuda.current_device()))
        cs.start()
        tg = settled(lambda: torch.bmm(X, XT, out=A))
        ta = settled(lambda: torch.bmm(A, X, out=Y))
        clk = cs.stop()
        fl = 2.0 * m * m * n * b
        res["gram_ms"] += tg
        res["apply_ms"] += ta
        res["flops"] += fl
        res["groups"].append({"m": m, "n": n, "batch": b, "gram_TFLOP/s": fl / (tg / 1e3) / 1e12,
                              "apply_TFLOP/s": fl / (ta / 1e3) / 1e12, "clocks": clk})
        del X, A, Y, XT
    torch.cuda.empty_cache()
    for k in ("gram", "apply"):
        tf = res["flops"] / (res[k + "_ms"] / 1e3) / 1e12
        res[k + "_TFLOP/s"] = tf
        res[k + "_frac_of_bf16_burst"] = tf / pk["bf16_tflops"]
    res["note"] = ("torch.bmm on the same (m, n) groups, M = %d workers per call; one Newton-Schulz iteration's "
                   "two GEMMs; each call timed after %.1f s of the same call" % (M, settle_s))
    return res


def measure_ns_sweep(smo, stream, pk, grid=SWEEP_GRID):
    """The Newton-Schulz sweep: TFLOP/s of PolarNS (spectral P=2) on one
    8192^2 matrix, 64 x 1024^2 and 256 x 512x2048, M=8 workers of Gaussian
    input, over K in {5, 10}, cubic and quintic, bf16 (tcgen05) and fp32
    (SIMT).  Flops per iteration and matrix: 4 m^2 n (cubic), 4 m^2 n + 2 m^3
    (quintic), m = min dim, n = max dim.  The fp32 8192^2 case is timed with
    one worker (one 8192^2 matrix already fills the GPU with tiles) to bound
    the run; its flop rate is per worker like the others."""
    import torch
    out = []
    for K, order, prec in grid:
        for name, shp in synth.SWEEP_SHAPES.items():
            Mw = 1 if (prec == "fp32" and name == "single_8192") else 8
            fl_ns = (smo.SIGNMUON_NS_QUINTIC if order == "quintic" else 0) | \
                    (smo.SIGNMUON_NS_FP32 if prec == "fp32" else 0)
            h = smo.SignMuon(shp, Mw, beta=0.9, lam=0.0, K=K, eps=1e-7, scale="spectral", P=2, flags=fl_ns,
                             stream=stream.cuda_stream)
            X = synth.device_gaussian(h.d, Mw, seed=5)
            U = torch.empty_like(X)
            xs, us = [X[m] for m in range(Mw)], [U[m] for m in range(Mw)]
            reps, warm = (3, 1) if prec == "bf16" else (1, 1)
            ms = _events_time(lambda: h.polar(xs, us), reps, stream, warm=warm)
            gram_ns = bool(smo.signmuon_plan_tables(shp, Mw, K, "spectral", 2, fl_ns)["gram_ns"])
            if gram_ns:
                fl = sum(ns_kind_flops(shp, Mw, K, True).values())
            else:
                per_it = sum(4.0 * min(r, c) ** 2 * max(r, c) + (2.0 * min(r, c) ** 3 if order == "quintic" else 0.0)
                             for r, c in shp)
                fl = per_it * K * Mw
            tf = fl / (ms / 1e3) / 1e12
            e = {"shape": name, "K": K, "order": order, "precision": prec, "M": Mw, "TFLOP/s": tf, "ms": ms,
                 "flops": fl, "ns_form": "gram space" if gram_ns else "x space"}
            if prec == "bf16":
                e["frac_of_bf16_burst"] = tf / pk["bf16_tflops"]
            else:
                e["frac_of_fp32_simt_peak"] = tf / FP32_SIMT_PEAK_TFLOPS
            out.append(e)
            h.close()
            del X, U, xs, us
            torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    import sign_muon_optimizer_b200 as smo

    stream = torch.cuda.current_stream()
    # SIGNMUON_ASYNC: the step does not wait for the GPU after each call; the
    # device still checks the momentum norms every step (a non-finite one
    # leaves W untouched) and signmuon_sync reads that status once, inside
    # the timed region
    flags = (smo.SIGNMUON_POST_POLAR if WL["post_polar"] else 0) | smo.SIGNMUON_ASYNC
    opt = smo.SignMuon(SHAPES, M, beta=HP["beta"], lam=HP["lam"], K=K_NS, eps=HP["eps"], scale=WL["scale"],
                       P=WL["P"], flags=flags, stream=stream.cuda_stream)
    W = synth.device_weights0(SHAPES, config_id=3 + rank)
    pool = [synth.device_gradients(SHAPES, M, WL["sigma"], step=s, config_id=3 + rank) for s in range(2)]
    gptrs = [[pool[s][m] for m in range(M)] for s in range(2)]
    torch.cuda.synchronize()

    for i in range(args.warmup):
        opt.step(W, gptrs[i % 2], HP["eta"])
    opt.sync()
    launches0 = smo.signmuon_kernel_launches()
    sampler = ClockSampler(gpu_smi_id(local))
    sampler.start()
    time.sleep(0.2)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(args.steps):
        opt.step(W, gptrs[i % 2], HP["eta"])
    opt.sync()   # raises if any timed step saw a non-finite momentum norm
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    launches = smo.signmuon_kernel_launches() - launches0
    ms = max_over_ranks(ev0.elapsed_time(ev1), "cuda")
    # per-kernel breakdown: the same steps again with an event pair around
    # every launch (outside the timed region: the events serialise the stream)
    opt.profile(True)
    opt.profile_read()
    for i in range(args.steps):
        opt.step(W, gptrs[i % 2], HP["eta"])
    opt.sync()
    prof = opt.profile_read()
    opt.profile(False)
    ms_per_step = ms / args.steps
    value = job_throughput(world, args.steps, ms)

    pk, pk_kind = peaks()
    steps = args.steps
    gram_ns = bool(smo.signmuon_plan_tables(SHAPES, M, K_NS, WL["scale"], WL["P"], flags)["gram_ns"])
    kind_fl = {"ns_" + k: v for k, v in ns_kind_flops(SHAPES, M, K_NS, gram_ns).items()}
    if WL["post_polar"]:
        kind_fl.update({"post_" + k: v for k, v in ns_kind_flops(SHAPES, 1, K_NS, gram_ns).items()})
    flops = sum(kind_fl.values())                 # as run: X space or Gram space
    gemm_kinds = ["ns_gram", "ns_square", "ns_apply", "post_gram", "post_square", "post_apply"]
    gemm_ms = sum(prof[k][0] for k in gemm_kinds)
    gemm_launches = sum(prof[k][1] for k in gemm_kinds)
    tflops = flops * steps / (gemm_ms / 1e3) / 1e12 if gemm_ms > 0 else None
    # the burst peak is the denominator; frac_of_sustained gives the same
    # against the power-capped figure that a seconds-long loop settles at
    peak_tc = pk["bf16_tflops"]
    roofline = {"kernel": "k_gemm_tc (grouped Newton-Schulz GEMM, tcgen05)", "bound": "tensor",
                "achieved": tflops, "peak": peak_tc, "unit": "TFLOP/s",
                "frac": (tflops / peak_tc) if tflops else None, "traffic": gemm_traffic_from_profile(),
                "peak_kind": f"bf16 burst, {pk_kind}",
                "flops_per_launch": flops / max(1, gemm_launches / steps),
                "avg_launch_ms": gemm_ms / max(1, gemm_launches),
                "timed_region_ms": ms,
                "frac_of_sustained": (tflops / pk["bf16_tflops_sustained"]) if tflops else None}
    hbm = hbm_bytes_per_step(SHAPES, M, WL["P"], WL["post_polar"])
    kernels = {}
    for kind, (kms, n) in prof.items():
        if n == 0:
            continue
        e = {"ms_per_step": kms / steps, "launches_per_step": n / steps}
        if kind in gemm_kinds:
            if kind_fl.get(kind):
                e["TFLOP/s"] = kind_fl[kind] / (kms / steps / 1e3) / 1e12
                e["frac_of_bf16_burst"] = e["TFLOP/s"] / peak_tc
        elif kind in hbm:
            e["GB/s"] = hbm[kind] / (kms / steps / 1e3) / 1e9
            e["frac_of_hbm"] = e["GB/s"] / pk["hbm_gbs"]
        kernels[kind] = e

    # end to end through the public API with host buffers (pinned)
    e2e = None
    if args.e2e_steps > 0:
        Wh = torch.empty(D, dtype=torch.float32, pin_memory=True)
        Wh.copy_(W)
        Gh = [torch.empty(D, dtype=torch.float32, pin_memory=True) for _ in range(M)]
        for m in range(M):
            Gh[m].copy_(pool[0][m])
        Wn, Gn = Wh.numpy(), [g.numpy() for g in Gh]
        opt.step_host(Wn, Gn, HP["eta"])
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        ev0.record(stream)
        for i in range(args.e2e_steps):
            opt.step_host(Wn, Gn, HP["eta"])
        ev1.record(stream)
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
        opt.sync()
        ems = max_over_ranks(max(ev0.elapsed_time(ev1), wall * 1e3), "cuda")
        # the copy link alone: the same host-to-device bytes as plain pinned copies
        h2d = (M + 1) * D * 4
        dst = torch.empty(D, dtype=torch.float32, device="cuda")
        dst.copy_(Gh[0], non_blocking=True)
        torch.cuda.synchronize()
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record()
        for src in [Wh] + Gh:
            dst.copy_(src, non_blocking=True)
        c1.record()
        torch.cuda.synchronize()
        h2d_gbs = h2d / (c0.elapsed_time(c1) / 1e3) / 1e9
        del dst
        e2e = {"value": job_throughput(world, args.e2e_steps, ems), "unit": "steps/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": D * 4,
               "h2d_copy_GBps": h2d_gbs, "copy_bound_steps_per_s": h2d_gbs * 1e9 / h2d,
               "api": "signmuon_step_host (pinned host W and G) with SIGNMUON_ASYNC: each step's gradients "
                      "come in on a copy stream while the step before runs and its W goes back; "
                      "copy_bound_steps_per_s = the host-to-device bytes alone at the rate of plain pinned copies"}
        del Gh, Wh

    # the other configurations (N = 1 only: the scaling runs time the headline alone)
    extras = None
    if rank == 0 and world == 1 and not args.no_extras:
        extras = {"resnet50": measure_resnet50(smo, stream, pk),
                  "llama_vote": measure_llama_vote(smo, stream, pk),
                  "ns_sweep": measure_ns_sweep(smo, stream, pk),
                  "cublas_same_shapes": measure_cublas_same_shapes(stream, pk)}

    if extras and extras.get("cublas_same_shapes") and kernels.get("ns_apply") and kernels.get("ns_gram"):
        # the same GEMM shapes through cuBLAS at the same power-capped clock
        cb = extras["cublas_same_shapes"]
        roofline["vs_cublas_same_shapes"] = {
            "apply": kernels["ns_apply"]["TFLOP/s"] / cb["apply_TFLOP/s"],
            "gram": kernels["ns_gram"]["TFLOP/s"] / cb["gram_TFLOP/s"],
            "note": "library TFLOP/s / cuBLAS TFLOP/s, both algorithmic 2 m^2 n per matrix"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t32 = 0.5 * (cpu_oracle_sample(0, "float32") + cpu_oracle_sample(1, "float32"))
        t64 = 0.5 * (cpu_oracle_sample(0, "float64") + cpu_oracle_sample(1, "float64"))
        cpu = {"value": 1.0 / (CPU_SCALE * t32), "unit": "steps/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": CPU_SAMPLE, "precision": "float32",
               "extrapolated": f"x{CPU_SCALE:.0f}: the sample's mean seconds times {CPU_SCALE:.0f}",
               "sample_s": t32,
               "float64": {"value": 1.0 / (CPU_SCALE * t64), "unit": "steps/s", "sample_s": t64}}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD_DESC, "M": M, "d": D,
                       "api": "signmuon_step with SIGNMUON_ASYNC; signmuon_sync once at the end of the timed steps",
                       "l2": "inputs larger than L2: 2.72 GB of gradients per step, two alternating sets",
                       "parallelism": "replicas" if world > 1 else "single GPU"},
            "roofline": roofline,
            # the same fraction against NVIDIA's nominal dense bf16 figure (context only)
            "roofline_spec": {"peak": 2250.0, "unit": "TFLOP/s", "kind": "nominal dense bf16",
                              "frac": (tflops / 2250.0) if tflops else None},
            # the vote's payload as the pages count it (no network: M workers on one GPU)
            "vote": {"payload_bytes_per_worker": (D + 7) // 8, "M": M, "acc_dtype": "int32 (byte-lane counters)",
                     "collective": "none (on-device vote)"},
            "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "clocks": clocks,
            "ns_tflops_per_step": flops / 1e12,
            # the Newton-Schulz form the planner chose, and the flops the same
            # iteration would take on X (context for the Gram-space form)
            "ns_form": "gram space" if gram_ns else "x space",
            "ns_tflops_per_step_on_x": ns_flops_per_step(SHAPES, M, K_NS, WL["post_polar"]) / 1e12,
            "workloads": extras,
        }
        print(json.dumps(line), flush=True)
    opt.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_secondary(args):
    """Secondary measurements (not the headline line): the LLaMA-layer vote
    (vote GB/s, one-bit and int8 ternary signs), the Newton-Schulz sweep (NS
    TFLOP/s), the ResNet-50 step and the named variants of the nanoGPT step
    (steps/s), one JSON line each."""
    import torch
    import sign_muon_optimizer_b200 as smo
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    pk, pk_kind = peaks()
    lines = []
    if args.workload in ("llama_vote", "vote_100m", "all"):
        # vote_100m: the same kernel on one 1 x 100,000,000 matrix (a small
        # case for profiler captures)
        small = args.workload == "vote_100m"
        shp_name = "1 x 100,000,000" if small else "LLaMA-layer shapes"
        for e in measure_llama_vote(smo, stream, pk, [(1, 100_000_000)] if small else None):
            lines.append(dict({"metric": f"vote GB/s ({shp_name}, M=16, {e['acc_dtype']} sums)", "value": e["GB/s"],
                               "unit": "GB/s", "peak_kind": pk_kind, "collective": "none (on-device vote)"}, **e))
    if args.workload in ("ns_sweep", "ns_sweep_full", "all"):
        # ns_sweep: K = 5 cubic bf16; ns_sweep_full: the sweep's whole grid
        grid = SWEEP_GRID if args.workload == "ns_sweep_full" else [(5, "cubic", "bf16")]
        for e in measure_ns_sweep(smo, stream, pk, grid):
            lines.append(dict({"metric": f"NS TFLOP/s ({e['shape']}, M={e['M']}, K={e['K']} {e['order']} "
                                         f"{e['precision']}, spectral P=2)", "value": e["TFLOP/s"],
                               "unit": "TFLOP/s", "peak_kind": pk_kind}, **e))
    if args.workload in ("ternary_vote", "all"):
        # the int8 ternary wire's vote: d bytes per worker instead of d/8
        shapes = synth.LLAMA_LAYER_SHAPES
        Mv = synth.WORKLOADS["llama_vote"]["M"]
        d = synth.numel(shapes)
        g = torch.Generator(device="cuda")
        g.manual_seed(6)
        signs = [torch.randint(-1, 2, (d + 16,), generator=g, device="cuda", dtype=torch.int8) for _ in range(Mv)]
        h = smo.SignMuon(shapes, Mv, flags=smo.SIGNMUON_VOTE_ONLY, stream=stream.cuda_stream)
        sums = torch.empty(d, device="cuda", dtype=torch.int32)
        maj = torch.empty(d, device="cuda", dtype=torch.int8)
        ms = _events_time(lambda: h.vote_ternary(signs, d, sums, maj), 5, stream)
        nbytes = Mv * d + 4.0 * d + d
        gbs = nbytes / (ms / 1e3) / 1e9
        lines.append({"metric": "ternary vote GB/s (LLaMA-layer shapes, M=16, int8 signs, int32 sums)", "value": gbs,
                      "unit": "GB/s", "frac_of_hbm": gbs / pk["hbm_gbs"], "peak_kind": pk_kind, "ms": ms,
                      "bytes": nbytes, "d": d, "M": Mv, "payload_bytes_per_worker": d, "acc_dtype": "int32",
                      "collective": "none (on-device vote)"})
        h.close()
        del signs, sums, maj
        torch.cuda.empty_cache()
    if args.workload in ("variants", "all"):
        # the named variants on the headline shapes (nanoGPT, M=8, K=5), one
        # step each; split = local signs + vote step through a caller buffer
        base = smo.SIGNMUON_POST_POLAR if WL["post_polar"] else 0
        variants = [("sign-muon", base, WL["P"]), ("tie_plus", base | smo.SIGNMUON_TIE_PLUS, WL["P"]),
                    ("ternary", base | smo.SIGNMUON_TERNARY, WL["P"]),
                    ("normalized_sign", smo.SIGNMUON_NORMALIZED_SIGN, WL["P"]),
                    ("after_only", smo.SIGNMUON_POST_POLAR | smo.SIGNMUON_POLAR_AFTER_ONLY, WL["P"]),
                    ("muon_mean", smo.SIGNMUON_MUON_MEAN, WL["P"]),
                    ("pi_warm_P1", base | smo.SIGNMUON_PI_WARM, 1), ("cold_P1", base, 1), ("split", base, WL["P"]),
                    ("gram_space_ns", base | smo.SIGNMUON_NS_GRAM, WL["P"]),
                    ("cuda_graph", base | smo.SIGNMUON_ASYNC, WL["P"])]
        W = synth.device_weights0(SHAPES, config_id=7)
        G = synth.device_gradients(SHAPES, M, WL["sigma"], step=0, config_id=7)
        gl = [G[m] for m in range(M)]
        for name, flags, P in variants:
            # a graph is captured on a stream of its own (not the legacy default stream)
            vs = torch.cuda.Stream() if name == "cuda_graph" else stream
            h = smo.SignMuon(SHAPES, M, beta=HP["beta"], lam=HP["lam"], K=K_NS, eps=HP["eps"], scale=WL["scale"],
                             P=P, flags=flags, stream=vs.cuda_stream)
            if name == "split":
                buf = torch.empty(M * h.sign_stride(), dtype=torch.uint8, device="cuda")

                def one():
                    h.local_signs(W, gl, buf)
                    h.vote_step(W, buf, M, HP["eta"])
            elif name == "cuda_graph":
                # the whole step captured once on the handle's stream, then replayed
                h.step(W, gl, HP["eta"])
                h.sync()
                torch.cuda.synchronize()
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph, stream=vs):
                    h.step(W, gl, HP["eta"])

                def one():
                    with torch.cuda.stream(vs):
                        graph.replay()
            else:
                def one():
                    h.step(W, gl, HP["eta"])
            ms = _events_time(one, 10, vs)
            lines.append({"metric": f"Sign-Muon steps/s (nanoGPT-124M shapes, M=8, variant {name})",
                          "value": 1e3 / ms, "unit": "steps/s", "ms_per_step": ms, "flags": flags, "P": P})
            if name == "cuda_graph":
                h.sync()
                del graph
            h.close()
        del W, G, gl
        torch.cuda.empty_cache()
    if args.workload in ("resnet50", "all"):
        lines.append(measure_resnet50(smo, stream, pk))
    if args.workload in ("cublas", "all"):
        c = measure_cublas_same_shapes(stream, pk)
        lines.append(dict({"metric": "cuBLAS TFLOP/s on the nanoGPT step's Newton-Schulz shapes (M=8, bf16)",
                           "value": c["apply_TFLOP/s"], "unit": "TFLOP/s", "peak_kind": pk_kind}, **c))
    for ln in lines:
        print(json.dumps(ln), flush=True)
    return 0


def run_collectives(args):
    """The exchange of the multi-GPU step on its own (one JSON line from rank
    0; run under torchrun with N >= 2): the all-gather of packed signs and
    the SUM all-reduce of int8 sums timed over NCCL at message sizes from
    1 KB to 256 MB (max over ranks), the alpha-beta fit t = alpha + beta * n
    of each, and the fitted time of the nanoGPT payloads (ceil(d/8) bytes
    per rank gathered, d int8 bytes reduced) next to a direct measurement."""
    import datetime

    import torch
    import torch.distributed as dist

    from sign_muon_optimizer_b200.dist import fit_alpha_beta, time_collective
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world < 2:
        print(json.dumps({"metric": "exchange alpha-beta fit", "unavailable": "needs 2 or more ranks (torchrun)"}),
              flush=True)
        return 0
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
        device = f"cuda:{local}"
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        sizes = [1 << k for k in range(10, 29, 2)]
    else:  # the same exchange over gloo on the host (a check of this code path)
        device = "cpu"
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
        sizes = [1 << k for k in range(10, 21, 2)]
    packed, sums8 = (D + 7) // 8, D
    out = {"metric": "exchange alpha-beta fit", "n_gpus": world, "device": device, "sizes_bytes": sizes}
    for kind, payload in (("allgather", packed), ("allreduce", sums8)):
        ts = time_collective(kind, sizes, reps=5, device=device)
        alpha, beta = fit_alpha_beta(sizes, ts)
        direct = time_collective(kind, [payload], reps=2, device=device)[0]
        out[kind] = {"seconds": ts, "alpha_s": alpha, "beta_s_per_byte": beta,
                     "GB_per_s": (1.0 / beta / 1e9) if beta > 0 else None,
                     "nanogpt_payload_bytes": payload, "fitted_s": alpha + beta * payload, "measured_s": direct}
    if rank == 0:
        print(json.dumps(out), flush=True)
    dist.barrier()
    dist.destroy_process_group()
    return 0


def run_capture(args):
    """Profiler-capture mode (prints no bench line): the same step on the first
    L transformer layers of the nanoGPT shapes, M=8, a few steps.  Variants:
    "ternary" sends int8 ternary signs (written by the last GEMM, then the
    ternary vote kernels); "ragged" adds a 48-column matrix, so that the last
    GEMM's 32-column chunks straddle words of the bit stream (OR-ed in);
    "fp32" and "ternary-fp32" run the fp32 Newton-Schulz path, whose signs
    come from the pack and ternary sign kernels."""
    import torch
    import sign_muon_optimizer_b200 as smo
    shapes = SHAPES[: 4 * args.capture_layers]
    flags = smo.SIGNMUON_POST_POLAR if WL["post_polar"] else 0
    if args.capture_variant in ("ternary", "ternary-fp32"):
        flags |= smo.SIGNMUON_TERNARY
    if args.capture_variant in ("fp32", "ternary-fp32"):
        flags |= smo.SIGNMUON_NS_FP32
    if args.capture_variant == "ragged":
        shapes = shapes + [(768, 48)]
    opt = smo.SignMuon(shapes, M, beta=HP["beta"], lam=HP["lam"], K=K_NS, eps=HP["eps"], scale=WL["scale"],
                       P=WL["P"], flags=flags)
    W = synth.device_weights0(shapes, config_id=3)
    G = synth.device_gradients(shapes, M, WL["sigma"], step=0, config_id=3)
    for _ in range(args.steps):
        opt.step(W, [G[m] for m in range(M)], HP["eta"])
    torch.cuda.synchronize()
    print(f"capture run done: {len(shapes)} matrices, {args.steps} steps, "
          f"{smo.signmuon_kernel_launches()} kernel launches")
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the short passes of the ResNet-50, LLaMA-layer vote and NS sweep configurations")
    ap.add_argument("--capture-layers", type=int, default=0,
                    help="profiler capture mode on the first L layers; prints no bench line")
    ap.add_argument("--capture-variant", default="nanogpt", choices=["nanogpt", "ternary", "ragged", "fp32", "ternary-fp32"])
    ap.add_argument("--workload", default="nanogpt",
                    choices=["nanogpt", "llama_vote", "vote_100m", "ns_sweep", "ns_sweep_full", "resnet50",
                             "ternary_vote", "variants", "collectives", "cublas", "all"],
                    help="nanogpt: the headline line; the others print secondary measurements only")
    args = ap.parse_args()
    if args.capture_layers > 0:
        return run_capture(args)
    if args.workload == "collectives":
        return run_collectives(args)
    if args.workload != "nanogpt":
        return run_secondary(args)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
