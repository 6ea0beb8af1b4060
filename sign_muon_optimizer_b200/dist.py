"""Sign-Muon across GPUs: each rank holds some of the workers.

[paper] "SignMuon: 通信高效的分布式Muon优化" Algorithm 2: every worker computes its
momentum, polar factor and signs locally; the signs cross the network once;
every worker takes the majority and updates its own copy of W.  [blog]
"SignMuon: Matrix Directions, Majority Votes, and the Actual Bytes Sent" counts
the payload: ceil(d/8) bytes per worker for the packed bits, gathered from all
ranks (an all-gather; every rank then votes locally).

Three exchanges are offered:
- "allgather": every rank gathers all workers' packed (or int8 ternary) signs
  and votes over them.  The payload is M_local * ceil(d/8) bytes per rank.
- "allreduce": each rank adds up its own workers' signs, and an integer SUM
  all-reduce adds the ranks' sums (Algorithm 2's form).  The payload is d
  bytes per rank with int8 sums (SIGNMUON_ACC_INT8, at most 127 workers in
  all), or 4d with int32 sums.
- "peer": no data collective at all.  Each rank's sign buffers are mapped
  into every other rank once (CUDA IPC); every step the vote kernel reads
  all ranks' packed bits directly, over NVLink for the peers' (loads only, no
  multicast).  The buffers alternate between two slots from step to step, so
  that the status all-reduce of a step, which every rank enters only after
  its previous vote finished, is the only synchronisation needed: a rank
  writes slot t % 2 at step t while its peers may still read slot (t-1) % 2.

This module is plumbing only.  The arithmetic runs in libsignmuon.so:
signmuon_local_signs before the exchange; after it, signmuon_vote_step, or
signmuon_vote / signmuon_vote_ternary then signmuon_sums_step.
torch.distributed moves the bytes, plus one all-reduce of a status flag.
The flag lets every rank take the same collective path when one rank's
momentum turns non-finite.  Ranks must call step() in lockstep, with the
same shapes, flags and exchange.
"""
from __future__ import annotations

import contextlib
import time

import numpy as np
import torch
import torch.distributed as dist

from . import (SIGNMUON_ACC_INT8, SIGNMUON_ASYNC, SIGNMUON_E_NONFINITE, SIGNMUON_TERNARY, SignMuon, SignMuonError,
               signmuon_ipc_close, signmuon_ipc_get_handle, signmuon_ipc_open)


class DistSignMuon:
    """One rank's share of an M = world_size * M_local worker Sign-Muon step.

    ``step(W, G, eta)`` takes this rank's replica of W (device float[d]) and
    its M_local gradients, and leaves W equal on every rank.  The global
    worker order is rank-major: rank r holds workers r*M_local ...
    (r+1)*M_local - 1.  ``exchange`` is "allgather" or "allreduce" (see the
    module text).  ``opt`` may be given to reuse an existing handle, or any
    object with the same methods (local_signs, vote_step, vote_step_ptrs,
    vote, vote_ternary, sums_step, sign_stride, and sync for a handle made
    with SIGNMUON_ASYNC) and attributes (d, flags).  ``ipc`` replaces the CUDA
    IPC mapping of the "peer" exchange (an object with alloc, handle,
    address, open and close).  With SIGNMUON_ASYNC every step waits for the
    local half's status before the exchange, so that a failed rank stops all
    ranks as it does without the flag.
    """

    def __init__(self, shapes, M_local=1, beta=0.9, lam=0.01, K=5, eps=1e-7, scale="fro", P=1, flags=0,
                 group=None, device=None, opt=None, exchange="allgather", ipc=None):
        if exchange not in ("allgather", "allreduce", "peer"):
            raise ValueError(f"unknown exchange {exchange!r}")
        self.exchange = exchange
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.M_local = int(M_local)
        self.M = self.world * self.M_local
        if self.M > 256:
            raise ValueError(f"{self.M} workers in all; the vote takes at most 256")
        self.opt = opt if opt is not None else SignMuon(shapes, M_local, beta, lam, K, eps, scale, P, flags)
        self.stride = int(self.opt.sign_stride())
        if device is None:
            device = torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else "cpu"
        self.device = torch.device(device)
        self.local = torch.zeros(self.M_local * self.stride, dtype=torch.uint8, device=self.device)
        self._flag = torch.zeros(1, dtype=torch.int32, device=self.device)
        # torch orders its collectives after the current stream; make that the
        # handle's stream, so that the exchange waits for the library's kernels
        # and the vote after it waits for the exchange
        self._stream = None
        if self.device.type == "cuda":
            ptr = getattr(self.opt, "stream", None)
            self._stream = (torch.cuda.ExternalStream(ptr, device=self.device) if ptr
                            else torch.cuda.default_stream(self.device))
        flags = int(getattr(self.opt, "flags", flags))
        self.ternary = bool(flags & SIGNMUON_TERNARY)
        # An asynchronous handle returns from local_signs before its status is
        # known; the status all-reduce must carry that status, so the step
        # waits for it (signmuon_sync) before the flag is set.
        self.async_status = bool(flags & SIGNMUON_ASYNC)
        if exchange == "allgather":
            self.gathered = torch.zeros(self.M * self.stride, dtype=torch.uint8, device=self.device)
        elif exchange == "peer":
            self.ipc = ipc if ipc is not None else _CudaIpc()
            self.slots = [self.ipc.alloc(self.M_local * self.stride, self.device) for _ in range(2)]
            mine = [self.ipc.handle(b) for b in self.slots]
            everyone = [None] * self.world
            dist.all_gather_object(everyone, mine, group=self.group)
            # slot_ptr[r][k]: the address, in this process, of rank r's slot k
            self.slot_ptr = []
            for r in range(self.world):
                if r == self.rank:
                    self.slot_ptr.append([self.ipc.address(b) for b in self.slots])
                else:
                    self.slot_ptr.append([self.ipc.open(hd) for hd in everyone[r]])
            self.t = 0
        else:
            acc8 = bool(flags & SIGNMUON_ACC_INT8)
            if acc8 and self.M > 127:
                raise ValueError(f"int8 sums overflow for {self.M} workers (at most 127)")
            self.sums = torch.zeros(int(self.opt.d), dtype=torch.int8 if acc8 else torch.int32, device=self.device)
            self.views = [self.local[m * self.stride:] for m in range(self.M_local)]

    @property
    def payload_bytes(self):
        """Bytes each rank contributes to the exchange per step (for "peer",
        the bytes of its signs that every other rank reads)."""
        if self.exchange in ("allgather", "peer"):
            return self.local.numel()
        return self.sums.numel() * self.sums.element_size()

    def close(self):
        """Unmap the peers' sign buffers ("peer" exchange)."""
        if self.exchange == "peer":
            for r, ptrs in enumerate(self.slot_ptr):
                if r != self.rank:
                    for p in ptrs:
                        self.ipc.close(p)
            self.slot_ptr = []

    def step(self, W, G, eta, clocks=None):
        """One step.  With a ``clocks`` dict, adds this step's phase times in
        ms to its keys ([blog] "The experiment needs three clocks"; the
        gradient clock is the caller's):
        - local_ms: momentum, polar factor and signs, the status all-reduce,
          and, for the all-reduce exchange, the local vote;
        - exchange_ms: the all-gather or the SUM all-reduce;
        - finish_ms: the vote or majority, the post-vote step and the update;
        - total_ms: the whole step."""
        with torch.cuda.stream(self._stream) if self._stream is not None else contextlib.nullcontext():
            self._step(W, G, eta, clocks)

    def _step(self, W, G, eta, clocks):
        clk = _PhaseClock(self.device) if clocks is not None else None
        t0 = clk.mark() if clk else None
        err = None
        if self.exchange == "peer":
            slot = self.t % 2
            self.t += 1
            own = self.slots[slot]
        else:
            own = self.local
        try:
            self.opt.local_signs(W, G, own, self.stride)
            if self.async_status:
                # raises the deferred error of this call (or of an earlier
                # asynchronous call on the handle) before the flag is set
                self.opt.sync()
            self._flag.fill_(1)
        except SignMuonError as e:
            err = e
            self._flag.fill_(0)
        # every rank takes this collective, and the next one only if all are ok
        dist.all_reduce(self._flag, op=dist.ReduceOp.MIN, group=self.group)
        if int(self._flag.item()) == 0:
            if err is not None:
                raise err
            raise SignMuonError(SIGNMUON_E_NONFINITE, "another rank's step failed; W was not updated")
        if self.exchange == "allgather":
            t1 = clk.mark() if clk else None
            dist.all_gather_into_tensor(self.gathered, self.local, group=self.group)
            t2 = clk.mark() if clk else None
            self.opt.vote_step(W, self.gathered, self.M, eta, self.stride)
        elif self.exchange == "peer":
            # every rank's signs of this step are complete (the all-reduce
            # above); the vote reads them where they are, rank-major
            t1 = t2 = clk.mark() if clk else None
            ptrs = [self.slot_ptr[r][slot] + m * self.stride for r in range(self.world) for m in range(self.M_local)]
            self.opt.vote_step_ptrs(W, ptrs, eta)
        else:
            d = int(self.opt.d)
            if self.ternary:
                self.opt.vote_ternary(self.views, d, self.sums, None)
            else:
                self.opt.vote(self.views, d, self.sums, None)
            t1 = clk.mark() if clk else None
            dist.all_reduce(self.sums, op=dist.ReduceOp.SUM, group=self.group)
            t2 = clk.mark() if clk else None
            self.opt.sums_step(W, self.sums, eta)
        if clk:
            t3 = clk.mark()
            for key, a, b in (("local_ms", t0, t1), ("exchange_ms", t1, t2), ("finish_ms", t2, t3),
                              ("total_ms", t0, t3)):
                clocks[key] = clocks.get(key, 0.0) + clk.ms(a, b)

    def replicas_agree(self, W):
        """True on every rank when the ranks' W agree (the [blog] replica
        check): the min and max over ranks of two checksums of W's bit
        patterns (their sum and their sum of squares, wrapping in int64) must
        be equal."""
        bits = W.detach().contiguous().view(torch.int32).to(torch.int64)
        c = torch.stack([bits.sum(), (bits * bits).sum()])
        lo, hi = c.clone(), c.clone()
        dist.all_reduce(lo, op=dist.ReduceOp.MIN, group=self.group)
        dist.all_reduce(hi, op=dist.ReduceOp.MAX, group=self.group)
        return bool(torch.equal(lo, hi))


class _CudaIpc:
    """The sign buffers of the "peer" exchange: device allocations whose CUDA
    IPC handles the other ranks open (libsignmuon's signmuon_ipc_* calls)."""

    def alloc(self, nbytes, device):
        return torch.zeros(nbytes, dtype=torch.uint8, device=device)

    def handle(self, buf):
        return signmuon_ipc_get_handle(buf.data_ptr())

    def address(self, buf):
        return buf.data_ptr()

    def open(self, hd):
        handle, offset = hd
        base = signmuon_ipc_open(handle)
        self._bases = getattr(self, "_bases", {})
        self._bases[base + offset] = base
        return base + offset

    def close(self, ptr):
        base = self._bases.pop(ptr, None)
        if base is not None:
            signmuon_ipc_close(base)


class _PhaseClock:
    """Phase boundaries on the device (CUDA events on the current stream,
    read after a synchronize) or, for a CPU device, on the host clock."""

    def __init__(self, device):
        self.cuda = torch.device(device).type == "cuda"

    def mark(self):
        if self.cuda:
            e = torch.cuda.Event(enable_timing=True)
            e.record()
            return e
        return time.perf_counter()

    def ms(self, a, b):
        if self.cuda:
            b.synchronize()
            return float(a.elapsed_time(b))
        return (b - a) * 1e3


def fit_alpha_beta(nbytes, seconds):
    """Least-squares fit of the alpha-beta model t = alpha + beta * n ([paper]
    §6: alpha the start-up latency in s, beta the time per byte in s/byte)
    to collective timings at several message sizes."""
    n = np.asarray(nbytes, np.float64)
    t = np.asarray(seconds, np.float64)
    A = np.stack([np.ones_like(n), n], axis=1)
    (alpha, beta), *_ = np.linalg.lstsq(A, t, rcond=None)
    return float(alpha), float(beta)


def allreduce_time_model(alpha, beta, M, nbytes, rounds):
    """[paper] §6 per-iteration estimate of one all-reduce over M ranks:
    alpha * R(M) + 2 (1 - 1/M) * s * beta, with R(M) the rounds on the
    critical path and s the payload in bytes."""
    return alpha * rounds + 2.0 * (1.0 - 1.0 / M) * nbytes * beta


def time_collective(kind, nbytes_list, reps=5, group=None, device="cpu"):
    """Seconds per call of one collective at each message size, the max over
    ranks: kind "allgather" (each rank gives n uint8 bytes) or "allreduce"
    (a SUM over n int8 bytes).  One untimed call per size first."""
    world = dist.get_world_size(group)
    clk = _PhaseClock(device)
    out = []
    for n in nbytes_list:
        n = int(n)
        if kind == "allgather":
            src = torch.zeros(n, dtype=torch.uint8, device=device)
            dst = torch.zeros(n * world, dtype=torch.uint8, device=device)

            def call():
                dist.all_gather_into_tensor(dst, src, group=group)
        elif kind == "allreduce":
            buf = torch.zeros(n, dtype=torch.int8, device=device)

            def call():
                dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=group)
        else:
            raise ValueError(kind)
        call()
        dist.barrier(group=group)
        a = clk.mark()
        for _ in range(reps):
            call()
        b = clk.mark()
        t = torch.tensor([clk.ms(a, b) / 1e3 / reps], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
        out.append(float(t.item()))
    return out
