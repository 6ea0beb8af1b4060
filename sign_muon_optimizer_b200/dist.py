"""Sign-Muon across GPUs: each rank holds some of the workers.

[paper] "SignMuon: 通信高效的分布式Muon优化" Algorithm 2: every worker computes its
momentum, polar factor and signs locally; the signs cross the network once;
every worker takes the majority and updates its own copy of W.  [blog]
"SignMuon: Matrix Directions, Majority Votes, and the Actual Bytes Sent" counts
the payload: ceil(d/8) bytes per worker for the packed bits, gathered from all
ranks (an all-gather; every rank then votes locally).

This module is plumbing only.  The arithmetic runs in libsignmuon.so:
signmuon_local_signs before the exchange, and signmuon_vote_step after it.
torch.distributed moves the bytes: one all-gather of the packed (or int8
ternary) signs, plus one all-reduce of a status flag.  The flag lets every
rank take the same collective path when one rank's momentum turns
non-finite.  Ranks must call step() in lockstep, with the same shapes and flags.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import SIGNMUON_E_NONFINITE, SignMuon, SignMuonError


class DistSignMuon:
    """One rank's share of an M = world_size * M_local worker Sign-Muon step.

    ``step(W, G, eta)`` takes this rank's replica of W (device float[d]) and
    its M_local gradients, and leaves W equal on every rank.  The global
    worker order is rank-major: rank r holds workers r*M_local ...
    (r+1)*M_local - 1.  ``opt`` may be given to reuse an existing handle, or
    any object with the same local_signs / vote_step / sign_stride methods.
    """

    def __init__(self, shapes, M_local=1, beta=0.9, lam=0.01, K=5, eps=1e-7, scale="fro", P=1, flags=0,
                 group=None, device=None, opt=None):
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
        self.gathered = torch.zeros(self.M * self.stride, dtype=torch.uint8, device=self.device)
        self._flag = torch.zeros(1, dtype=torch.int32, device=self.device)

    @property
    def payload_bytes(self):
        """Bytes each rank contributes to the all-gather per step."""
        return self.local.numel()

    def step(self, W, G, eta):
        err = None
        try:
            self.opt.local_signs(W, G, self.local, self.stride)
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
        dist.all_gather_into_tensor(self.gathered, self.local, group=self.group)
        self.opt.vote_step(W, self.gathered, self.M, eta, self.stride)

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
