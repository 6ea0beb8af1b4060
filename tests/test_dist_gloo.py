"""The multi-GPU driver's exchange (sign_muon_optimizer_b200.dist) on the CPU:
world size 2 over gloo, with a stand-in for the library's two halves of the
step (the signs are the one-bit signs of the gradients themselves, and the
vote follows the oracle).  It checks what the driver itself adds: the
rank-major worker order of the all-gather, identical W on every rank (and
the replica check), and that a failure on one rank makes every rank raise
without updating W and without hanging in a collective."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import synth
from oracle import signmuon_ref as ref

SHAPES = [(6, 10), (9, 5)]
M_LOCAL = 2


class _StandIn:
    """local_signs / vote_step / vote / sums_step / sign_stride with the
    library's layout (int32 sums; flags 0)."""

    def __init__(self, fail=False, deferred=False):
        import sign_muon_optimizer_b200 as smo
        self.d = synth.numel(SHAPES)
        self.nb = ref.packed_nbytes(self.d)
        # deferred: behave like a handle made with SIGNMUON_ASYNC, whose
        # local_signs returns OK and whose sync() reports the failure
        self.flags = smo.SIGNMUON_ASYNC if deferred else 0
        self.fail = fail
        self.deferred = deferred
        self.pending = False
        self.seen = None

    def sign_stride(self):
        return (self.nb + 15) // 16 * 16

    def local_signs(self, W, G, out, stride):
        import sign_muon_optimizer_b200 as smo
        if self.fail and not self.deferred:
            raise smo.SignMuonError(smo.SIGNMUON_E_NONFINITE, "planted failure")
        self.pending = self.fail
        for m, g in enumerate(G):
            out[m * stride: m * stride + self.nb] = torch.from_numpy(ref.pack_bits(ref.sign_bits(g.numpy())))

    def sync(self):
        import sign_muon_optimizer_b200 as smo
        if self.pending:
            self.pending = False
            raise smo.SignMuonError(smo.SIGNMUON_E_NONFINITE, "planted deferred failure")

    def vote_step(self, W, signs, M, eta, stride):
        self.seen = signs.clone()
        packed = [signs[j * stride: j * stride + self.nb].numpy() for j in range(M)]
        maj = ref.majority(ref.vote_sums_from_bits(packed, self.d))
        W.copy_(torch.from_numpy(ref.update(W.numpy(), maj.astype(np.float32), eta)))

    def vote_step_ptrs(self, W, ptrs, eta):
        # the stand-in's "device pointers" are host addresses (file mappings)
        import ctypes
        packed = [np.frombuffer(ctypes.string_at(p, self.nb), dtype=np.uint8) for p in ptrs]
        self.seen = torch.from_numpy(np.concatenate(packed))
        maj = ref.majority(ref.vote_sums_from_bits(packed, self.d))
        W.copy_(torch.from_numpy(ref.update(W.numpy(), maj.astype(np.float32), eta)))

    def vote(self, views, d, sums, majority):
        sums.copy_(torch.from_numpy(ref.vote_sums_from_bits([v[: self.nb].numpy() for v in views], d)))

    def sums_step(self, W, sums, eta):
        self.seen = sums.clone()
        maj = ref.majority(sums.numpy())
        W.copy_(torch.from_numpy(ref.update(W.numpy(), maj.astype(np.float32), eta)))


class _FileIpc:
    """Stand-in for the CUDA IPC mapping of the "peer" exchange: each rank's
    buffers are shared files, mapped by every rank; a handle is the file name."""

    def __init__(self, root, rank):
        self.root, self.rank, self.n, self.keep = root, rank, 0, []

    def alloc(self, nbytes, device):
        path = os.path.join(self.root, f"rank{self.rank}_buf{self.n}")
        self.n += 1
        mm = np.memmap(path, dtype=np.uint8, mode="w+", shape=(nbytes,))
        self.keep.append(mm)
        t = torch.from_numpy(mm)
        t.path = path
        return t

    def handle(self, buf):
        return (buf.path, int(buf.numel()))

    def address(self, buf):
        return buf.data_ptr()

    def open(self, hd):
        path, n = hd
        mm = np.memmap(path, dtype=np.uint8, mode="r", shape=(n,))
        self.keep.append(mm)
        return mm.ctypes.data

    def close(self, ptr):
        pass


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, fail_rank, q, exchange="allgather", deferred=False, root=None, steps=1):
    import torch.distributed as dist

    from sign_muon_optimizer_b200.dist import DistSignMuon
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        opt = _StandIn(fail=(rank == fail_rank), deferred=deferred)
        ipc = _FileIpc(root, rank) if exchange == "peer" else None
        drv = DistSignMuon(SHAPES, M_local=M_LOCAL, opt=opt, device="cpu", exchange=exchange, ipc=ipc)
        W = torch.from_numpy(synth.weights0(SHAPES, 5))
        raised = False
        clocks = {}
        for step in range(1, steps + 1):
            G = synth.gradients(SHAPES, world * M_LOCAL, 1.0, step=step, config_id=5)
            mine = [torch.from_numpy(g) for g in G[rank * M_LOCAL:(rank + 1) * M_LOCAL]]
            try:
                drv.step(W, mine, 0.02, clocks=clocks)
            except Exception as e:  # noqa: BLE001
                raised = type(e).__name__
                break
        agree = drv.replicas_agree(W)
        q.put((rank, W.numpy().copy(), None if opt.seen is None else opt.seen.numpy(), raised, agree,
               drv.payload_bytes, clocks))
    finally:
        dist.destroy_process_group()


def _run(fail_rank, exchange="allgather", deferred=False, root=None, steps=1):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, fail_rank, q, exchange, deferred, root, steps))
             for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        r, W, seen, raised, agree, payload, clocks = q.get(timeout=120)
        out[r] = dict(W=W, seen=seen, raised=raised, agree=agree, payload=payload, clocks=clocks)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return out


def test_exchange_gathers_in_rank_order_and_replicas_agree():
    out = _run(fail_rank=-1)
    world = 2
    M = world * M_LOCAL
    G = synth.gradients(SHAPES, M, 1.0, step=1, config_id=5)
    d = synth.numel(SHAPES)
    nb = ref.packed_nbytes(d)
    stride = (nb + 15) // 16 * 16
    packed = [ref.pack_bits(ref.sign_bits(g)) for g in G]
    w0 = synth.weights0(SHAPES, 5)
    want = ref.update(w0, ref.majority(ref.vote_sums_from_bits(packed, d)).astype(np.float32), 0.02)
    for r in range(world):
        assert out[r]["raised"] is False
        assert out[r]["agree"] is True
        assert out[r]["payload"] == M_LOCAL * stride
        assert np.array_equal(out[r]["W"].view(np.uint32), want.view(np.uint32))
        for j in range(M):  # global worker j sits at slot j on every rank
            assert np.array_equal(out[r]["seen"][j * stride: j * stride + nb], packed[j])
        c = out[r]["clocks"]
        assert set(c) == {"local_ms", "exchange_ms", "finish_ms", "total_ms"}
        assert all(v >= 0.0 for v in c.values())
        assert abs(c["local_ms"] + c["exchange_ms"] + c["finish_ms"] - c["total_ms"]) <= 1e-6 * max(1.0, c["total_ms"])


def test_allreduce_exchange_adds_the_ranks_sums():
    # each rank sums its own two workers' signs; the SUM all-reduce must give
    # every rank the sums over all four workers, and the same W
    out = _run(fail_rank=-1, exchange="allreduce")
    M = 2 * M_LOCAL
    G = synth.gradients(SHAPES, M, 1.0, step=1, config_id=5)
    d = synth.numel(SHAPES)
    packed = [ref.pack_bits(ref.sign_bits(g)) for g in G]
    sums = ref.vote_sums_from_bits(packed, d)
    w0 = synth.weights0(SHAPES, 5)
    want = ref.update(w0, ref.majority(sums).astype(np.float32), 0.02)
    for r in range(2):
        assert out[r]["raised"] is False and out[r]["agree"] is True
        assert out[r]["payload"] == 4 * d       # int32 sums
        assert np.array_equal(out[r]["seen"], sums)
        assert np.array_equal(out[r]["W"].view(np.uint32), want.view(np.uint32))


def test_peer_exchange_votes_on_every_ranks_mapped_signs(tmp_path):
    """The "peer" exchange: no data collective, each rank's sign buffers are
    mapped by the other rank (here files stand in for CUDA IPC), the vote
    reads all four workers' signs in rank-major order, and the two buffer
    slots alternate: three steps must give both ranks the W of the oracle's
    three sequential votes."""
    out = _run(fail_rank=-1, exchange="peer", root=str(tmp_path), steps=3)
    M = 2 * M_LOCAL
    d = synth.numel(SHAPES)
    nb = ref.packed_nbytes(d)
    w = synth.weights0(SHAPES, 5)
    for step in (1, 2, 3):
        G = synth.gradients(SHAPES, M, 1.0, step=step, config_id=5)
        packed = [ref.pack_bits(ref.sign_bits(g)) for g in G]
        w = ref.update(w, ref.majority(ref.vote_sums_from_bits(packed, d)).astype(np.float32), 0.02)
    stride = (nb + 15) // 16 * 16
    for r in range(2):
        assert out[r]["raised"] is False and out[r]["agree"] is True
        assert out[r]["payload"] == M_LOCAL * stride
        assert np.array_equal(out[r]["W"].view(np.uint32), w.view(np.uint32))
        # the last vote saw worker j's signs at slot j (rank-major)
        for j in range(M):
            assert np.array_equal(out[r]["seen"][j * nb:(j + 1) * nb], packed[j])


@pytest.mark.parametrize("deferred", [False, True])
@pytest.mark.parametrize("exchange", ["allgather", "allreduce", "peer"])
def test_one_failing_rank_stops_every_rank_without_update(exchange, deferred, tmp_path):
    # deferred: the failing rank's handle is asynchronous, so its local half
    # returns OK and only its sync() reports the failure
    out = _run(fail_rank=1, exchange=exchange, deferred=deferred, root=str(tmp_path))
    w0 = synth.weights0(SHAPES, 5)
    for r in range(2):
        assert out[r]["raised"] == "SignMuonError"
        assert out[r]["seen"] is None           # nobody voted
        assert np.array_equal(out[r]["W"], w0)  # nobody updated
        assert out[r]["agree"] is True
        assert out[r]["clocks"] == {}          # a failed step records no times


def test_alpha_beta_fit_recovers_the_model():
    from sign_muon_optimizer_b200.dist import allreduce_time_model, fit_alpha_beta
    alpha, beta = 7.5e-6, 1.0 / 150e9
    sizes = [1 << k for k in range(10, 31, 4)]
    a, b = fit_alpha_beta(sizes, [alpha + beta * n for n in sizes])
    assert abs(a - alpha) <= 1e-12 and abs(b - beta) <= 1e-9 * beta
    # one rank moves nothing; the transfer term tends to 2 s beta for many ranks
    assert allreduce_time_model(alpha, beta, 1, 1 << 20, 0) == 0.0
    assert allreduce_time_model(alpha, beta, 1, 1 << 20, 3) == 3 * alpha
    big = allreduce_time_model(alpha, beta, 10 ** 9, 1 << 20, 1)
    assert abs(big - (alpha + 2 * (1 << 20) * beta)) <= 1e-9 * big


def _time_rank(rank, world, port, q):
    import torch.distributed as dist

    from sign_muon_optimizer_b200.dist import time_collective
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sizes = [1 << 10, 1 << 16, 1 << 20]
        q.put((rank, time_collective("allgather", sizes, reps=2), time_collective("allreduce", sizes, reps=2)))
    finally:
        dist.destroy_process_group()


def test_collective_timings_are_the_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_time_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict((r, (ag, ar)) for r, ag, ar in (q.get(timeout=120) for _ in range(2)))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1]                    # both ranks report the max
    for ts in res[0]:
        assert len(ts) == 3 and all(t > 0.0 for t in ts)


def test_too_many_workers_is_rejected():
    # 2 ranks x 200 workers exceed the vote's 256: checked before any collective
    import torch.distributed as dist

    from sign_muon_optimizer_b200.dist import DistSignMuon
    port = _free_port()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("gloo", store=store, rank=0, world_size=1)
    try:
        with pytest.raises(ValueError):
            DistSignMuon(SHAPES, M_local=257, opt=_StandIn(), device="cpu")
    finally:
        dist.destroy_process_group()
