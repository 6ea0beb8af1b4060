"""GPU checks of the step in two halves (signmuon_local_signs, signmuon_vote_step).

[paper] "SignMuon: 通信高效的分布式Muon优化" Algorithm 2 runs the polar step and the
sign on each worker, exchanges the signs once, and lets every worker vote and
update its own copy of W.  The halves must reproduce signmuon_step bit for bit,
and workers split over several handles (ranks), whose signs are put side by
side as an all-gather would, must give every rank the W of one handle that
holds all the workers.  The ranks run one after the other on one GPU (no
kernel waits on another).  The file name sorts it after the other GPU suites.
"""
import numpy as np
import pytest

import synth

from gpu_helpers import dev, host

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import sign_muon_optimizer_b200 as smo  # noqa: E402

HP = dict(beta=0.9, lam=0.01, eta=0.02, eps=1e-7)
FUSED = [(64, 96), (96, 64), (128, 256)]          # every cols % 32 == 0: signs packed in the GEMM
RAGGED = [(3, 5), (130, 70), (64, 147)]

CASES = {
    "bf16_fused": (FUSED, 0),
    "fp32": (RAGGED, smo.SIGNMUON_NS_FP32),
    "post_polar": (RAGGED, smo.SIGNMUON_POST_POLAR),
    "normalized_sign": (FUSED, smo.SIGNMUON_NORMALIZED_SIGN),
    "ternary": (RAGGED, smo.SIGNMUON_TERNARY),
    "ternary_post_polar": (FUSED, smo.SIGNMUON_TERNARY | smo.SIGNMUON_POST_POLAR),
    "after_only": (RAGGED, smo.SIGNMUON_POST_POLAR | smo.SIGNMUON_POLAR_AFTER_ONLY | smo.SIGNMUON_TIE_PLUS),
}


def _opt(shapes, M, flags):
    return smo.SignMuon(shapes, M, beta=HP["beta"], lam=HP["lam"], K=5, eps=HP["eps"], scale="spectral", P=2,
                        flags=flags)


def _bits(W):
    return host(W).view(np.uint32)


@pytest.mark.parametrize("case", sorted(CASES))
def test_halves_equal_the_step(case):
    shapes, flags = CASES[case]
    M = 4
    w0 = synth.weights0(shapes, 91)
    whole, halves = _opt(shapes, M, flags), _opt(shapes, M, flags)
    Wa, Wb = dev(w0), dev(w0)
    buf = torch.zeros(M * halves.sign_stride(), dtype=torch.uint8, device="cuda")
    for step in (1, 2):
        G = [dev(g) for g in synth.gradients(shapes, M, 1.0, step=step, config_id=91)]
        whole.step(Wa, G, HP["eta"])
        halves.local_signs(Wb, G, buf)
        halves.vote_step(Wb, buf, M, HP["eta"])
        assert np.array_equal(_bits(Wa), _bits(Wb)), f"step {step}"
        for m in range(M):
            a, b = torch.zeros(whole.d, device="cuda"), torch.zeros(whole.d, device="cuda")
            whole.get_momentum(m, a)
            halves.get_momentum(m, b)
            assert np.array_equal(_bits(a), _bits(b))
    if flags & (smo.SIGNMUON_POST_POLAR | smo.SIGNMUON_NORMALIZED_SIGN):
        a, b = torch.zeros(whole.d, device="cuda"), torch.zeros(whole.d, device="cuda")
        whole.get_direction(a)
        halves.get_direction(b)
        assert np.array_equal(_bits(a), _bits(b))
    else:
        with pytest.raises(smo.SignMuonError) as ei:
            halves.get_direction(torch.zeros(whole.d, device="cuda"))
        assert ei.value.status == smo.SIGNMUON_E_UNSUPPORTED


@pytest.mark.parametrize("case", ["bf16_fused", "post_polar", "ternary"])
def test_two_ranks_equal_one_handle(case):
    """Two ranks of two workers each write their signs into the halves of one
    buffer (the all-gather's result); both then vote over the four workers and
    must land on the W of one four-worker handle, for two steps."""
    shapes, flags = CASES[case]
    M, ranks = 4, 2
    w0 = synth.weights0(shapes, 93)
    single = _opt(shapes, M, flags)
    parts = [_opt(shapes, M // ranks, flags) for _ in range(ranks)]
    stride = single.sign_stride()
    assert all(p.sign_stride() == stride for p in parts)
    W = dev(w0)
    Wr = [dev(w0) for _ in range(ranks)]
    gathered = torch.zeros(M * stride, dtype=torch.uint8, device="cuda")
    per = M // ranks
    for step in (1, 2):
        G = [dev(g) for g in synth.gradients(shapes, M, 1.0, step=step, config_id=93)]
        single.step(W, G, HP["eta"])
        for r in range(ranks):
            parts[r].local_signs(Wr[r], G[r * per:(r + 1) * per], gathered[r * per * stride:])
        for r in range(ranks):
            parts[r].vote_step(Wr[r], gathered, M, HP["eta"])
        for r in range(ranks):
            assert np.array_equal(_bits(Wr[r]), _bits(W)), f"rank {r}, step {step}"


def test_vote_only_handle_votes_and_updates():
    shapes = FUSED
    M = 3
    w0 = synth.weights0(shapes, 95)
    full = _opt(shapes, M, 0)
    voter = smo.SignMuon(shapes, 1, flags=smo.SIGNMUON_VOTE_ONLY)
    W, Wv = dev(w0), dev(w0)
    G = [dev(g) for g in synth.gradients(shapes, M, 1.0, step=1, config_id=95)]
    buf = torch.zeros(M * full.sign_stride(), dtype=torch.uint8, device="cuda")
    full.local_signs(W, G, buf)
    full.vote_step(W, buf, M, HP["eta"])
    voter.vote_step(Wv, buf, M, HP["eta"])
    assert np.array_equal(_bits(W), _bits(Wv))


def test_split_argument_checks():
    shapes = FUSED
    opt = _opt(shapes, 2, 0)
    d = opt.d
    W = torch.zeros(d, device="cuda")
    G = [torch.zeros(d, device="cuda") for _ in range(2)]
    buf = torch.zeros(2 * opt.sign_stride() + 64, dtype=torch.uint8, device="cuda")
    for call in (lambda: opt.local_signs(W, G, buf, stride=opt.sign_stride() - 16),
                 lambda: opt.local_signs(W, G, buf, stride=opt.sign_stride() + 8),
                 lambda: opt.vote_step(W, buf, 0, 0.1),
                 lambda: opt.vote_step(W, buf, 257, 0.1)):
        with pytest.raises(smo.SignMuonError) as ei:
            call()
        assert ei.value.status == smo.SIGNMUON_E_INVALID
    opt.local_signs(W, G, buf)
    with pytest.raises(smo.SignMuonError) as ei:
        opt.get_signs(0, torch.zeros(d // 8 + 16, dtype=torch.uint8, device="cuda"))
    assert ei.value.status == smo.SIGNMUON_E_UNSUPPORTED
    muon = _opt(shapes, 2, smo.SIGNMUON_MUON_MEAN)
    for call in (lambda: muon.local_signs(W, G, buf), lambda: muon.vote_step(W, buf, 2, 0.1)):
        with pytest.raises(smo.SignMuonError) as ei:
            call()
        assert ei.value.status == smo.SIGNMUON_E_UNSUPPORTED


@pytest.mark.parametrize("case", ["bf16_fused", "post_polar", "ternary", "normalized_sign"])
def test_sums_step_equals_the_step(case):
    """[paper] Algorithm 2's form of the exchange: the workers' signs summed
    (here by the library's own vote on one handle's buffer), then the majority
    of the sums and the rest of the step; W and D bit for bit."""
    shapes, flags = CASES[case]
    M = 4
    w0 = synth.weights0(shapes, 97)
    whole, halves = _opt(shapes, M, flags), _opt(shapes, M, flags)
    Wa, Wb = dev(w0), dev(w0)
    stride = halves.sign_stride()
    buf = torch.zeros(M * stride, dtype=torch.uint8, device="cuda")
    sums = torch.zeros(halves.d, dtype=torch.int32, device="cuda")
    views = [buf[m * stride:] for m in range(M)]
    for step in (1, 2):
        G = [dev(g) for g in synth.gradients(shapes, M, 1.0, step=step, config_id=97)]
        whole.step(Wa, G, HP["eta"])
        halves.local_signs(Wb, G, buf)
        if flags & smo.SIGNMUON_TERNARY:
            halves.vote_ternary(views, halves.d, sums, None)
        else:
            halves.vote(views, halves.d, sums, None)
        halves.sums_step(Wb, sums, HP["eta"])
        assert np.array_equal(_bits(Wa), _bits(Wb)), f"step {step}"
    a, b = torch.zeros(whole.d, device="cuda"), torch.zeros(whole.d, device="cuda")
    whole.get_direction(a)
    halves.get_direction(b)
    assert np.array_equal(_bits(a), _bits(b))


@pytest.mark.parametrize("acc8", [False, True])
def test_two_ranks_adding_their_sums_equal_one_handle(acc8):
    """Two ranks each sum their own two workers' signs (int32, or int8 as
    Algorithm 2's d-byte payload); the sums are added as the SUM all-reduce
    would, and both ranks land on the W of one four-worker handle."""
    shapes, flags = CASES["bf16_fused"]
    flags |= smo.SIGNMUON_ACC_INT8 if acc8 else 0
    M, ranks, per = 4, 2, 2
    w0 = synth.weights0(shapes, 99)
    single = _opt(shapes, M, flags)
    parts = [_opt(shapes, per, flags) for _ in range(ranks)]
    stride = single.sign_stride()
    W, Wr = dev(w0), [dev(w0) for _ in range(ranks)]
    dt = torch.int8 if acc8 else torch.int32
    local = [torch.zeros(per * stride, dtype=torch.uint8, device="cuda") for _ in range(ranks)]
    part_sums = [torch.zeros(single.d, dtype=dt, device="cuda") for _ in range(ranks)]
    for step in (1, 2):
        G = [dev(g) for g in synth.gradients(shapes, M, 1.0, step=step, config_id=99)]
        single.step(W, G, HP["eta"])
        for r in range(ranks):
            parts[r].local_signs(Wr[r], G[r * per:(r + 1) * per], local[r])
            parts[r].vote([local[r][m * stride:] for m in range(per)], single.d, part_sums[r], None)
        total = part_sums[0] + part_sums[1]          # the all-reduce's sum
        for r in range(ranks):
            parts[r].sums_step(Wr[r], total, HP["eta"])
            assert np.array_equal(_bits(Wr[r]), _bits(W)), f"rank {r}, step {step}"


@pytest.mark.parametrize("case", sorted(CASES))
def test_vote_step_ptrs_equals_the_step(case):
    """signmuon_vote_step_ptrs: every worker's signs in a buffer of its own,
    reached through a list of pointers (as the peers' mapped buffers are on a
    node of GPUs), two ranks' handles emulated one after the other: W of both
    ranks equals one four-worker handle's, bit for bit, for two steps."""
    shapes, flags = CASES[case]
    M, ranks, per = 4, 2, 2
    w0 = synth.weights0(shapes, 101)
    single = _opt(shapes, M, flags)
    parts = [_opt(shapes, per, flags) for _ in range(ranks)]
    stride = single.sign_stride()
    W, Wr = dev(w0), [dev(w0) for _ in range(ranks)]
    # separate allocations, one per rank, with 16 bytes in front so that no
    # buffer starts where an allocation starts
    raw = [torch.zeros(per * stride + 16, dtype=torch.uint8, device="cuda") for _ in range(ranks)]
    local = [b[16:] for b in raw]
    ptrs = [local[r].data_ptr() + m * stride for r in range(ranks) for m in range(per)]
    for step in (1, 2):
        G = [dev(g) for g in synth.gradients(shapes, M, 1.0, step=step, config_id=101)]
        single.step(W, G, HP["eta"])
        for r in range(ranks):
            parts[r].local_signs(Wr[r], G[r * per:(r + 1) * per], local[r])
        for r in range(ranks):
            parts[r].vote_step_ptrs(Wr[r], ptrs, HP["eta"])
            assert np.array_equal(_bits(Wr[r]), _bits(W)), f"rank {r}, step {step}"
    if flags & (smo.SIGNMUON_POST_POLAR | smo.SIGNMUON_NORMALIZED_SIGN):
        a, b = torch.zeros(single.d, device="cuda"), torch.zeros(single.d, device="cuda")
        single.get_direction(a)
        parts[1].get_direction(b)
        assert np.array_equal(_bits(a), _bits(b))


def test_vote_step_ptrs_argument_checks():
    shapes = FUSED
    opt = _opt(shapes, 2, 0)
    W = torch.zeros(opt.d, device="cuda")
    buf = torch.zeros(2 * opt.sign_stride() + 64, dtype=torch.uint8, device="cuda")
    good = [buf.data_ptr(), buf.data_ptr() + opt.sign_stride()]
    for ptrs in ([], [buf.data_ptr(), buf.data_ptr() + 8], [buf.data_ptr(), 0], [buf.data_ptr()] * 257):
        with pytest.raises(smo.SignMuonError) as ei:
            opt.vote_step_ptrs(W, ptrs, 0.1)
        assert ei.value.status == smo.SIGNMUON_E_INVALID
    muon = _opt(shapes, 2, smo.SIGNMUON_MUON_MEAN)
    with pytest.raises(smo.SignMuonError) as ei:
        muon.vote_step_ptrs(W, good, 0.1)
    assert ei.value.status == smo.SIGNMUON_E_UNSUPPORTED


def _peer_rank(rank, world, port, shapes, flags, q):
    """One rank of the "peer" exchange on the one GPU of this run: its sign
    buffers are mapped into the other process by CUDA IPC and the vote kernel
    reads them there (on a node, over NVLink).  No kernel waits for another
    rank: the ranks meet only in the host-side status all-reduce."""
    import datetime
    import os

    import torch.distributed as dist

    import sign_muon_optimizer_b200 as smo_r
    from sign_muon_optimizer_b200.dist import DistSignMuon
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        per = 2
        opt = smo_r.SignMuon(shapes, per, beta=HP["beta"], lam=HP["lam"], K=5, eps=HP["eps"], scale="spectral", P=2,
                             flags=flags)
        drv = DistSignMuon(shapes, M_local=per, opt=opt, device="cuda", exchange="peer")
        W = torch.from_numpy(synth.weights0(shapes, 103)).cuda()
        for step in (1, 2, 3):
            G = synth.gradients(shapes, world * per, 1.0, step=step, config_id=103)
            drv.step(W, [torch.from_numpy(g).cuda() for g in G[rank * per:(rank + 1) * per]], HP["eta"])
        torch.cuda.synchronize()
        q.put((rank, W.cpu().numpy().copy(), drv.replicas_agree(W)))
        drv.close()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", ["bf16_fused", "post_polar"])
def test_peer_exchange_through_cuda_ipc_equals_one_handle(case):
    import socket

    import torch.multiprocessing as mp
    shapes, flags = CASES[case]
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_peer_rank, args=(r, 2, port, shapes, flags, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict((r, (w, agree)) for r, w, agree in (q.get(timeout=300) for _ in range(2)))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    single = _opt(shapes, 4, flags)
    W = dev(synth.weights0(shapes, 103))
    for step in (1, 2, 3):
        single.step(W, [dev(g) for g in synth.gradients(shapes, 4, 1.0, step=step, config_id=103)], HP["eta"])
    for r in range(2):
        assert got[r][1] is True
        assert np.array_equal(got[r][0].view(np.uint32), _bits(W)), f"rank {r}"
