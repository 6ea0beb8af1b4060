"""Host-side logic of bench.py: the multi-process timing reduction (world size
2 over gloo on the CPU), the reference arm's rank handling and the
algorithmic flop and byte counts the roofline divides by."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        my_ms = [12.5, 30.25][rank]
        ms = bench.max_over_ranks(my_ms, "cpu")
        q.put((rank, ms, bench.job_throughput(world, 10, ms)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms, value in got:
        assert ms == 30.25                      # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * 10 / 0.03025)   # both ranks' steps over that time


def test_max_over_ranks_single_process():
    assert bench.max_over_ranks(7.0) == 7.0
    assert bench.job_throughput(1, 50, 1000.0) == pytest.approx(50.0)


def test_reference_arm_nonzero_rank_does_nothing(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")

    class A:
        steps, warmup, gpus = 2, 3, 2

    def boom(*a, **k):
        raise AssertionError("rank 1 must not run the oracle")
    monkeypatch.setattr(bench, "cpu_oracle_sample", boom)
    assert bench.run_reference(A()) == 0
    assert capsys.readouterr().out == ""


def test_nanogpt_flop_count():
    # 12 layers x (768^2 x (2304 + 768 + 3072 + 3072)) x 4 flops per cubic
    # iteration x 5 iterations x (8 workers + the post-vote problem)
    assert bench.ns_flops_per_step(synth.NANOGPT_SHAPES, 8, 5, True) == 11_741_366_845_440
    assert bench.ns_flops_per_step(synth.NANOGPT_SHAPES, 8, 5, False) == 8 * 1_304_596_316_160


def test_ns_kind_flops_x_and_gram_space():
    # one 768 x 3072 matrix, K = 5, one problem set: on X five Grams and five
    # applies of 2 m^2 n; in Gram space one of each plus 12 m x m products
    m, n = 768, 3072
    x = bench.ns_kind_flops([(m, n)], 1, 5, False)
    g = bench.ns_kind_flops([(n, m)], 1, 5, True)
    assert x == {"gram": 5 * 2 * m * m * n, "square": 0, "apply": 5 * 2 * m * m * n}
    assert g == {"gram": 2 * m * m * n, "square": 12 * 2 * m ** 3, "apply": 2 * m * m * n}
    assert sum(g.values()) <= 0.5 * sum(x.values())     # 40 m^3 against 80 m^3 at n = 4 m
    assert bench.ns_kind_flops([(m, n)], 8, 5, True)["square"] == 8 * g["square"]


def test_hbm_bytes_counts():
    d = synth.numel(synth.NANOGPT_SHAPES)
    b = bench.hbm_bytes_per_step(synth.NANOGPT_SHAPES, 8, 2, True)
    assert d == 84_934_656
    assert b["momentum"] == d * 116          # W once + 8 x (G + Mom r/w + bf16 X)
    assert b["pack"] == d * 8 * 4.125        # fp32 U read + one bit written per worker
    assert b["vote"] == d + 2 * d            # 8 bits per entry read, bf16 X written
    # 3 passes (P = 2), 8 workers + the post-vote set, 48 Grams of side 768:
    # the bf16 entries on and above the diagonal of the symmetric Gram
    assert b["power_iter"] == 3 * 9 * 48 * (768 * 769 // 2) * 2


def test_cpu_sample_is_one_144th():
    assert bench.CPU_SCALE == 144.0


def _collectives_rank(rank, world, port, q):
    import contextlib
    import io
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.run_collectives(None)
    q.put((rank, rc, buf.getvalue()))


def test_collectives_workload_over_gloo_world2():
    """bench.py --workload collectives on two host ranks (gloo): one JSON line
    from rank 0 with an alpha-beta fit per exchange."""
    import json
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_collectives_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict((r, (rc, out)) for r, rc, out in (q.get(timeout=300) for _ in range(2)))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][0] == 0 and res[1][0] == 0 and res[1][1] == ""
    line = json.loads(res[0][1].strip().splitlines()[-1])
    assert line["n_gpus"] == 2 and line["device"] == "cpu"
    for kind in ("allgather", "allreduce"):
        assert len(line[kind]["seconds"]) == len(line["sizes_bytes"])
        assert line[kind]["measured_s"] > 0 and line[kind]["nanogpt_payload_bytes"] > 0
