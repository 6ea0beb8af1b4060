"""The planner's tables (signmuon_plan_tables, host only) against the layout
rules the kernels rely on, for random mixes of matrix shapes, worker counts
and precision flags (hypothesis, derandomized):

- every X / A region and power-iteration vector lies inside its buffer, and
  none overlaps another;
- every base and row stride keeps rows on 16-byte boundaries (the TMA rule);
- the 4096-entry chunks cover each matrix exactly once, in order;
- the GEMM tile lists have the tile counts their shapes need, for every
  operation, for M workers and for one.

A planner mistake here would be an out-of-range access on the GPU."""
import pytest

hyp = pytest.importorskip("hypothesis")
from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402

import sign_muon_optimizer_b200 as smo  # noqa: E402

GRAM, SQUARE, APPLY = 0, 1, 2


def _ceil(a, b):
    return -(-a // b)


def _disjoint_inside(regions, limit):
    regions = sorted((s, e) for s, e in regions if e > s)
    end = 0
    for s, e in regions:
        assert s >= end, f"overlap at {s}"
        end = e
    assert end <= limit


def _check(shapes, M, flags, spectral):
    t = smo.signmuon_plan_tables(shapes, M, 5, "spectral" if spectral else "fro", 2, flags)
    t["_K"], t["_gram"] = 5, bool(flags & smo.SIGNMUON_NS_GRAM)
    fp32 = bool(flags & smo.SIGNMUON_NS_FP32)
    d = sum(r * c for r, c in shapes)
    assert t["d"] == d and t["dpad"] >= d and t["dpad"] % 64 == 0
    assert t["nb"] == _ceil(d, 8) and t["nb_pad"] >= t["nb"] and t["nb_pad"] % 16 == 0
    assert t["device_bytes"] == smo.signmuon_plan(shapes, M, 5, "spectral" if spectral else "fro", 2,
                                                  flags)["device_bytes"]

    # shape groups, in order of first appearance
    distinct = list(dict.fromkeys(shapes))
    groups = t["groups"]
    assert [(g[0], g[1]) for g in groups] == distinct
    first = 0
    for (rows, cols, ld, g, gld, wide, count, gfirst, x_base, a_base) in groups:
        assert ld == _ceil(cols, 8) * 8 and g == min(rows, cols) and gld == _ceil(g, 8) * 8
        assert wide == (1 if rows <= cols else 0) and count == shapes.count((rows, cols))
        assert gfirst == first
        first += count
        assert x_base % 8 == 0 and a_base % 8 == 0      # 16-byte aligned bf16 bases
    _disjoint_inside([(g[8], g[8] + M * g[6] * g[0] * g[2]) for g in groups], t["x_elems"])
    _disjoint_inside([(g[9], g[9] + M * g[6] * g[3] * g[4]) for g in groups], t["a_elems"])

    # matrices and their place in the flat vector and in their group
    off, seen = 0, {}
    for i, (moff, rows, cols, gi, q) in enumerate(t["mats"]):
        assert (rows, cols) == shapes[i] and moff == off
        assert groups[gi][0:2] == [rows, cols] and q == seen.get(gi, 0)
        assert t["group_mats"][groups[gi][7] + q] == i
        seen[gi] = q + 1
        off += rows * cols

    # chunks of the elementwise kernels: each matrix exactly once, in order
    chunks = t["chunks"]
    for i, (r, c) in enumerate(shapes):
        c0, nc = t["mat_chunk0"][i], t["mat_nchunks"][i]
        assert nc == _ceil(r * c, 4096)
        pos = 0
        for mat, ln, start in chunks[c0:c0 + nc]:
            assert mat == i and start == pos and 0 < ln <= 4096
            pos += ln
        assert pos == r * c
    assert sum(t["mat_nchunks"]) == len(chunks)

    # GEMM tile lists
    for op in (GRAM, SQUARE, APPLY):
        for slot, nw in ((0, M), (1, 1)):
            table = t["tiles"][2 * op + slot]
            tg = table["groups"]
            assert sorted(x[0] for x in tg) == list(range(len(groups)))
            start = 0
            for (gi, Md, Nd, Kd, BM, BN, sym, tm, tn, batch, tstart) in tg:
                rows, cols, _, g = groups[gi][:4]
                if op == GRAM:
                    assert (Md, Nd, Kd) == (g, g, max(rows, cols))
                elif op == SQUARE:
                    assert (Md, Nd, Kd) == (g, g, g)
                else:
                    assert (Md, Nd, Kd) == (rows, cols, g)
                if fp32:
                    assert (BM, BN) == (128, 128) and sym == 0
                else:
                    assert BM == 256 and BN in (128, 256)
                    assert sym == (1 if (op in (GRAM, SQUARE) and BN == 256) else 0)
                assert tm == _ceil(Md, BM) and tn == _ceil(Nd, BN)
                assert batch == nw * groups[gi][6] and tstart == start
                per = tm * (tm + 1) // 2 if sym else tm * tn
                start += per * batch
            assert table["total"] == start

    # X space or Gram space (bf16 cubic, K >= 2): the form with fewer tile
    # flops, both counted with the Gram and the m x m products on square
    # 256 x 256 upper-triangle tiles (Gram space runs them so: its stored
    # iterates must be exactly symmetric)
    K = t.get("_K")
    if K is not None and not fp32:
        def sym_flops(kdim):
            return sum(2 * 256 * 256 * kdim(g) * (_ceil(g[3], 256) * (_ceil(g[3], 256) + 1) // 2) * M * g[6]
                       for g in groups)
        apply_f = 0
        for (gi, Md, Nd, Kd, BM, BN, sym, tm, tn, batch, tstart) in t["tiles"][2 * APPLY]["groups"]:
            apply_f += 2 * BM * BN * Kd * tm * tn * batch
        gram_f = sym_flops(lambda g: max(g[0], g[1]))
        sq_f = sym_flops(lambda g: g[3])
        xs = K * (gram_f + apply_f)
        gs = gram_f + (3 * K - 3) * sq_f + apply_f
        big = all(g[3] >= 256 for g in groups)
        want = (not t["quintic"]) and K >= 2 and big and t.get("_gram") and gs < 0.85 * xs
        assert t["gram_ns"] == (1 if want else 0)
        if want:
            for op in (GRAM, SQUARE):
                for slot in (0, 1):
                    assert all(x[4] == 256 and x[5] == 256 and x[6] == 1 for x in t["tiles"][2 * op + slot]["groups"])
    elif K is not None:
        assert t["gram_ns"] == 0

    # power iteration: problem p = worker * n_mats + matrix
    n = len(shapes)
    gs = [min(r, c) for r, c in shapes]
    assert t["prob_g"] == gs * M
    assert t["u_elems_one"] == sum(gs) and t["u_elems"] == M * sum(gs)
    _disjoint_inside([(u, u + g) for u, g in zip(t["uoff"], t["prob_g"])], t["u_elems"])
    # the one-problem-set power iteration (worker 0's offsets) also runs on the
    # warm-start buffer of u_elems_one floats
    _disjoint_inside([(u, u + g) for u, g in zip(t["uoff"][:n], t["prob_g"][:n])], t["u_elems_one"])
    for p, aoff in enumerate(t["prob_aoff"]):
        w, i = divmod(p, n)
        mat = t["mats"][i]
        grp = groups[mat[3]]
        assert aoff == grp[9] + (w * grp[6] + mat[4]) * grp[3] * grp[4]
        assert t["prob_gld"][p] == grp[4]
    # symmetric power iteration: the 128 x 128 tiles on and above each Gram's
    # diagonal, each once and carrying its problem's offsets (one table load
    # per block); 128-row slices numbered per problem from soff; partial-sum
    # slots (nt x nt x 128 per problem) disjoint
    tiles_of, slices_of = {}, {}
    for k, (p, bi, bj, aoff, uoff, poff, g, gld) in enumerate(t["pi_tiles"]):
        tiles_of.setdefault(p, []).append((bi, bj))
        assert (k < t["n_pi_tiles_one"]) == (p < n)        # worker 0's tiles come first
        assert (aoff, uoff, poff, g, gld) == (t["prob_aoff"][p], t["uoff"][p], t["poff"][p],
                                              t["prob_g"][p], t["prob_gld"][p])
    for k, (p, bi, uoff, poff, g, soff) in enumerate(t["pi_slices"]):
        slices_of.setdefault(p, []).append(bi)
        assert (k < t["n_pi_slices_one"]) == (p < n)       # and its slices
        assert (uoff, poff, g, soff) == (t["uoff"][p], t["poff"][p], t["prob_g"][p], t["soff"][p])
        assert k == soff + bi                              # a problem's slices are contiguous
    spans = []
    for p in range(M * n):
        nt = _ceil(t["prob_g"][p], 128)
        assert sorted(tiles_of[p]) == [(i, j) for i in range(nt) for j in range(i, nt)]
        assert slices_of[p] == list(range(nt))
        spans.append((t["poff"][p], t["poff"][p] + nt * nt * 128))
    assert t["n_pi_slices"] == len(t["pi_slices"])
    _disjoint_inside(spans, t["part_elems"])
    assert t["part_elems"] == sum(_ceil(g, 128) ** 2 * 128 for g in t["prob_g"])
    # tensor-core tile schedules
    for table in t["tiles"]:
        _schedule_ok(table)


shape = st.tuples(st.integers(1, 300), st.integers(1, 300))


@settings(max_examples=120, deadline=None, derandomize=True)
@given(st.lists(shape, min_size=1, max_size=5), st.integers(0, 3), st.integers(1, 9), st.integers(0, 7),
       st.booleans())
def test_plan_tables_follow_the_layout_rules(base, repeat, M, fl, spectral):
    shapes = base + base[:repeat]                  # repeated shapes share a group
    flags = ((smo.SIGNMUON_NS_FP32 if fl & 1 else 0) | (smo.SIGNMUON_NS_QUINTIC if fl & 2 else 0)
             | (smo.SIGNMUON_POST_POLAR if fl & 4 else 0))
    _check(shapes, M, flags, spectral)


@pytest.mark.parametrize("name", ["nanogpt", "resnet50"])
def test_plan_tables_of_the_bench_workloads(name):
    import synth
    wl = synth.WORKLOADS[name]
    _check([tuple(s) for s in wl["shapes"]], wl["M"], smo.SIGNMUON_POST_POLAR, True)


def _schedule_ok(table):
    """A tensor-core launch's tile schedule against a plain restatement: each
    tile, in list order, to the least-loaded of the clusters (ties to the
    lower index), a tile costing ceil(K / 64) + 3; kept only when its
    makespan is under 0.97 of round robin's."""
    import heapq
    total, ncl = table["total"], table["clusters"]
    cost = []
    for (gi, Md, Nd, Kd, BM, BN, sym, tm, tn, batch, tstart) in table["groups"]:
        per = tm * (tm + 1) // 2 if sym else tm * tn
        assert tstart == len(cost)
        cost += [(Kd + 63) // 64 + 3] * (per * batch)
    assert len(cost) == total
    if total == 0:
        assert table["sched"] == []
        return
    rr = [0] * ncl
    for t, c in enumerate(cost):
        rr[t % ncl] += c
    heap = [(0, c) for c in range(ncl)]
    lists = [[] for _ in range(ncl)]
    for t, c in enumerate(cost):
        load, cl = heapq.heappop(heap)
        lists[cl].append(t)
        heapq.heappush(heap, (load + c, cl))
    greedy = max(load for load, _ in heap)
    assert table["makespan_rr"] == max(rr) and table["makespan_greedy"] == greedy
    if greedy < 0.97 * max(rr):
        starts = [0]
        for l in lists:
            starts.append(starts[-1] + len(l))
        assert table["sched"] == starts + [t for l in lists for t in l]
        assert sorted(table["sched"][ncl + 1:]) == list(range(total))   # every tile once
    else:
        assert table["sched"] == []


@pytest.mark.parametrize("name", ["resnet50", "nanogpt"])
def test_tile_schedules(name):
    """The ResNet-50 set (tiles of K = 64 .. 4608 in one launch) gets a
    greedy schedule for its M-worker Gram launch, about 14 % shorter than
    round robin; the nanoGPT launches, whose tiles are alike, keep round
    robin."""
    import synth
    wl = synth.WORKLOADS[name]
    t = smo.signmuon_plan_tables([tuple(s) for s in wl["shapes"]], wl["M"], wl["K"], wl["scale"], wl["P"],
                                 smo.SIGNMUON_POST_POLAR)
    for table in t["tiles"]:
        _schedule_ok(table)
    gram = t["tiles"][0]
    if name == "resnet50":
        assert gram["sched"] and gram["makespan_greedy"] < 0.9 * gram["makespan_rr"]
    else:
        assert all(table["sched"] == [] for table in t["tiles"])


def test_gram_space_choice():
    """With SIGNMUON_NS_GRAM the nanoGPT set (every matrix 768 x n, n = 768..3072)
    runs its bf16 cubic iteration in Gram space; without the flag, and for
    square matrices, Grams under 256, quintic, fp32 and K < 2, it stays on X."""
    import synth
    shp = [tuple(s) for s in synth.NANOGPT_SHAPES]
    G = smo.SIGNMUON_NS_GRAM
    plan = lambda shapes, K=5, flags=G: smo.signmuon_plan_tables(shapes, 8, K, "spectral", 2, flags)["gram_ns"]
    assert plan(shp) == 1
    assert plan(shp, flags=0) == 0                                    # the default iterates on X
    assert plan([(768, 3072)]) == 1 and plan([(3072, 768)]) == 1     # either orientation
    assert plan([(768, 768)]) == 0 and plan([(1024, 1024)]) == 0     # square: more flops in Gram space
    assert plan([(128, 256), (96, 300)]) == 0                         # small Grams stay on X
    assert plan([(768, 3072), (200, 3000)]) == 0                      # ... every one of them
    assert plan(shp, K=1) == 0
    assert plan(shp, flags=G | smo.SIGNMUON_NS_QUINTIC) == 0
    assert plan(shp, flags=G | smo.SIGNMUON_NS_FP32) == 0
    # the extra m x m buffers (B, A2, Q0, Q1) are part of the device bytes
    t1 = smo.signmuon_plan_tables(shp, 8, 5, "spectral", 2, G)
    t2 = smo.signmuon_plan_tables(shp, 8, 5, "spectral", 2, 0)
    assert t1["device_bytes"] - t2["device_bytes"] == 4 * t1["a_elems"] * 2


def test_plan_tables_size_query_and_errors():
    import ctypes
    arr = (ctypes.c_int64 * 2)(4, 6)
    need = ctypes.c_int64(0)
    assert smo._lib.signmuon_plan_tables(arr, 1, 2, 5, 0, 1, 0, None, 0, ctypes.byref(need)) == 0
    assert need.value > 2
    small = ctypes.create_string_buffer(8)
    assert smo._lib.signmuon_plan_tables(arr, 1, 2, 5, 0, 1, 0, small, 8, ctypes.byref(need)) == \
        smo.SIGNMUON_E_INVALID
    with pytest.raises(smo.SignMuonError):
        smo.signmuon_plan_tables([(0, 4)], 2)
