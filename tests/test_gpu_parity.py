"""GPU parity: every CUDA path, called through the C ABI, against the CPU
oracle on the same seeded inputs, element by element.

The bar is bit-exactness for every dtype: fp32 and int32 reduce in the ring
order on both sides; bf16 is folded in fp32 and rounded once by the one-shot
paths and rounded per hop by the ring and tree schedules, on both sides
alike.  bf16 results are also checked against an fp64 reduction within the
stated tolerance (abs 1e-2, rel 1e-2).
"""
import numpy as np
import pytest
import torch

import oracle
import ring_all_reduce_virtual_b200 as rrv
from conftest import golden_lines
from gpu_util import assert_bits_equal, empty_like_ranks, to_dev, to_host
from ring_all_reduce_virtual_b200 import synth

pytestmark = pytest.mark.gpu

ALGOS = ["ring", "oneshot", "tree", "tree_oneshot", "two_shot", "double_ring", "auto"]
ORACLE = {
    "double_ring": oracle.double_ring_allreduce,
    "two_shot": oracle.fold_ring_order,
    "ring": oracle.ring_allreduce,
    "oneshot": oracle.fold_ring_order,
    "auto": oracle.fold_ring_order,
    "tree": oracle.tree_schedule,
    "tree_oneshot": oracle.tree_fold,
}
PER_HOP = ("ring", "tree", "double_ring")  # bf16 schedules that round at every hop
TILE = {"f32": 2048, "bf16": 4096, "f16": 4096, "i32": 2048}  # elements per tile of the N-input fold kernels
TILE_MOVE = {"f32": 4096, "bf16": 8192, "f16": 8192, "i32": 4096}  # per tile of the 1- and 2-input kernels


def _dist(op, dtype):
    if dtype == "i32":
        return "int"
    if op in ("sum", "avg"):
        return "full"  # full mantissas: a fold in the wrong order gives other bits
    return "prod" if op == "prod" else "uniform"


def _run(n, count, dtype, op, algo, seed=0, offsets=None):
    x = synth.ranks(seed, n, count, _dist(op, dtype), dtype)
    want = [a.copy() for a in x]
    ORACLE[algo](want, op)
    d = to_dev(x, offsets)
    rrv.all_reduce(d, op, algo)
    got = to_host(d)
    assert_bits_equal(got, want, f"{algo} {dtype} {op} n={n} count={count}")
    return x, got


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from ring_all_reduce_virtual_b200.build import build

    build()


def test_library_runs_sm100a_code():
    """The runtime loads the library's kernels as code built for compute
    capability 10.0 (sm_100a)."""
    import ctypes

    from ring_all_reduce_virtual_b200 import _lib

    v = ctypes.c_int(0)
    _lib.check(_lib.lib().rr_binary_version(ctypes.byref(v)), "rr_binary_version")
    assert v.value == 100


# -------------------------------------------------------- worked example --

@pytest.mark.parametrize("algo", ALGOS)
def test_worked_example(algo):
    exp = {}
    for ln in golden_lines("five_primitives_4rank.txt"):
        head, rest = ln.split(":", 1)
        p = head.split()
        if len(p) == 2:
            exp.setdefault(p[0], {})[int(p[1])] = [float(v) for v in rest.split()]
    x = synth.ranks(0, 4, 4, "arange")
    d = to_dev(x)
    rrv.all_reduce(d, "sum", algo)
    for r, t in enumerate(to_host(d)):
        assert t.tolist() == exp["all_reduce"][r]
    d = to_dev(x)
    rs = empty_like_ranks(4, 1, "f32")
    rrv.reduce_scatter(d, rs)
    ag = empty_like_ranks(4, 4, "f32")
    rrv.all_gather(rs, ag)
    a2a = empty_like_ranks(4, 4, "f32")
    rrv.all_to_all(d, a2a)
    for r in range(4):
        assert to_host(rs)[r].tolist() == exp["reduce_scatter"][r]
        assert to_host(ag)[r].tolist() == exp["all_gather"][r]
        assert to_host(a2a)[r].tolist() == exp["all_to_all"][r]


# ------------------------------------------------------ all-reduce parity --

@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16", "i32"])
@pytest.mark.parametrize("op", ["sum", "avg", "max", "min", "prod"])
def test_allreduce_every_op_and_dtype(algo, dtype, op):
    if dtype == "i32" and op == "avg":
        pytest.skip("AVG is not defined for int32")
    n = 5
    count = 3 * TILE[dtype] * n + 37  # several tiles per chunk and a ragged tail
    x, got = _run(n, count, dtype, op, algo, seed=1)
    if dtype in ("bf16", "f16") and op in ("sum", "avg"):
        widen = oracle.bf16_to_f32 if dtype == "bf16" else oracle.f16_to_f32
        wide = np.stack([widen(v) for v in x]).astype(np.float64)
        ref, mag = wide.sum(0), np.abs(wide).sum(0)
        if op == "avg":
            ref, mag = ref / n, mag / n
        g = widen(got[0]).astype(np.float64)
        if algo in PER_HOP:
            # partials rounded to 16 bits after every hop: recursive summation
            # in bf16 (u = 2^-8) or fp16 (u = 2^-11), |error| <= gamma_{N-1} *
            # sum |x| (Higham 4.2)
            u = 2.0 ** -8 if dtype == "bf16" else 2.0 ** -11
            gamma = (n - 1) * u / (1 - (n - 1) * u)
            assert np.all(np.abs(g - ref) <= gamma * mag + 1e-30)
        else:  # fp32 accumulation, one rounding: the stated abs/rel 1e-2
            assert np.allclose(g, ref, atol=1e-2, rtol=1e-2)


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("n", [1, 2, 3, 4, 7, 8, 16])
@pytest.mark.parametrize("count", [0, 1, 3, 4, 5, 17, 1000, 4096, 70001])
def test_allreduce_sizes(algo, n, count):
    _run(n, count, "f32", "sum", algo, seed=2)


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
def test_allreduce_64_ranks(algo, dtype):
    _run(64, 64 * 700 + 3, dtype, "sum", algo, seed=3)


@pytest.mark.parametrize("algo", ["ring", "oneshot", "tree_oneshot"])
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
def test_allreduce_shared_misalignment(algo, dtype):
    # every base 1 element past a 16-byte boundary: vector path after a head
    n = 4
    _run(n, 5 * TILE[dtype] + 11, dtype, "sum", algo, seed=4, offsets=[1] * n)


@pytest.mark.parametrize("algo", ["ring", "oneshot", "tree", "tree_oneshot"])
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
def test_allreduce_mixed_misalignment(algo, dtype):
    # bases disagree modulo 16 bytes: the scalar path
    n = 4
    _run(n, 3 * TILE[dtype] + 5, dtype, "avg", algo, seed=5, offsets=[0, 1, 2, 3])


def test_fold_order_fixture():
    # the hand-derived rounding fixture: ring order gives 0 everywhere,
    # a pairwise tree gives 1 for element 0
    g = {ln.split(":")[0]: [float(v) for v in ln.split(":")[1].split()] for ln in golden_lines("fold_order.txt")}
    big = np.float32(2.0 ** 24)
    x = [np.zeros(4, dtype=np.float32) for _ in range(4)]
    for i in range(4):
        for k, v in enumerate([np.float32(1), big, np.float32(1), -big]):
            x[(i + k) % 4][i] = v
    for algo in ("ring", "oneshot", "auto"):
        d = to_dev(x)
        rrv.all_reduce(d, "sum", algo)
        for t in to_host(d):
            assert t.tolist() == g["ring_order"]
    d = to_dev(x)
    rrv.all_reduce(d, "sum", "tree_oneshot")
    assert to_host(d)[0][0] == 1.0


@pytest.mark.parametrize("algo", ["tree", "tree_oneshot"])
@pytest.mark.parametrize("count", [4, 4096, 5])
def test_tree_order_with_unpaired_ranks_golden(algo, count):
    """The hand-derived fixture of the tree's order for N = 3, 5, 6, 7 (an
    unpaired rank carried up to the next level), on every element of buffers
    of one vector, of many tiles (bulk-copy tree fold and the single-launch
    tree schedule) and of a ragged size."""
    from conftest import golden_lines

    for ln in golden_lines("tree_order_unpaired.txt"):
        n_s, xs, want = ln.split(":")
        vals = [np.float32(float(v)) for v in xs.split()]
        x = [np.full(count, v, dtype=np.float32) for v in vals]
        d = to_dev(x)
        rrv.all_reduce(d, "sum", algo)
        for r, g in enumerate(to_host(d)):
            assert np.all(g == np.float32(float(want))), (algo, n_s, r, g[:4])
    rrv.check_timeouts()


def test_max_signed_zero_ties_follow_the_fold():
    n = 4
    x = [np.full(n, -1.0, dtype=np.float32) for _ in range(n)]
    for i in range(n):
        x[i][i] = 0.0
        x[(i + 1) % n][i] = -0.0
    for algo in ("ring", "oneshot"):
        want = [a.copy() for a in x]
        ORACLE[algo](want, "max")
        d = to_dev(x)
        rrv.all_reduce(d, "max", algo)
        assert_bits_equal(to_host(d), want, algo)


# ----------------------------------------------------------- ring steps --

@pytest.mark.parametrize("n", [2, 3, 4, 8])
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("op", ["sum", "avg"])
def test_ring_steps_track_the_oracle_state(n, dtype, op):
    # after every one of the 2(N-1) steps the device buffers equal the
    # oracle's per-rank chunk arrays bit for bit
    count = 3 * TILE_MOVE[dtype] * n + 13
    x = synth.ranks(6, n, count, "uniform", dtype)
    d = to_dev(x)
    host = [a.copy() for a in x]
    for phase in ("reduce_scatter", "all_gather"):
        for s in range(n - 1):
            oracle.ring_step(host, op, oracle.PHASE_RS if phase == "reduce_scatter" else oracle.PHASE_AG, s)
            rrv.ring_step(d, op, phase, s)
            assert_bits_equal(to_host(d), host, f"{phase} step {s}")
            st = rrv.last_stats()
            assert st["launches"] == 1


def test_ring_stats_match_the_schedule():
    n, count = 4, 1024
    d = to_dev(synth.ranks(7, n, count, "uniform"))
    rrv.all_reduce(d, "sum", "ring")  # buffers at one 16-byte phase: the whole schedule in one launch
    st = rrv.last_stats()
    assert st["algo"] == "ring" and st["steps"] == 6 and st["launches"] == 1
    assert 0 < st["launch_ns"] <= st["host_ns"]
    assert st["bytes_sent_max"] == 6144  # [P4]: 2(n-1)/n x 4096 bytes
    assert st["hbm_bytes"] == 5 * 3 * 4096
    rrv.all_reduce(d, "sum", "oneshot")
    st = rrv.last_stats()
    assert st["launches"] == 1 and st["hbm_bytes"] == 2 * 4 * 4096
    rrv.all_reduce(d, "sum", "two_shot")  # the ring's per-rank volume in 2 steps
    st = rrv.last_stats()
    assert st["launches"] == 2 and st["steps"] == 2 and st["bytes_sent_max"] == 6144
    rrv.all_reduce(d, "sum", "double_ring")  # the same volume, half to each neighbour
    st = rrv.last_stats()
    want = oracle.double_ring_allreduce(synth.ranks(7, n, count, "uniform"))
    assert st["launches"] == 1 and st["bytes_sent_max"] == int(want.max()) == 6144
    rrv.all_reduce(d, "sum", "tree")
    st = rrv.last_stats()
    assert st["launches"] == 1 and st["steps"] == 4
    # buffers at different 16-byte phases: one launch per step, the same counts
    m = to_dev(synth.ranks(7, n, count, "uniform"), offsets=[0, 1, 2, 3])
    rrv.all_reduce(m, "sum", "ring")
    st = rrv.last_stats()
    assert st["launches"] == 6 and st["steps"] == 6 and st["bytes_sent_max"] == 6144
    rrv.all_reduce(m, "sum", "tree")
    assert rrv.last_stats()["launches"] == 4


# --------------------------------------------- reduce-scatter, all-gather --

@pytest.mark.parametrize("n", [1, 2, 3, 4, 8, 64])
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16", "i32"])
def test_reduce_scatter_all_gather_all_to_all(n, dtype):
    per = 2 * TILE_MOVE[dtype] + 9
    x = synth.ranks(8, n, n * per, "int" if dtype == "i32" else "uniform", dtype)
    d = to_dev(x)
    for op in ("sum", "max") if dtype not in ("bf16", "f16") else ("sum", "avg"):
        rs = empty_like_ranks(n, per, dtype)
        rrv.reduce_scatter(d, rs, op)
        assert_bits_equal(to_host(rs), oracle.reduce_scatter([a.copy() for a in x], op), f"rs {op}")
    ag = empty_like_ranks(n, n * per, dtype)
    rrv.all_gather(rs, ag)
    assert_bits_equal(to_host(ag), oracle.all_gather(to_host(rs)), "ag")
    a2a = empty_like_ranks(n, n * per, dtype)
    rrv.all_to_all(d, a2a)
    assert_bits_equal(to_host(a2a), oracle.all_to_all(x), "a2a")


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16", "i32"])
@pytest.mark.parametrize("shift", [1, 2, 3, 5, 7])
def test_copies_to_another_phase(dtype, shift):
    """All-gather and all-to-all blocks of a length that is `shift` elements
    past a whole number of 16-byte vectors, over several tiles: block q lands
    q * shift elements out of phase with its source, so the copies take the
    shift through shared memory; and the fused/staged bucket paths on tensors
    whose bucket offsets take every phase."""
    L = 4 if dtype in ("f32", "i32") else 8
    if shift >= L:
        pytest.skip("shift within one vector")
    n = 3
    per = 3 * TILE_MOVE[dtype] + shift
    x = synth.ranks(11 + shift, n, per, "int" if dtype == "i32" else "full", dtype)
    ag = empty_like_ranks(n, n * per, dtype)
    rrv.all_gather(to_dev(x), ag)
    assert_bits_equal(to_host(ag), oracle.all_gather(x), f"ag shift {shift}")
    y = synth.ranks(12 + shift, n, n * per, "int" if dtype == "i32" else "full", dtype)
    a2a = empty_like_ranks(n, n * per, dtype)
    rrv.all_to_all(to_dev(y), a2a)
    assert_bits_equal(to_host(a2a), oracle.all_to_all(y), f"a2a shift {shift}")
    if dtype == "i32":
        return
    numels = [shift, 20000 + shift, 3, 30001, 17]  # later tensors start at every phase, over several tiles
    host = _grad_set(13 + shift, n, numels, dtype)
    want = [[g.copy() for g in rank] for rank in host]
    cap = 1 << 30
    oracle.bucket_sync(want, cap, "avg")
    plan = rrv.BucketPlan(numels, dtype, cap)
    grads = [to_dev(rank) for rank in host]
    numel = plan.info(0)[2]
    buckets = [torch.empty(numel, dtype=torch.float32, device="cuda") for _ in range(n)]
    plan.pack(0, grads, buckets)
    rrv.all_reduce(buckets, "sum", "oneshot")
    plan.unpack(0, buckets, grads, "avg")
    for r in range(n):
        assert_bits_equal(to_host(grads[r]), want[r], f"staged bucket rank {r}")


@pytest.mark.parametrize("op", ["sum", "avg", "min", "prod"])
def test_rs_then_ag_equals_allreduce(op):
    n, per = 8, 3000
    x = synth.ranks(9, n, n * per, "prod" if op == "prod" else "uniform")
    d = to_dev(x)
    rs = empty_like_ranks(n, per, "f32")
    ag = empty_like_ranks(n, n * per, "f32")
    rrv.reduce_scatter(d, rs, op)
    rrv.all_gather(rs, ag)
    rrv.all_reduce(d, op, "ring")
    assert_bits_equal(to_host(ag), to_host(d), op)


# --------------------------------------------------------------- buckets --

def _grad_set(seed, n, numels, dtype="bf16"):
    return [synth.rank_grads(seed, r, numels, "normal", dtype) for r in range(n)]


def test_direct_bucket_syncs_in_a_cuda_graph():
    """Direct bucket syncs are launched as programmatic dependents of the
    stream's previous kernel: back-to-back syncs of every bucket, captured
    into one CUDA graph and replayed twice on fresh gradients, give the
    oracle's bits (and the eager calls the same)."""
    n = 8
    numels = [5, 3000, 64, 1, 9000, 77, 20000, 333, 4096, 12345]
    cap = 4096 * 2  # four buckets
    host = _grad_set(21, n, numels)
    want = [[g.copy() for g in rank] for rank in host]
    oracle.bucket_sync(want, cap, "avg")
    plan = rrv.BucketPlan(numels, "bf16", cap)
    assert plan.num_buckets > 3
    grads = [to_dev(rank) for rank in host]
    gs = rrv.GradSet(grads)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm the library's per-device state outside the capture
        for b in range(plan.num_buckets):
            plan.all_reduce(b, gs, "avg", s)
    s.synchronize()
    for r in range(n):
        assert_bits_equal(to_host(grads[r]), want[r], f"eager rank {r}")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for b in range(plan.num_buckets):
            plan.all_reduce(b, gs, "avg", s)
    for _ in range(2):
        for r in range(n):  # fresh gradients in the captured buffers
            for t, h in enumerate(host[r]):
                grads[r][t].copy_(to_dev([h])[0])
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        for r in range(n):
            assert_bits_equal(to_host(grads[r]), want[r], f"graph rank {r}")
    del g


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("op", ["avg", "sum"])
def test_bucket_staged_and_fused_match_the_oracle(dtype, op):
    n = 8
    numels = [5, 3000, 64, 1, 9000, 77, 0, 20000, 333, 4096]
    cap = 4 * 4096 * (4 if dtype == "f32" else 2)
    host = _grad_set(10, n, numels, dtype)
    want = [[g.copy() for g in rank] for rank in host]
    oracle.bucket_sync(want, cap, op)
    plan = rrv.BucketPlan(numels, dtype, cap)
    # staged: pack -> one-shot SUM on the fp32 buckets -> unpack
    grads = [to_dev(rank) for rank in host]
    for b in range(plan.num_buckets):
        numel = plan.info(b)[2]
        buckets = [torch.empty(max(numel, 1), dtype=torch.float32, device="cuda") for _ in range(n)]
        plan.pack(b, grads, buckets)
        packed = to_host(buckets)
        rrv.all_reduce([t[:numel] for t in buckets], "sum", "oneshot")
        plan.unpack(b, buckets, grads, op)
        # the packed bucket is the exact widening of the gradients
        bo, off = [], []
        first, cnt, _ = plan.info(b)
        for t in range(first, first + cnt):
            w = {"bf16": oracle.bf16_to_f32, "f16": oracle.f16_to_f32}.get(dtype, np.asarray)(host[0][t])
            assert np.array_equal(packed[0][plan.tensor(t)[1]:plan.tensor(t)[1] + numels[t]], w)
    for r in range(n):
        assert_bits_equal(to_host(grads[r]), want[r], f"staged rank {r}")
    # fused: one pass over the gradients
    grads = [to_dev(rank) for rank in host]
    for b in range(plan.num_buckets):
        plan.all_reduce(b, grads, op)
    for r in range(n):
        assert_bits_equal(to_host(grads[r]), want[r], f"fused rank {r}")


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("op", ["avg", "sum"])
def test_bucket_range_matches_per_bucket_syncs(dtype, op):
    """A bucket range shares launches but keeps every bucket's own chunking:
    the whole plan at once, and a sub-range that leaves the other buckets
    alone.  300 tensors x 8 ranks (2400 gradient pointers) need more than one
    launch."""
    n = 8
    rng = np.random.default_rng(31)
    numels = [int(v) for v in rng.integers(0, 3000, size=300)]
    numels[7] = 70001  # one tensor larger than the cap: a bucket of its own
    cap = 3000 * (4 if dtype == "f32" else 2)
    host = _grad_set(12, n, numels, dtype)
    want = [[g.copy() for g in rank] for rank in host]
    oracle.bucket_sync(want, cap, op)
    plan = rrv.BucketPlan(numels, dtype, cap)
    nb = plan.num_buckets
    assert nb > 50
    grads = [to_dev(rank) for rank in host]
    plan.all_reduce_range(0, nb, grads, op)
    st = rrv.last_stats()
    assert 1 < st["launches"] < nb
    for r in range(n):
        assert_bits_equal(to_host(grads[r]), want[r], f"range rank {r}")
    # buckets 3 .. nb-4 only: their tensors reduced, the rest untouched
    first, last = 3, nb - 4
    t_lo = plan.info(first)[0]
    t_hi = plan.info(last)[0] + plan.info(last)[1]
    grads = [to_dev(rank) for rank in host]
    plan.all_reduce_range(first, last - first + 1, grads, op)
    for r in range(n):
        got = to_host(grads[r])
        exp = [want[r][t] if t_lo <= t < t_hi else host[r][t] for t in range(len(numels))]
        assert_bits_equal(got, exp, f"sub-range rank {r}")


def test_bucket_fused_misaligned_tensors():
    # tensors carved out of one flat allocation at odd element offsets
    n = 4
    numels = [7, 1001, 3, 2500, 64]
    host = _grad_set(11, n, numels)
    want = [[g.copy() for g in rank] for rank in host]
    oracle.bucket_sync(want, 1000, "avg")
    plan = rrv.BucketPlan(numels, "bf16", 1000)
    grads = []
    for r in range(n):
        flat = torch.zeros(sum(numels) + 8 * len(numels), dtype=torch.bfloat16, device="cuda")
        ts, o = [], 1 + r
        for g in host[r]:
            t = flat[o:o + g.size]
            t.copy_(torch.from_numpy(g.view(np.int16)).cuda().view(torch.bfloat16))
            ts.append(t)
            o += g.size + 3
        grads.append(ts)
    for b in range(plan.num_buckets):
        plan.all_reduce(b, grads, "avg")
    for r in range(n):
        assert_bits_equal(to_host(grads[r]), want[r], f"rank {r}")


# ------------------------------------------------------ host buffers --

@pytest.mark.parametrize("algo", ["auto", "oneshot", "tree_oneshot", "ring"])
@pytest.mark.parametrize("count", [1000, (8 << 20) // 4 * 3 + 17])  # below and above one 8 MiB slice
def test_allreduce_host_buffers(algo, count):
    # host -> device -> reduce -> host, pipelined in slices for the one-shot
    # algorithms; ordered on a side stream; host and device both hold the result
    n = 4
    x = synth.ranks(12, n, count, "uniform")
    want = [a.copy() for a in x]
    ORACLE[algo](want, "avg")
    host = [torch.from_numpy(a.copy()).pin_memory() for a in x]
    dev = [torch.full((count,), float("nan"), device="cuda") for _ in range(n)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        rrv.all_reduce_host(host, dev, "avg", algo, side)
    side.synchronize()
    assert_bits_equal([h.numpy() for h in host], want, "host")
    assert_bits_equal(to_host(dev), want, "device")


def test_bucket_views_layout_equals_fused_bucket_sync():
    # gradients as views into one flat bf16 buffer per bucket and rank: a
    # plain one-shot all-reduce of the flat buffer gives the fused bucket
    # sync's bits (same chunking over the bucket's flat index, same fold)
    n = 8
    numels = [5, 3000, 64, 1, 9000, 77, 20000, 333, 4096]
    host = _grad_set(13, n, numels)
    want = [[g.copy() for g in rank] for rank in host]
    oracle.bucket_sync(want, 4 * 4096 * 2, "avg")
    plan = rrv.BucketPlan(numels, "bf16", 4 * 4096 * 2)
    flats, views = plan.flat_buffers(n, "cuda")
    for r in range(n):
        for t, g in enumerate(host[r]):
            views[r][t].copy_(torch.from_numpy(g.view(np.int16)).cuda().view(torch.bfloat16))
    for b in range(plan.num_buckets):
        rrv.all_reduce(flats[b], "avg", "oneshot")
    for r in range(n):
        assert_bits_equal(to_host(views[r]), want[r], f"rank {r}")


# ------------------------------------------------- overlapped bucket sync --

def _reducer_setup(n, numels, cap, seed):
    host = _grad_set(seed, n, numels)
    want = [[g.copy() for g in rank] for rank in host]
    oracle.bucket_sync(want, cap, "avg")
    src = [to_dev(rank) for rank in host]  # the "backward" copies these into the gradients
    grads = [[torch.zeros_like(t) for t in rank] for rank in src]
    plan = rrv.BucketPlan(numels, "bf16", cap)
    return host, want, src, grads, plan


def _backward_step(red, src, grads, stream):
    # a synthetic backward on `stream`: gradients become final one tensor at a
    # time, in the plan's order; each is marked ready right after
    for t in range(len(grads[0])):
        for r in range(len(grads)):
            grads[r][t].copy_(src[r][t])
        red.ready(t, stream)
    red.finish(stream)


def test_reducer_overlaps_bucket_syncs_with_backward():
    n = 8
    numels = [4096, 5, 30000, 64, 9000, 1, 12000, 333]
    host, want, src, grads, plan = _reducer_setup(n, numels, 8192, 20)
    assert plan.num_buckets > 2
    compute = torch.cuda.Stream()
    compute.wait_stream(torch.cuda.current_stream())
    red = rrv.Reducer(plan, grads, "avg")
    with torch.cuda.stream(compute):
        _backward_step(red, src, grads, compute)
        _backward_step(red, src, grads, compute)  # a second step reuses the reducer
    compute.synchronize()
    for r in range(n):
        assert_bits_equal(to_host(grads[r]), want[r], f"rank {r}")


def test_reducer_step_captured_in_a_cuda_graph():
    n = 4
    numels = [2048, 7, 20000, 100, 5000]
    host, want, src, grads, plan = _reducer_setup(n, numels, 4096, 21)
    red = rrv.Reducer(plan, grads, "avg")
    compute = torch.cuda.Stream()
    compute.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(compute):
        _backward_step(red, src, grads, compute)  # warm-up outside the graph
    compute.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=compute):
        _backward_step(red, src, grads, compute)
    for _ in range(2):
        for rank in grads:
            for t in rank:
                t.zero_()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        for r in range(n):
            assert_bits_equal(to_host(grads[r]), want[r], f"rank {r}")


def test_reducer_refuses_an_incomplete_step():
    n = 2
    numels = [100, 200, 300]
    host, want, src, grads, plan = _reducer_setup(n, numels, 500, 22)
    red = rrv.Reducer(plan, grads, "avg")
    red.ready(0)
    with pytest.raises(rrv.RRError):
        red.ready(0)  # twice in one step
    with pytest.raises(rrv.RRError):
        red.finish()  # tensors 1 and 2 never marked
    red.ready(1)
    red.ready(2)
    red.finish()


# ------------------------------------------------------------- bf16 wire --

@pytest.mark.parametrize("algo", ["ring", "oneshot", "auto"])
@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 8, 16])
@pytest.mark.parametrize("op", ["sum", "avg"])
def test_allreduce_bf16_wire(algo, n, op):
    for count in (1, 7, 3 * TILE["f32"] * n + 37):
        x = synth.ranks(14, n, count, "uniform")
        want = [a.copy() for a in x]
        (oracle.ring_allreduce_wire if algo == "ring" else oracle.fold_wire)(want, op)
        d = to_dev(x)
        rrv.all_reduce_wire(d, op, "bf16", algo)
        assert_bits_equal(to_host(d), want, f"wire {algo} n={n} count={count}")


def test_bf16_wire_golden_on_gpu():
    g = {ln.split(":")[0]: [float(v) for v in ln.split(":")[1].split()] for ln in golden_lines("bf16_wire.txt")}
    for algo in ("ring", "oneshot"):
        d = to_dev([np.array(g["inputs_rank0"], np.float32), np.array(g["inputs_rank1"], np.float32)])
        rrv.all_reduce_wire(d, "sum", "bf16", algo)
        for t in to_host(d):
            assert t.tolist() == g["bf16_wire"]


# ----------------------------------------------------- registered rank sets --

@pytest.mark.parametrize("algo", ["oneshot", "ring", "tree_oneshot", "auto"])
def test_rank_set_matches_the_oracle_across_reuse(algo):
    """A RankSet is marshalled once and reused: each call still reduces the
    tensors' current contents."""
    n, count = 8, 3 * TILE["f32"] * 8 + 11
    x = synth.ranks(21, n, count, "uniform")
    d = to_dev(x)
    rs = rrv.RankSet(d)
    want = [a.copy() for a in x]
    ORACLE[algo](want, "sum")
    rrv.all_reduce(rs, "sum", algo)
    assert_bits_equal(to_host(d), want, f"rank set {algo} first call")
    y = synth.ranks(22, n, count, "uniform")
    for t, a in zip(d, y):  # in place: same storage, new values
        t.copy_(torch.from_numpy(a))
    want = [a.copy() for a in y]
    ORACLE[algo](want, "avg")
    rrv.all_reduce(rs, "avg", algo)
    assert_bits_equal(to_host(d), want, f"rank set {algo} reused")


@pytest.mark.parametrize("algo", ["oneshot", "ring", "auto"])
def test_rank_set_bound_call_matches_the_oracle(algo):
    """RankSet.bind converts the arguments once; calling it twice reduces
    twice (the second call reduces the first one's result)."""
    n, count = 8, 8 * 1000 + 3
    x = synth.ranks(33, n, count, "full")
    d = to_dev(x)
    call = rrv.RankSet(d).bind("avg", algo)
    call()
    call()
    want = [a.copy() for a in x]
    oracle.fold_ring_order(want, "avg")
    oracle.fold_ring_order(want, "avg")
    assert_bits_equal(to_host(d), want, f"bound {algo}")


def test_auto_picks_by_the_table_for_the_buffers_alignment():
    """AUTO takes the measured table's choice for the call's rank count, size
    and alignment class -- aligned buffers the aligned points, buffers whose
    16-byte phases differ the points measured with such buffers -- and the
    result has the ring's bits either way."""
    from conftest import picker_table

    _, rows, _ = picker_table()
    mixed = [r for r in rows if r[2] == 2]
    for n in (2, 3, 8):
        count = 1000 * n + 3
        x = synth.ranks(35 + n, n, count, "full")
        want = [a.copy() for a in x]
        oracle.fold_ring_order(want, "sum")
        d = to_dev(x)
        rrv.all_reduce(d, "sum", "auto")
        assert rrv.last_stats()["algo"] == rrv.pick_algo(n, count, "f32")
        assert_bits_equal(to_host(d), want, f"auto aligned n={n}")
        m = to_dev(x, offsets=[r % 4 for r in range(n)])
        rrv.all_reduce(m, "sum", "auto")
        if mixed:
            near = min({r[0] for r in mixed}, key=lambda k: (abs(np.log2(k / n)), k))
            pts = {r[1]: r[3] for r in mixed if r[0] == near}
            lb = int(round(np.log2(count * 4)))
            assert rrv.last_stats()["algo"] == pts[min(pts, key=lambda b: (abs(b - lb), b))]
        assert_bits_equal(to_host(m), want, f"auto mixed n={n}")


def test_rank_set_ring_steps_and_wire():
    n, count = 4, 5000
    x = synth.ranks(23, n, count, "uniform")
    d = to_dev(x)
    rs = rrv.RankSet(d)
    for phase in ("reduce_scatter", "all_gather"):
        for s in range(n - 1):
            rrv.ring_step(rs, "sum", phase, s)
    want = [a.copy() for a in x]
    oracle.ring_allreduce(want, "sum")
    assert_bits_equal(to_host(d), want, "rank set ring steps")
    d = to_dev(x)
    rrv.all_reduce_wire(rrv.RankSet(d), "sum", "bf16", "oneshot")
    want = [a.copy() for a in x]
    oracle.fold_wire(want, "sum")
    assert_bits_equal(to_host(d), want, "rank set wire")


def test_wire_refuses_non_fp32_tensors():
    d = [torch.zeros(16, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    with pytest.raises(TypeError):
        rrv.all_reduce_wire(d, "sum", "bf16", "oneshot")
    with pytest.raises(TypeError):
        rrv.all_reduce_wire(rrv.RankSet(d), "sum", "bf16", "oneshot")


def test_bucket_calls_refuse_gradients_that_do_not_match_the_plan():
    """Sizes, tensor count and dtype of the gradients, and the size of the
    fp32 bucket buffers, are checked before anything is enqueued."""
    numels = [100, 300, 50]
    plan = rrv.BucketPlan(numels, "bf16", 1000)
    good = [[torch.zeros(m, dtype=torch.bfloat16, device="cuda") for m in numels] for _ in range(2)]
    plan.all_reduce(0, good, "avg")  # matches
    short = [[torch.zeros(m - (t == 1), dtype=torch.bfloat16, device="cuda") for t, m in enumerate(numels)]
             for _ in range(2)]
    fewer = [[torch.zeros(m, dtype=torch.bfloat16, device="cuda") for m in numels[:2]] for _ in range(2)]
    fp32 = [[torch.zeros(m, device="cuda") for m in numels] for _ in range(2)]
    ragged = [good[0], [torch.zeros(m + 1, dtype=torch.bfloat16, device="cuda") for m in numels]]
    for bad in (short, fewer, fp32):
        with pytest.raises(ValueError):
            plan.all_reduce(0, bad, "avg")
        with pytest.raises(ValueError):
            plan.all_reduce_range(0, plan.num_buckets, bad, "avg")
        with pytest.raises(ValueError):
            rrv.Reducer(plan, bad)
    with pytest.raises(ValueError):
        rrv.GradSet(ragged)
    numel = plan.info(0)[2]
    small = [torch.zeros(numel - 1, device="cuda") for _ in range(2)]
    with pytest.raises(ValueError):
        plan.pack(0, good, small)
    with pytest.raises(ValueError):
        plan.unpack(0, small, good, "avg")
    gs = rrv.GradSet(good)
    plan.all_reduce(0, gs, "avg")
    plan.all_reduce(0, gs, "avg")  # checked once, reused


# ------------------------------------------------- bulk-copy one-shot path --

@pytest.mark.parametrize("n", [2, 3, 4, 5, 7, 8, 12, 16, 24, 32, 48, 64])
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16", "i32"])
@pytest.mark.parametrize("op", ["sum", "avg", "max", "min", "prod"])
def test_bulk_copy_one_shot(n, dtype, op):
    """Aligned buffers take the one-shot that stages tiles with bulk async
    copies (rank counts 2, 4, 8, 16, 32, 64 fixed at compile time, the others
    as a kernel argument).  count = n*C - (n-1) with C a multiple of 8 makes
    the last chunk end n-1 elements short, inside a vector, so the elements
    past its last whole vector take plain loads."""
    if dtype == "i32" and op == "avg":
        pytest.skip("AVG is not defined for int32")
    C = 8 * 2000
    count = n * C - (n - 1)
    x, _ = _run(n, count, dtype, op, "oneshot", seed=50 + n)
    rrv.check_timeouts()


@pytest.mark.parametrize("n", [3, 4, 6, 8, 24])
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("off", [1, 2, 3])
def test_bulk_copy_one_shot_shared_phase(n, dtype, off):
    """Every rank's buffer `off` elements past a 16-byte boundary, and chunks
    whose length is not a whole number of vectors: each chunk's segment has
    its own scalar head and tail around the bulk-copied vectors, for the
    one-shot (SUM and AVG) and the two-shot's first shot (owner only)."""
    count = n * 3001 + 5
    _run(n, count, dtype, "avg", "oneshot", seed=40 + n, offsets=[off] * n)
    _run(n, count, dtype, "sum", "two_shot", seed=41 + n, offsets=[off] * n)
    rrv.check_timeouts()


@pytest.mark.parametrize("n", [3, 8])
@pytest.mark.parametrize("layout", ["aligned", "mixed"])
def test_bulk_copy_host_slices(n, layout):
    """The host-buffer all-reduce folds each 8 MiB slice as its own launch
    over an element range that cuts chunks: the bulk-copy fold (or, with
    device buffers at different 16-byte phases, the staged kernel) clipped to
    [lo, hi), against the oracle's whole-buffer fold."""
    count = (8 << 20) // 4 * 2 + 4099  # three slices, the last one short
    x = synth.ranks(44 + n, n, count, "full")
    want = [a.copy() for a in x]
    oracle.fold_ring_order(want, "sum")
    host = [torch.from_numpy(a.copy()).pin_memory() for a in x]
    if layout == "aligned":
        dev = [torch.empty(count, device="cuda") for _ in range(n)]
    else:
        dev = [torch.empty(count + 4, device="cuda")[(3 * r + 1) % 4:][:count] for r in range(n)]
    rrv.all_reduce_host(host, dev, "sum", "oneshot")
    torch.cuda.synchronize()
    assert_bits_equal([h.numpy() for h in host], want, f"host slices n={n}")
    rrv.check_timeouts()


def test_bulk_copy_timeouts_are_reported_and_the_context_survives():
    """With RR_DEBUG_BULK_TIMEOUT=1 every barrier expects one arrival more
    than the copying thread makes, so every first bounded wait runs out.  The
    whole CTA then skips its tile (the buffers keep their inputs: nothing
    partly folded is stored), the missing arrival is made and the second wait
    confirms that the tile's copies landed before the CTA left.  Both the
    one-shot and the fused bucket sync report it through RR_ERR_TIMEOUT with
    the tile count, and the context still runs another collective."""
    import os
    import subprocess
    import sys

    script = r'''
import torch, numpy as np
import ring_all_reduce_virtual_b200 as rrv
def report():
    try:
        rrv.check_timeouts()
        print("NO TIMEOUT")
    except rrv.RRError as e:
        print("TIMEOUT", e.status, str(e))
x = [torch.full((2048,), float(r + 1), device="cuda") for r in range(2)]
rrv.all_reduce(x, "sum", "oneshot")  # bulk path: aligned, 2 chunks of 1024 floats, one tile each
report()
assert torch.all(x[0] == 1.0) and torch.all(x[1] == 2.0), "a skipped tile was stored"
plan = rrv.BucketPlan([4096], "bf16", 1 << 20)  # one bucket, 2 chunks of 2048 bf16, one tile each
g = [[torch.full((4096,), float(r + 1), device="cuda").to(torch.bfloat16)] for r in range(2)]
plan.all_reduce(0, g, "sum")
report()
assert torch.all(g[0][0] == 1.0) and torch.all(g[1][0] == 2.0), "a skipped bucket tile was stored"
rrv.check_timeouts()  # cleared
y = [torch.full((2048,), float(r + 1), device="cuda") for r in range(3)]
rrv.all_reduce(y, "sum", "ring")  # another path on the same context
assert torch.all(y[0] == 6.0) and torch.all(y[2] == 6.0)
print("CONTEXT OK")
'''
    env = dict(os.environ, RR_DEBUG_BULK_TIMEOUT="1")
    out = subprocess.run([sys.executable, "-c", script], env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("TIMEOUT")]
    assert len(lines) == 2, out.stdout
    for ln in lines:
        assert ln.startswith("TIMEOUT 4") and "on 2 tiles" in ln and "not seen to land: 0" in ln, ln
    assert "CONTEXT OK" in out.stdout, out.stdout


@pytest.mark.parametrize("n", [2, 3, 4, 5, 6, 7, 8, 12, 16, 24])
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16", "i32"])
@pytest.mark.parametrize("op", ["sum", "avg", "max", "min", "prod"])
def test_bulk_copy_reduce_scatter_and_tree_order(n, dtype, op):
    """Parts (reduce-scatter, any rank count) and buffers (tree order, 2-8,
    12 and 16 ranks, an unpaired block carried up) of whole 16-byte vectors at
    aligned addresses take the bulk-copy kernels: same bits as the oracle."""
    if dtype == "i32" and op == "avg":
        pytest.skip("AVG is not defined for int32")
    per = 8 * 1500
    x = synth.ranks(60 + n, n, n * per, _dist(op, dtype), dtype)
    rs = empty_like_ranks(n, per, dtype)
    rrv.reduce_scatter(to_dev(x), rs, op)
    assert_bits_equal(to_host(rs), oracle.reduce_scatter([a.copy() for a in x], op), f"bulk rs {op}")
    _run(n, n * per, dtype, op, "tree_oneshot", seed=70 + n)
    rrv.check_timeouts()


@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64])
@pytest.mark.parametrize("op", ["sum", "avg"])
def test_bulk_copy_bf16_wire(n, op):
    C = 8 * 2000
    count = n * C - (n - 1)  # a ragged last chunk: its last elements take plain loads
    x = synth.ranks(80 + n, n, count, "uniform")
    want = [a.copy() for a in x]
    oracle.fold_wire(want, op)
    d = to_dev(x)
    rrv.all_reduce_wire(d, op, "bf16", "oneshot")
    assert_bits_equal(to_host(d), want, f"bulk wire n={n}")
    rrv.check_timeouts()


@pytest.mark.parametrize("n", [2, 3, 5, 8, 64])
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16", "i32"])
def test_aligned_all_gather_and_two_shot(n, dtype):
    """Parts of whole 16-byte vectors at aligned addresses (the vector path
    with no scalar head or tail) for the all-gather and the two-shot; the
    two-shot count leaves a short last chunk."""
    per = 8 * 1500
    x = synth.ranks(90 + n, n, per, "int" if dtype == "i32" else "uniform", dtype)
    ag = empty_like_ranks(n, n * per, dtype)
    rrv.all_gather(to_dev(x), ag)
    assert_bits_equal(to_host(ag), oracle.all_gather(x), f"bulk ag n={n}")
    if n <= 8:
        count = n * per - 8 * (n - 1)  # C = per: the last chunk is 8(N-1) elements short
        _run(n, count, dtype, "sum", "two_shot", seed=95 + n)
    rrv.check_timeouts()


@pytest.mark.parametrize("n", [2, 3, 5, 8, 16, 64])
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16", "i32"])
def test_one_shot_over_ranks_at_different_phases(n, dtype):
    """Rank buffers whose addresses differ modulo 16 bytes: each rank's tile is
    staged at its own shift and every output gets whole vectors at its own
    phase (plus scalar heads and tails); ragged chunks over several tiles,
    every op, the two-shot's owner-only first shot, the tree's order, the
    reduce-scatter and the bf16 wire too."""
    L = 4 if dtype in ("f32", "i32") else 8
    offsets = [(3 * r + 1) % L for r in range(n)]
    if len(set(offsets)) == 1:
        offsets[0] = (offsets[0] + 1) % L
    count = n * 1500 + 7
    ops = ("sum", "max", "min", "prod") if dtype == "i32" else ("sum", "avg", "max", "prod")
    for op in ops:
        _run(n, count, dtype, op, "oneshot", seed=400 + n, offsets=offsets)
    _run(n, count, dtype, "sum", "two_shot", seed=410 + n, offsets=offsets)
    _run(n, 3, dtype, "sum", "oneshot", seed=420 + n, offsets=offsets)  # fewer elements than ranks
    for op in ops[:2]:  # the tree's pairwise order, staged the same way (up to 16 ranks)
        _run(n, count, dtype, op, "tree_oneshot", seed=450 + n, offsets=offsets)
    # the reduce-scatter: inputs at the ranks' phases, outputs at other ones
    per = 1500 + 3
    x = synth.ranks(430 + n, n, n * per, _dist("sum", dtype), dtype)
    rs = to_dev([np.zeros(per, dtype=a.dtype) for a in x], offsets=offsets[::-1])
    op = "max" if dtype == "i32" else "avg"
    rrv.reduce_scatter(to_dev(x, offsets=offsets), rs, op)
    assert_bits_equal(to_host(rs), oracle.reduce_scatter([a.copy() for a in x], op), f"rs {op} n={n}")
    if dtype == "f32":  # the bf16 wire format of the one-shot
        y = synth.ranks(440 + n, n, count, "full")
        want = [a.copy() for a in y]
        oracle.fold_wire(want, "avg")
        d = to_dev(y, offsets=offsets)
        rrv.all_reduce_wire(d, "avg", "bf16", "oneshot")
        assert_bits_equal(to_host(d), want, f"wire n={n}")


def _near_midpoints(rng, n, size):
    """fp32 values next to n * m, m a midpoint between neighbouring fp32
    values: the quotients closest to a rounding boundary."""
    m = (rng.integers(1 << 23, 1 << 24, size=size) + 0.5) * np.exp2(rng.integers(-140, 100, size=size) - 23.0)
    near = (m * n).astype(np.float32)
    near = np.concatenate([near, np.nextafter(near, np.float32(np.inf)), np.nextafter(near, np.float32(0))])
    return near[np.isfinite(near)]


@pytest.mark.parametrize("n", [3, 5, 6, 7, 12, 24, 48, 63])
@pytest.mark.parametrize("algo", ["oneshot", "two_shot", "ring"])
def test_avg_quotient_hard_cases(n, algo):
    """AVG's quotient for rank counts that are not powers of two, on the
    values whose quotient lies closest to an fp32 rounding boundary, on
    subnormals, zeros, infinities and random bits of every binade: rank 0
    holds the values, every other rank zeros, so each element's fold is the
    value itself and the result is its quotient by N -- IEEE's, bit for bit,
    and the oracle's."""
    rng = np.random.default_rng(300 + n)
    bits = rng.integers(0, 0x7F800000, size=4096, dtype=np.uint32) | (rng.integers(0, 2, 4096, dtype=np.uint32) << 31)
    special = np.array([0.0, np.inf, -np.inf, 1e-45, -1e-45, 1.1754942e-38, 3.4028235e38, 1.0, 3.0], dtype=np.float32)
    x0 = np.concatenate([bits.view(np.float32), special, _near_midpoints(rng, n, 2048)]).astype(np.float32)
    x = [x0] + [np.zeros_like(x0) for _ in range(n - 1)]
    want = [a.copy() for a in x]
    oracle.fold_ring_order(want, "avg")
    quot = x0 / np.float32(n)
    for w in want:
        assert np.array_equal(bits_of(w), bits_of(quot))  # the oracle: IEEE's quotient
    d = to_dev(x)
    rrv.all_reduce(d, "avg", algo)
    assert_bits_equal(to_host(d), want, f"avg {algo} n={n}")


def bits_of(a):
    return np.ascontiguousarray(a).view(np.uint32)


@pytest.mark.parametrize("n", [3, 5, 8, 12, 16])
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("off", [0, 1, 3])
def test_tree_order_bulk_heads_and_tails(n, dtype, off):
    """The tree-order one-shot on the bulk-copy fold with every buffer at one
    16-byte phase: a scalar head (buffers `off` elements past a boundary) and
    a ragged tail, folded in the tree's order by tile 0, whole vectors
    between, over several tiles."""
    L = 4 if dtype == "f32" else 8
    if off >= L:
        pytest.skip("offset within one vector")
    count = 3 * TILE[dtype] + 5
    for op in ("sum", "avg"):
        _run(n, count, dtype, op, "tree_oneshot", seed=170 + n + off, offsets=[off] * n)
    rrv.check_timeouts()


@pytest.mark.parametrize("n", [2, 5, 9, 13])
@pytest.mark.parametrize("dtype", ["f32", "bf16", "i32"])
@pytest.mark.parametrize("layout", ["same", "mixed"])
def test_one_to_many_copies_by_output_phase(n, dtype, layout):
    """The all-gather and the two-shot's broadcast write several outputs per
    work item when every output sits at one 16-byte phase ("same": all one
    element past a boundary, so each block has a scalar head) and one output
    per item otherwise ("mixed"); rank counts that leave a partial last group
    of outputs, sources at other phases, parts over several tiles."""
    L = 4 if dtype in ("f32", "i32") else 8
    per = 2 * TILE_MOVE[dtype] + 3
    src_off = [(3 * r + 2) % L for r in range(n)]
    out_off = [1] * n if layout == "same" else [r % L for r in range(n)]
    x = synth.ranks(140 + n, n, per, "int" if dtype == "i32" else "full", dtype)
    zero = [np.zeros(n * per, dtype=a.dtype) for a in x]
    ag = to_dev(zero, offsets=out_off)
    rrv.all_gather(to_dev(x, offsets=src_off), ag)
    assert_bits_equal(to_host(ag), oracle.all_gather(x), f"ag {layout} n={n}")
    count = n * per - 5
    _run(n, count, dtype, "sum", "two_shot", seed=150 + n, offsets=out_off)


@pytest.mark.parametrize("n", [2, 3, 4, 5, 8, 12, 16, 24, 33, 64])
@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
def test_bucket_sync_bulk_path_with_heads_and_tails(n, dtype):
    """Tensors at odd element offsets, the same on every rank: the fused
    bucket sync takes the bulk-copy fold, whose tile 0 folds each segment's
    elements before its first 16-byte boundary and after its last whole
    vector with plain loads."""
    numels = [7, 1001, 3, 2500, 64, 12345, 1]
    es = 4 if dtype == "f32" else 2
    host = _grad_set(13, n, numels, dtype)
    want = [[g.copy() for g in rank] for rank in host]
    cap = 3000 * es
    oracle.bucket_sync(want, cap, "avg")
    plan = rrv.BucketPlan(numels, dtype, cap)
    td = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[dtype]
    grads = []
    for r in range(n):
        flat = torch.zeros(sum(numels) + 8 * len(numels) + 8, dtype=td, device="cuda")
        ts, o = [], 1  # every rank: the same odd offsets
        for g in host[r]:
            t = flat[o:o + g.size]
            t.copy_(torch.from_numpy(g.view(np.int16) if dtype == "bf16" else g).cuda().view(td))
            ts.append(t)
            o += g.size + 3
        grads.append(ts)
    plan.all_reduce_range(0, plan.num_buckets, grads, "avg")
    for r in range(n):
        assert_bits_equal(to_host(grads[r]), want[r], f"rank {r}")
    rrv.check_timeouts()


C_GPU_CLIENT = r"""
#include <stdio.h>
#include <cuda_runtime_api.h>
#include "rr.h"

/* The pages' 4-rank example from plain C: x_r = arange(4) + 10 r; the
 * all-reduce (SUM) is [60, 64, 68, 72] on every rank, the reduce-scatter
 * gives rank r element r of it, and the all-gather of those parts is the
 * all-reduce again. */
int main(void)
{
    enum { N = 4, C = 4 };
    float* d[N];
    float* part[N];
    float* ag[N];
    for (int r = 0; r < N; ++r) {
        float h[C];
        for (int i = 0; i < C; ++i) h[i] = (float)(i + 10 * r);
        if (cudaMalloc((void**)&d[r], sizeof h) != cudaSuccess) return 1;
        if (cudaMalloc((void**)&part[r], sizeof(float)) != cudaSuccess) return 1;
        if (cudaMalloc((void**)&ag[r], sizeof h) != cudaSuccess) return 1;
        cudaMemcpy(d[r], h, sizeof h, cudaMemcpyHostToDevice);
    }
    if (rr_reduce_scatter((const void* const*)d, (void* const*)part, N, 1, RR_F32, RR_SUM, RR_ALGO_AUTO, 0) != RR_OK)
        return 2;
    if (rr_allreduce((void* const*)d, N, C, RR_F32, RR_SUM, RR_ALGO_RING, 0) != RR_OK) return 3;
    if (rr_all_gather((const void* const*)part, (void* const*)ag, N, 1, RR_F32, RR_ALGO_AUTO, 0) != RR_OK) return 4;
    if (cudaDeviceSynchronize() != cudaSuccess) return 5;
    const float want[C] = {60.f, 64.f, 68.f, 72.f};
    for (int r = 0; r < N; ++r) {
        float h[C], g[C], p;
        cudaMemcpy(h, d[r], sizeof h, cudaMemcpyDeviceToHost);
        cudaMemcpy(g, ag[r], sizeof g, cudaMemcpyDeviceToHost);
        cudaMemcpy(&p, part[r], sizeof p, cudaMemcpyDeviceToHost);
        for (int i = 0; i < C; ++i)
            if (h[i] != want[i] || g[i] != want[i]) return 6;
        if (p != want[r]) return 7;
        cudaFree(d[r]);
        cudaFree(part[r]);
        cudaFree(ag[r]);
    }
    printf("c gpu client ok\n");
    return 0;
}
"""


def test_c_client_reproduces_the_four_rank_example(tmp_path):
    """The boundary from plain C on the GPU (no Python, no torch): cudaMalloc'd
    rank buffers, the ring all-reduce, reduce-scatter and all-gather of the
    pages' 4-rank worked example."""
    import os
    import shutil
    import subprocess

    from ring_all_reduce_virtual_b200 import _lib

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "client_gpu.c"
    src.write_text(C_GPU_CLIENT)
    exe = tmp_path / "client_gpu"
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    lib_dir = os.path.dirname(_lib.LIB_PATH)
    cuda_lib = "/usr/local/cuda/lib64"
    r = subprocess.run([gcc, "-std=c11", "-Wall", "-Werror", "-I", os.path.join(root, "include"),
                        "-I", "/usr/local/cuda/include", str(src), "-o", str(exe), "-L", lib_dir, "-lrr_virtual",
                        "-L", cuda_lib, "-lcudart", f"-Wl,-rpath,{lib_dir}", f"-Wl,-rpath,{cuda_lib}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and "c gpu client ok" in run.stdout, (run.returncode, run.stdout, run.stderr)
