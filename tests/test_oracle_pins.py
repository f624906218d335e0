"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here retypes the oracle's formulas: each test checks the oracle
against a value the pages print (golden fixtures), a closed form, an
invariant, a library routine on a case that reduces to it, an error bound, or
brute force on tiny inputs.  ``test_mutants_are_caught`` then shows that each
planted mistake in the oracle fails at least one of these pins.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from conftest import golden_lines
from ring_all_reduce_virtual_b200 import synth


def _vals(line):
    return [float(v) for v in line.split(":", 1)[1].split()]


def _arange4(dtype="f32"):
    return synth.ranks(0, 4, 4, "arange", dtype)


# ------------------------------------------------------ worked example --

def _p4_expect():
    t = {}
    for ln in golden_lines("five_primitives_4rank.txt"):
        head, rest = ln.split(":", 1)
        parts = head.split()
        if len(parts) == 2:
            t.setdefault(parts[0], {})[int(parts[1])] = [float(v) for v in rest.split()]
        else:
            t[parts[0]] = rest.strip()
    return t


@pytest.mark.parametrize("dtype", ["f32", "i32", "bf16", "f16"])
@pytest.mark.parametrize("path", ["ring", "fold", "naive", "tree", "tree_fold"])
def test_worked_example_allreduce(path, dtype):
    exp = _p4_expect()
    x = _arange4(dtype)
    for r in range(4):
        assert _as_float(x[r]).tolist() == exp["input"][r]
    {"ring": oracle.ring_allreduce, "fold": oracle.fold_ring_order, "naive": oracle.naive_allreduce,
     "tree": oracle.tree_schedule, "tree_fold": oracle.tree_fold}[path](x, "sum")
    for r in range(4):
        assert _as_float(x[r]).tolist() == exp["all_reduce"][r]


def _as_float(a):
    return oracle.bf16_to_f32(a) if a.dtype == np.uint16 else a.astype(np.float64)


def test_worked_example_rs_ag_a2a():
    exp = _p4_expect()
    x = _arange4()
    rs = oracle.reduce_scatter(x, "sum")
    ag = oracle.all_gather(rs)
    a2a = oracle.all_to_all(x)
    ar = [a.copy() for a in x]
    oracle.ring_allreduce(ar, "sum")
    for r in range(4):
        assert rs[r].tolist() == exp["reduce_scatter"][r]
        assert ag[r].tolist() == exp["all_gather"][r]
        assert a2a[r].tolist() == exp["all_to_all"][r]
    same = all(np.array_equal(ag[r], ar[r]) for r in range(4))
    assert str(same) == exp["rs_then_ag_equals_ar"]


def test_worked_example_avg_is_sum_over_n():
    # [P3] section 3: the gathered sum is divided by 4 -> (60, 64, 68, 72) / 4
    x = _arange4()
    oracle.ring_allreduce(x, "avg")
    for r in range(4):
        assert x[r].tolist() == [15.0, 16.0, 17.0, 18.0]


# ------------------------------------------------------- byte accounting --

def test_ring_bytes_golden():
    g = dict(ln.split(":", 1) for ln in golden_lines("ring_bytes_4rank.txt"))
    n, m = int(g["ranks"]), int(g["elements_per_rank"])
    x = [torch.randn(m, generator=torch.Generator().manual_seed(r)).numpy() for r in range(n)]
    assert x[0].nbytes == int(g["bytes_per_rank"])
    ref = np.sum(np.stack(x).astype(np.float64), axis=0)
    sent = oracle.ring_allreduce(x, "sum")
    assert sent.tolist() == [int(v) for v in g["sent"].split()]
    # the page's own check against the library all-reduce: allclose(atol=1e-5)
    atol = float(g["matches_library_all_reduce_atol"])
    for r in range(n):
        assert np.allclose(x[r], ref, atol=atol)


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 7, 8, 16, 64])
def test_ring_bytes_closed_form(n):
    # [P3] section 4 / [P4]: each rank sends 2(N-1)/N * S when N divides the count
    for per in [1, 3, 16]:
        count = n * per
        x = synth.ranks(1, n, count, "uniform")
        sent = oracle.ring_allreduce(x)
        s = count * 4
        assert sent.tolist() == [2 * (n - 1) * s // n] * n


@pytest.mark.parametrize("n,count", [(3, 10), (4, 5), (8, 3), (5, 0), (16, 17)])
def test_ring_bytes_ragged_total(n, count):
    # each step is a permutation of the N chunks, so all ranks together send
    # exactly S per step whatever the split: 2(N-1) * S in all
    x = synth.ranks(2, n, count, "uniform")
    sent, trace = oracle.ring_allreduce(x, trace=True)
    assert int(sent.sum()) == 2 * (n - 1) * count * 4
    for phase in (0, 1):
        for s in range(n - 1):
            evs = [e for e in trace if e["phase"] == phase and e["step"] == s]
            assert sorted(e["send_idx"] for e in evs) == list(range(n))


# ------------------------------------------------- the 4-GPU walkthrough --

def test_p3_four_gpu_walkthrough():
    # pow2 inputs: rank r holds 2^r, so a summed value names its contributors
    lines = golden_lines("four_gpu_walkthrough.txt")
    n = 4
    x = synth.ranks(0, n, 4, "pow2")
    events = {}
    holds = {}
    for s in range(n - 1):
        events[s] = oracle.ring_step(x, "sum", oracle.PHASE_RS, s)
        holds[s] = [a.copy() for a in x]
    for ln in lines:
        head, rest = ln.split(":", 1)
        if head.startswith("send"):
            s = int(head.split()[1])
            sender, chunk, recv = map(int, rest.split())
            e = events[s][sender]
            assert (e["send_idx"], e["dst"]) == (chunk, recv)
        elif head.startswith("holds"):
            s = int(head.split()[1])
            left, right = rest.split("=")
            gpu, chunk = map(int, left.split())
            contrib = sum(2 ** int(v) for v in right.split())
            assert holds[s][gpu][chunk] == contrib
        elif head == "steps":
            _, trace = oracle.ring_allreduce(synth.ranks(0, n, 4, "pow2"), trace=True)
            assert len({(e["phase"], e["step"]) for e in trace}) == int(rest)


@pytest.mark.parametrize("n", [2, 3, 4, 5, 8])
def test_after_reduce_scatter_each_rank_owns_one_full_chunk(n):
    # [P3] section 3 / [P4]: after N-1 steps every rank holds exactly one
    # chunk reduced over all N ranks, a different one on each rank
    x = synth.ranks(0, n, n, "pow2")
    for s in range(n - 1):
        oracle.ring_step(x, "sum", oracle.PHASE_RS, s)
    full = 2 ** n - 1
    owned = [[k for k in range(n) if x[r][k] == full] for r in range(n)]
    assert all(len(o) == 1 for o in owned)
    assert sorted(o[0] for o in owned) == list(range(n))


# --------------------------------------------------- fold order (rounding) --

def _fold_fixture():
    n = 4
    big = np.float32(2.0 ** 24)
    x = [np.zeros(n, dtype=np.float32) for _ in range(n)]
    pattern = [np.float32(1), big, np.float32(1), -big]
    for i in range(n):
        for k, v in enumerate(pattern):
            x[(i + k) % n][i] = v
    return x


def test_fold_order_golden():
    g = {ln.split(":")[0]: _vals(ln) for ln in golden_lines("fold_order.txt")}
    for f in (oracle.ring_allreduce, oracle.fold_ring_order):
        x = _fold_fixture()
        f(x, "sum")
        for r in range(4):
            assert x[r].tolist() == g["ring_order"]
    # a reduce-scatter followed by an all-gather gives the same bits
    x = _fold_fixture()
    ag = oracle.all_gather(oracle.reduce_scatter(x, "sum"))
    for r in range(4):
        assert ag[r].tolist() == g["ring_order"]
    # the sampled fold agrees, and the other starts give the fixture's values
    x = _fold_fixture()
    vals = np.stack(x)
    for key, off in (("ring_order", 0), ("start_plus_1", 1), ("start_plus_2", 2), ("start_plus_3", 3)):
        start = (np.arange(4) + off) % 4
        assert oracle.fold_samples(vals, start).tolist() == g[key]


def test_naive_rank_order_on_fold_fixture():
    # the naive method folds in rank order 0..3; element 0 starts at rank 0
    # (same as the ring), element 3 starts at rank 0 = its chunk + 1
    g = {ln.split(":")[0]: _vals(ln) for ln in golden_lines("fold_order.txt")}
    x = _fold_fixture()
    oracle.naive_allreduce(x, "sum")
    assert x[0][0] == g["ring_order"][0]
    assert x[0][3] == g["start_plus_1"][3]


# ------------------------------------------------------------ brute force --

def _np_reduce(x, op):
    a = np.stack([_as_float(v) for v in x])
    if op in ("sum", "avg"):
        r = a.sum(0)
        return r / len(x) if op == "avg" else r
    return {"max": a.max(0), "min": a.min(0), "prod": a.prod(0)}[op]


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("op", ["sum", "max", "min", "prod"])
@pytest.mark.parametrize("dtype", ["f32", "i32", "bf16"])
def test_brute_force_integer_data(n, op, dtype):
    # integer-valued inputs small enough that every order is exact: all
    # oracle paths agree bit for bit with numpy's reduction in float64
    for count in [0, 1, n - 1 if n > 1 else 1, 2 * n + 3, 37]:
        lo, hi = (-3, 4) if op == "prod" else (-100, 100)
        if dtype == "bf16" and op == "sum":
            lo, hi = -16, 16
        if dtype == "bf16" and op == "prod":
            lo, hi = -2, 3
        rng = np.random.default_rng([n, count])
        raw = [rng.integers(lo, hi, size=count) for _ in range(n)]
        x0 = [synth.cast(v, dtype) for v in raw]
        want = _np_reduce(x0, op)
        for path in (oracle.ring_allreduce, oracle.fold_ring_order, oracle.naive_allreduce,
                     oracle.tree_schedule, oracle.tree_fold):
            x = [v.copy() for v in x0]
            path(x, op)
            for r in range(n):
                assert np.array_equal(_as_float(x[r]), want), (path.__name__, r)


def test_avg_is_one_division_of_the_sum():
    # AVG = fl(SUM / N): check against numpy's float32 division of the fold
    for n in [3, 5, 8]:
        x = synth.ranks(4, n, 1000, "uniform")
        s = [v.copy() for v in x]
        oracle.ring_allreduce(s, "sum")
        oracle.ring_allreduce(x, "avg")
        assert np.array_equal(x[0], (s[0] / np.float32(n)).astype(np.float32))


# ---------------------------------------------------- fp32 error bound --

@pytest.mark.parametrize("n", [2, 3, 4, 8, 16, 64])
@pytest.mark.parametrize("dist", ["uniform", "normal"])
def test_fp32_fold_within_error_bound(n, dist):
    # |fl(sum) - sum| <= gamma_{N-1} * sum |x|, gamma_k = k u / (1 - k u),
    # u = 2^-24 (recursive summation, Higham, Accuracy and Stability, 4.2)
    count = 4 * n + 5
    x = synth.ranks(5, n, count, dist)
    a = np.stack(x).astype(np.float64)
    exact, mag = a.sum(0), np.abs(a).sum(0)
    oracle.ring_allreduce(x, "sum")
    u = 2.0 ** -24
    gamma = (n - 1) * u / (1 - (n - 1) * u)
    # the float64 reference itself may be off by N ulps of float64
    assert np.all(np.abs(x[0].astype(np.float64) - exact) <= (gamma + 1e-14) * mag)


def test_prod_within_error_bound():
    n = 64
    x = synth.ranks(6, n, 999, "prod")
    exact = np.prod(np.stack(x).astype(np.float64), axis=0)
    oracle.ring_allreduce(x, "prod")
    u = 2.0 ** -24
    gamma = (n - 1) * u / (1 - (n - 1) * u)
    assert np.all(np.abs(x[0] - exact) <= (gamma + 1e-14) * np.abs(exact))


# ------------------------------------------------- two oracle paths agree --

@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 8, 13, 16])
@pytest.mark.parametrize("op", ["sum", "avg", "max", "min", "prod"])
def test_ring_steps_equal_direct_fold_fp32(n, op):
    for count in [0, 1, n, 3 * n + 1, 257]:
        dist = "prod" if op == "prod" else "uniform"
        x = synth.ranks(7, n, count, dist)
        y = [v.copy() for v in x]
        oracle.ring_allreduce(x, op)
        oracle.fold_ring_order(y, op)
        for r in range(n):
            assert np.array_equal(x[r].view(np.uint32), y[r].view(np.uint32))
            assert np.array_equal(x[r].view(np.uint32), x[0].view(np.uint32))


# ---------------------- the timed ring and the sampled fold vs the pinned ones --
# ``ring_allreduce_omp`` (the timed CPU baseline) and ``fold_samples`` (the
# checker of every sampled full-size GPU test) are separate code in the C
# file.  Each is held here to a pinned path bit for bit: the OpenMP ring to
# the message-stepping ring, the sampled fold to the whole-buffer fold.

def _draw(seed, n, count, op, dtype):
    dist = "int" if dtype == "i32" else ("prod" if op == "prod" else "uniform")
    return synth.ranks(seed, n, count, dist, dtype)


def _ops_for(dtype):
    return ["sum", "max", "min", "prod"] + ([] if dtype == "i32" else ["avg"])


def _omp_matches(n, dtype, threads=(1, 4)):
    for op in _ops_for(dtype):
        for count in (0, 1, n + 1, 3 * n + 2, 1000):
            x = _draw(11, n, count, op, dtype)
            want = [v.copy() for v in x]
            oracle.ring_allreduce(want, op)
            for nt in threads:
                got = [v.copy() for v in x]
                oracle.ring_allreduce_omp(got, op, nt)
                for r in range(n):
                    assert np.array_equal(got[r].view(np.uint8), want[r].view(np.uint8)), (op, count, nt, r)


@pytest.mark.parametrize("n", [1, 2, 3, 5, 8, 13, 64])
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16", "i32"])
def test_ring_omp_equals_the_pinned_ring(n, dtype):
    # ragged (n + 1, 3n + 2, 1000) and empty counts, every op, one thread and
    # several: the parallel transfers of a step give the stepping ring's bits
    _omp_matches(n, dtype, (1, 4, os.cpu_count() or 1))


def _samples_match(n, dtype, m=200):
    count = 7 * n + 3  # ragged last chunk
    C = oracle.chunk_size(count, n)
    rng = np.random.default_rng([n, 12])
    idx = rng.integers(0, count, size=m)
    idx[:3] = [0, count - 1, min(C, count - 1)]  # first, last, a chunk boundary
    for op in _ops_for(dtype):
        x = _draw(12, n, count, op, dtype)
        want = [v.copy() for v in x]
        oracle.fold_ring_order(want, op)
        vals = np.stack(x)[:, idx]
        got = oracle.fold_samples(vals, idx // C, op)
        assert np.array_equal(got.view(np.uint8), want[0][idx].view(np.uint8)), op


@pytest.mark.parametrize("n", [1, 2, 3, 5, 8, 16, 64])
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16", "i32"])
def test_fold_samples_equals_the_pinned_fold(n, dtype):
    # random sample positions with their chunk index as the fold's start
    _samples_match(n, dtype)


def test_ring_bf16_per_hop_rounding_stays_near_fp32_fold():
    n, count = 8, 4096
    x = synth.ranks(8, n, count, "normal", "bf16")
    y = [v.copy() for v in x]
    oracle.ring_allreduce(x, "avg")
    oracle.fold_ring_order(y, "avg")
    a, b = oracle.bf16_to_f32(x[0]), oracle.bf16_to_f32(y[0])
    assert np.allclose(a, b, atol=1e-2, rtol=1e-2)


def test_bf16_fold_rounds_once_like_torch():
    # bf16 one-shot = fp32 fold of the widened values, then one RNE, which
    # torch's CPU conversion also performs
    n = 8
    x = synth.ranks(9, n, 3000, "normal", "bf16")
    wide = [oracle.bf16_to_f32(v) for v in x]
    oracle.fold_ring_order(wide, "avg")
    oracle.fold_ring_order(x, "avg")
    want = torch.from_numpy(wide[0]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(x[0], want)


# ------------------------------------------------------- max/min reading --

def test_max_min_match_numpy_without_ties():
    x = synth.ranks(10, 7, 500, "uniform")
    for op, f in (("max", np.max), ("min", np.min)):
        y = [v.copy() for v in x]
        oracle.ring_allreduce(y, op)
        assert np.array_equal(y[3], f(np.stack(x), axis=0))


def test_max_signed_zero_tie_keeps_left_operand():
    # stated reading: on ties the partial that arrived first is kept, so the
    # sign of a zero result tells where the fold started
    n = 4
    x = [np.full(n, -1.0, dtype=np.float32) for _ in range(n)]
    for i in range(n):
        x[i][i] = 0.0
        x[(i + 1) % n][i] = -0.0
    oracle.ring_allreduce(x, "max")
    assert all(not np.signbit(v) for v in x[0])


# ------------------------------------------------------------------- tree --

def test_tree_two_ranks_equals_ring_and_naive():
    x = synth.ranks(11, 2, 1001, "uniform")
    outs = []
    for f in (oracle.ring_allreduce, oracle.naive_allreduce, oracle.tree_schedule, oracle.tree_fold):
        y = [v.copy() for v in x]
        f(y, "sum")
        outs.append(y[1])
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


@pytest.mark.parametrize("n,steps", [(1, 0), (2, 2), (3, 4), (4, 4), (8, 6), (16, 8), (64, 12)])
def test_tree_steps_are_two_log2_n(n, steps):
    # [P3] section 6 table: 2 log2 N steps
    x = synth.ranks(12, n, 8, "int")
    assert oracle.tree_schedule(x) == steps


def test_tree_pairwise_order_on_rounding_fixture():
    # N=4 tree: (x0 + x1) + (x2 + x3).  With element 0 of the fold fixture,
    # x0 = 1, x1 = 2^24, x2 = 1, x3 = -2^24: (2^24) + (1 - 2^24) = 1.
    x = _fold_fixture()
    oracle.tree_schedule(x, "sum")
    assert x[0][0] == 1.0
    y = _fold_fixture()
    oracle.tree_fold(y, "sum")
    assert np.array_equal(x[2], y[2])


def _tree_unpaired_cases():
    for ln in golden_lines("tree_order_unpaired.txt"):
        n, xs, want = ln.split(":")
        yield int(n), [np.float32(float(v)) for v in xs.split()], float(want)


def test_tree_order_with_unpaired_ranks_golden():
    """The hand-derived fixture pins where a rank without a partner joins the
    pairwise tree (N = 3, 5, 6, 7), for the tree schedule and its fused form."""
    for n, xs, want in _tree_unpaired_cases():
        assert len(xs) == n
        for path in (oracle.tree_schedule, oracle.tree_fold):
            x = [np.array([v], dtype=np.float32) for v in xs]
            path(x, "sum")
            for r in range(n):
                assert float(x[r][0]) == want, (path.__name__, n, r, float(x[r][0]))


def test_tree_unpaired_mutant_is_caught():
    # kind 13: the unpaired rank joins the pair before it at the same level
    with oracle.mutant(13):
        with pytest.raises(AssertionError):
            test_tree_order_with_unpaired_ranks_golden()
    test_tree_order_with_unpaired_ranks_golden()


# ------------------------------------------------------------------- bf16 --

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(13)
    bits = rng.integers(0, 2 ** 32, size=200000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    ties = (np.arange(4096, dtype=np.uint32) << 16) | np.uint32(0x8000)
    f = np.concatenate([f, ties.view(np.float32)[np.isfinite(ties.view(np.float32))],
                        np.array([0.0, -0.0, np.inf, -np.inf, 3.4e38, -3.4e38, 1e-40, 1e-45], np.float32)])
    want = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f32_to_bf16(f), want)
    assert np.array_equal(oracle.bf16_to_f32(want), torch.from_numpy(want.view(np.int16)).view(
        torch.bfloat16).float().numpy())


def test_bf16_rounding_hand_cases():
    # 1 + 2^-8 is halfway between bf16 1.0 and 1 + 2^-7: ties to even -> 1.0
    # 1 + 3 * 2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6: even -> 1 + 2^-6
    x = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 1 + 2.0 ** -8 + 2.0 ** -20], dtype=np.float32)
    got = oracle.bf16_to_f32(oracle.f32_to_bf16(x))
    assert got.tolist() == [1.0, 1 + 2.0 ** -6, 1 + 2.0 ** -7]


# ---------------------------------------------------------------- buckets --

def test_bucket_plan_invariants_gpt_like():
    tensors = synth.grad_ready_order(synth.gpt_grad_tensors())
    numels = [m for _, m in tensors]
    assert len(numels) == 293 and sum(numels) == 1343868928
    cap = synth.BUCKET_CAP_BYTES
    b, off, nb = oracle.bucket_plan(numels, 2, cap)
    _check_plan(numels, 2, cap, b, off, nb)
    # tensors at least as large as the cap close the bucket they join
    for t, m in enumerate(numels):
        if m * 2 >= cap and t + 1 < len(numels):
            assert b[t + 1] == b[t] + 1


def _check_plan(numels, es, cap, b, off, nb):
    assert list(b) == sorted(b) and (len(b) == 0 or (b[0] == 0 and b[-1] == nb - 1))
    for k in range(nb):
        members = [t for t in range(len(numels)) if b[t] == k]
        assert members, "no empty buckets"
        o = 0
        for t in members:  # offsets are the running element count
            assert off[t] == o
            o += numels[t]
        sizes = [numels[t] * es for t in members]
        if k < nb - 1:
            assert sum(sizes) >= cap
        if len(sizes) > 1:  # closed as soon as it reached the cap
            assert sum(sizes[:-1]) < cap


def test_bucket_plan_invariants_admit_only_the_greedy_partition():
    """The invariants determine the plan: every other contiguous partition of
    a small example fails them (bf16, cap 60 bytes: 10 and 20 elements fill
    the first bucket exactly, 30 and 40 are buckets of their own)."""
    import itertools

    numels, es, cap = [10, 20, 30, 40], 2, 60
    b, off, nb = oracle.bucket_plan(numels, es, cap)
    assert list(b) == [0, 0, 1, 2]
    passing = []
    for cuts in itertools.product([0, 1], repeat=len(numels) - 1):  # 1 = a new bucket after tensor t
        bb = [0]
        for c in cuts:
            bb.append(bb[-1] + c)
        oo, run = [], {}
        for t, k in enumerate(bb):
            oo.append(run.get(k, 0))
            run[k] = run.get(k, 0) + numels[t]
        try:
            _check_plan(numels, es, cap, np.array(bb), np.array(oo, dtype=np.uint64), bb[-1] + 1)
            passing.append(bb)
        except AssertionError:
            pass
    assert passing == [[0, 0, 1, 2]]


@pytest.mark.parametrize("cap", [0, 1, 100, 4096, 10 ** 9])
def test_bucket_plan_invariants_random(cap):
    rng = np.random.default_rng(cap)
    numels = rng.integers(0, 3000, size=57).tolist()
    b, off, nb = oracle.bucket_plan(numels, 4, cap)
    _check_plan(numels, 4, cap, b, off, nb)


def test_bucket_sync_equal_ranks_average_to_themselves():
    # every rank holds the same bf16 gradients: the fp32 sum of 8 copies is
    # exact, so AVG returns each gradient unchanged; a misplaced offset or a
    # wrong division would not
    n = 8
    numels = [5, 300, 64, 1, 1000, 77]
    g = synth.rank_grads(14, 0, numels)
    grads = [[t.copy() for t in g] for _ in range(n)]
    oracle.bucket_sync(grads, cap_bytes=700, op="avg")
    for r in range(n):
        for t in range(len(numels)):
            assert np.array_equal(grads[r][t], g[t])


def test_bucket_sync_sum_of_small_integers_is_exact():
    n = 4
    numels = [10, 33, 7, 120]
    rng = np.random.default_rng(15)
    raw = [[rng.integers(-8, 8, size=m) for m in numels] for _ in range(n)]
    grads = [[synth.cast(v, "bf16") for v in rr] for rr in raw]
    oracle.bucket_sync(grads, cap_bytes=64, op="sum")
    for t in range(len(numels)):
        want = sum(raw[r][t] for r in range(n)).astype(np.float32)
        for r in range(n):
            assert np.array_equal(oracle.bf16_to_f32(grads[r][t]), want)


# ---------------------------------------------------------- a2a, rs, ag --

@pytest.mark.parametrize("n", [1, 2, 3, 4, 8])
def test_all_to_all_is_a_transpose_and_an_involution(n):
    per = 5
    x = synth.ranks(16, n, n * per, "int", "i32")
    y = oracle.all_to_all(x)
    blocks = np.stack([v.reshape(n, per) for v in x])  # [rank, block, elem]
    assert np.array_equal(np.stack([v.reshape(n, per) for v in y]), blocks.transpose(1, 0, 2))
    z = oracle.all_to_all(y)
    for r in range(n):
        assert np.array_equal(z[r], x[r])


@pytest.mark.parametrize("n", [1, 2, 3, 5, 8, 16])
@pytest.mark.parametrize("op", ["sum", "avg", "max", "min", "prod"])
def test_rs_then_ag_equals_ar_bitwise(n, op):
    count = n * 33
    dist = "prod" if op == "prod" else "uniform"
    x = synth.ranks(17, n, count, dist)
    ag = oracle.all_gather(oracle.reduce_scatter(x, op))
    oracle.ring_allreduce(x, op)
    for r in range(n):
        assert np.array_equal(ag[r].view(np.uint32), x[r].view(np.uint32))


# --------------------------------------------------------------- mutants --

def _pins():
    """A few pins as callables, for the mutant check."""
    return [
        lambda: test_worked_example_allreduce("ring", "f32"),
        lambda: test_worked_example_allreduce("fold", "f32"),
        test_worked_example_rs_ag_a2a,
        test_worked_example_avg_is_sum_over_n,
        test_ring_bytes_golden,
        test_p3_four_gpu_walkthrough,
        test_fold_order_golden,
        test_max_signed_zero_tie_keeps_left_operand,
        lambda: _omp_matches(5, "f32", (1, 3)),
        lambda: _samples_match(5, "f32"),
    ]


@pytest.mark.parametrize("kind", list(range(1, 10)) + [14, 15])
def test_mutants_are_caught(kind):
    # kinds (rr_oracle.c): 1 subtract instead of add, 2 AVG multiplies, 3
    # all-gather index off by one, 4 operands of the fold swapped, 5 last step
    # of each phase dropped, 6 one-shot fold starts one rank late, 7
    # reduce-scatter fold starts one rank late, 8 all-gather takes the wrong
    # rank's part, 9 all-to-all sends the wrong block, 14 the OpenMP ring
    # reads its own message slot instead of its left neighbour's, 15 the
    # sampled fold leaves out AVG's division
    failed = 0
    with oracle.mutant(kind):
        for pin in _pins():
            try:
                pin()
            except AssertionError:
                failed += 1
    assert failed > 0, f"mutant {kind} passed every pin"
    for pin in _pins():  # and the real oracle passes them all
        pin()


# ------------------------------------------------------------ double ring --

def _double_fixture():
    n = 4
    big = np.float32(2.0 ** 24)
    pattern = [np.float32(1), big, np.float32(1), -big]
    x = [np.zeros(8, dtype=np.float32) for _ in range(n)]
    for i in range(n):
        for k, v in enumerate(pattern):
            x[(i + k) % n][i] = v          # half A: upwards from rank i
            x[(i - k) % n][4 + i] = v      # half B: downwards from rank i
    return x


def test_double_ring_fold_order_golden():
    g = {ln.split(":")[0]: _vals(ln) for ln in golden_lines("double_ring_fold_order.txt")}
    for f in (oracle.double_ring_allreduce, oracle.fold_double_ring):
        x = _double_fixture()
        f(x, "sum")
        for r in range(4):
            assert x[r].tolist() == g["double_ring"]
    # half B folded upwards from its own chunk index instead
    x = _double_fixture()
    vals = np.stack([v[4:] for v in x])
    assert oracle.fold_samples(vals, np.arange(4)).tolist() == g["half_b_folded_upwards"][4:]


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("op", ["sum", "max", "min", "prod"])
def test_double_ring_brute_force_integer_data(n, op):
    for count in [0, 1, 2 * n - 1, 4 * n + 3]:
        lo, hi = (-3, 4) if op == "prod" else (-100, 100)
        rng = np.random.default_rng([n, count, 7])
        x = [synth.cast(rng.integers(lo, hi, size=count), "f32") for _ in range(n)]
        want = _np_reduce(x, op)
        oracle.double_ring_allreduce(x, op)
        for r in range(n):
            assert np.array_equal(x[r], want)


@pytest.mark.parametrize("n", [2, 3, 4, 8, 16])
def test_double_ring_bytes(n):
    # each step sends one chunk of each half to each neighbour: in all
    # 2(N-1) S, and 2(N-1)/N S per rank when 2N divides the count
    for per in (1, 5):
        count = 2 * n * per
        sent = oracle.double_ring_allreduce(synth.ranks(3, n, count, "uniform"))
        assert sent.tolist() == [2 * (n - 1) * count * 4 // n] * n
    sent = oracle.double_ring_allreduce(synth.ranks(3, n, 2 * n + 3, "uniform"))
    assert int(sent.sum()) == 2 * (n - 1) * (2 * n + 3) * 4


def test_double_ring_mutant_is_caught():
    with oracle.mutant(10):
        with pytest.raises(AssertionError):
            test_double_ring_brute_force_integer_data(4, "sum")


# ------------------------------------------------------------- bf16 wire --

def _wire_fixture():
    g = {ln.split(":")[0]: _vals(ln) for ln in golden_lines("bf16_wire.txt")}
    x = [np.array(g["inputs_rank0"], dtype=np.float32), np.array(g["inputs_rank1"], dtype=np.float32)]
    return g, x


def test_bf16_wire_golden():
    g, x = _wire_fixture()
    assert x[0][0] == 1 + 2.0 ** -10 and x[1][1] == 1 + 3 * 2.0 ** -9  # the fixture's values are exact
    for f in (oracle.ring_allreduce_wire, oracle.fold_wire):
        _, y = _wire_fixture()
        f(y, "sum")
        for r in range(2):
            assert y[r].tolist() == g["bf16_wire"]
    _, y = _wire_fixture()
    oracle.ring_allreduce(y, "sum")  # the exact fp32 ring for contrast
    assert y[0].tolist() == g["fp32_wire"]


@pytest.mark.parametrize("n", [2, 3, 4, 8])
def test_bf16_wire_is_lossless_on_small_integers(n):
    # every partial is an integer below 256 in magnitude: exactly
    # representable in bf16, so the wire changes nothing
    rng = np.random.default_rng([n, 11])
    x = [synth.cast(rng.integers(-20, 20, size=5 * n + 3), "f32") for _ in range(n)]
    y = [a.copy() for a in x]
    oracle.ring_allreduce_wire(x, "sum")
    oracle.ring_allreduce(y, "sum")
    for r in range(n):
        assert np.array_equal(x[r], y[r])


@pytest.mark.parametrize("n", [2, 4, 8, 16])
@pytest.mark.parametrize("op", ["sum", "avg"])
def test_bf16_wire_error_bound(n, op):
    # N-1 partials and the result are each rounded once to bf16 (relative
    # error <= 2^-8 each), every value bounded by sum |x|: the wire's error
    # against the fp64 reduction is at most about N * 2^-8 * sum |x|
    x = synth.ranks(12, n, 4000, "uniform")
    a = np.stack(x).astype(np.float64)
    exact, mag = a.sum(0), np.abs(a).sum(0)
    if op == "avg":
        exact, mag = exact / n, mag / n
    oracle.ring_allreduce_wire(x, op)
    err = np.abs(x[0].astype(np.float64) - exact)
    assert np.all(err <= n * 2.0 ** -8 * mag * (1 + 1e-3) + 1e-30)
    assert err.max() > 0  # and it is lossy on random data


def test_bf16_wire_mutant_is_caught():
    with oracle.mutant(11):
        with pytest.raises(AssertionError):
            test_bf16_wire_golden()


# ------------------------------------------------------------------ fp16 --
# The oracle converts fp16 with its own code from the IEEE 754 binary16
# definition; numpy's float16 conversion is an independent implementation of
# the same rounding, so it pins it on the cases that decide it.

def _f16_rounding_cases():
    rng = np.random.default_rng(41)
    finite = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    mid = ((finite[:-1] + finite[1:]) / 2).astype(np.float32)  # every tie, exact in fp32
    mid = np.concatenate([mid, [np.float32(65520.0)]])         # the tie above the largest finite
    x = np.concatenate([
        mid, np.nextafter(mid, np.float32(np.inf)), np.nextafter(mid, np.float32(0)),
        rng.standard_normal(200000).astype(np.float32) * np.float32(300),
        (rng.standard_normal(50000) * 1e-6).astype(np.float32),
        np.array([0.0, 65504, 65519.996, 65536, 1e30, 3.4e38, 2.0 ** -24, 2.0 ** -25, 2.0 ** -26, 1e-40,
                  np.inf], dtype=np.float32)])
    return np.concatenate([x, -x])


def test_f16_widening_matches_numpy_exhaustively():
    h = np.arange(65536, dtype=np.uint16).view(np.float16)
    got, want = oracle.f16_to_f32(h), h.astype(np.float32)
    nan = np.isnan(want)
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))
    assert np.isnan(got[nan]).all()


def test_f16_rounding_matches_numpy():
    x = _f16_rounding_cases()
    with np.errstate(over="ignore"):
        want = x.astype(np.float16)
    assert np.array_equal(oracle.f32_to_f16(x).view(np.uint16), want.view(np.uint16))
    nan = oracle.f32_to_f16(np.array([np.nan, -np.nan], np.float32))
    assert np.isnan(nan.astype(np.float32)).all()


def test_f16_rounding_hand_cases():
    # 1 + 2^-11 lies halfway between 1 and 1 + 2^-10: ties to even -> 1
    # 1 + 3 * 2^-11 lies halfway between 1 + 2^-10 and 1 + 2^-9: even -> 1 + 2^-9
    # 65520 lies halfway between 65504 (odd significand) and 2^16: -> infinity
    # 2^-25 lies halfway between 0 and 2^-24 (odd): -> 0; 3 * 2^-25 -> 2^-23
    x = np.array([1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 65519.0, 65520.0, 2.0 ** -25, 3 * 2.0 ** -25],
                 dtype=np.float32)
    got = oracle.f16_to_f32(oracle.f32_to_f16(x)).tolist()
    assert got == [1.0, 1 + 2.0 ** -9, 65504.0, float("inf"), 0.0, 2.0 ** -23]


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("op", ["sum", "max", "min", "prod"])
def test_f16_brute_force_integer_data(n, op):
    # integers whose every partial fold is below 2^11 are exact in fp16, so
    # every path equals numpy's float64 reduction
    lo, hi = {"sum": (-100, 100), "prod": (-2, 3)}.get(op, (-1000, 1000))
    for count in [0, 1, 2 * n + 3, 37]:
        rng = np.random.default_rng([n, count, 16])
        raw = [rng.integers(lo, hi, size=count) for _ in range(n)]
        x0 = [synth.cast(v, "f16") for v in raw]
        want = _np_reduce(x0, op)
        for path in (oracle.ring_allreduce, oracle.fold_ring_order, oracle.naive_allreduce,
                     oracle.tree_schedule, oracle.tree_fold, oracle.double_ring_allreduce):
            x = [v.copy() for v in x0]
            path(x, op)
            for r in range(n):
                assert np.array_equal(x[r].astype(np.float64), want), (path.__name__, r)


@pytest.mark.parametrize("n", [2, 4, 8, 16])
def test_f16_one_shot_rounds_once_and_ring_stays_within_bound(n):
    # one-shot: the fp32 ring-order fold of the widened values, rounded once
    # (numpy's rounding of the oracle's own fp32 fold); ring schedule: per-hop
    # rounding, within gamma_{N-1} * sum|x| of the fp64 sum, u = 2^-11
    x = synth.ranks(42, n, 5000, "uniform", "f16")
    wide = [v.astype(np.float32) for v in x]
    oracle.fold_ring_order(wide, "sum")
    one = [v.copy() for v in x]
    oracle.fold_ring_order(one, "sum")
    assert np.array_equal(one[0].view(np.uint16), wide[0].astype(np.float16).view(np.uint16))
    ring = [v.copy() for v in x]
    oracle.ring_allreduce(ring, "sum")
    exact = np.sum([v.astype(np.float64) for v in x], axis=0)
    u = 2.0 ** -11
    gamma = (n - 1) * u / (1 - (n - 1) * u)
    bound = gamma * np.sum([np.abs(v.astype(np.float64)) for v in x], axis=0) + u * np.abs(exact)
    assert (np.abs(ring[0].astype(np.float64) - exact) <= bound).all()


def test_f16_bucket_sync_of_small_integers_is_exact():
    n = 4
    numels = [10, 33, 7, 120]
    rng = np.random.default_rng(43)
    raw = [[rng.integers(-8, 8, size=m) for m in numels] for _ in range(n)]
    grads = [[synth.cast(v, "f16") for v in rr] for rr in raw]
    oracle.bucket_sync(grads, cap_bytes=64, op="sum")
    for t in range(len(numels)):
        want = sum(raw[r][t] for r in range(n)).astype(np.float16)
        for r in range(n):
            assert np.array_equal(grads[r][t], want)


def test_f16_rounding_mutant_is_caught():
    # kind 12: ties round away from zero instead of to even
    with oracle.mutant(12):
        with pytest.raises(AssertionError):
            test_f16_rounding_matches_numpy()
        with pytest.raises(AssertionError):
            test_f16_rounding_hand_cases()
    test_f16_rounding_matches_numpy()
