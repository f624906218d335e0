"""The five workloads at full size on the GPU, through the C ABI, against the
CPU oracle.

Where the oracle finishes the whole workload in seconds it checks every
element; otherwise it checks sampled elements one by one (every chunk
boundary plus random positions), and the GPU side is also checked for
properties that hold at any size (all ranks identical).  The calls use the
same API and launch configuration as ``bench.py``.
"""
import multiprocessing as mproc

import numpy as np
import pytest
import torch

import oracle
import ring_all_reduce_virtual_b200 as rrv
from gpu_util import assert_bits_equal, to_dev, to_host
from ring_all_reduce_virtual_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from ring_all_reduce_virtual_b200.build import build

    build()


def _sample_idx(count, n, k, seed):
    C = -(-count // n)
    rng = np.random.default_rng(seed)
    b = []
    for c in range(n + 1):
        b += [c * C - 2, c * C - 1, c * C, c * C + 1]
    idx = np.concatenate([np.array(b, dtype=np.int64), rng.integers(0, count, size=k), [0, count - 1]])
    return np.unique(idx[(idx >= 0) & (idx < count)])


def _gather(tensors, idx):
    it = torch.from_numpy(idx).to(tensors[0].device)
    return to_host([t.index_select(0, it) for t in tensors])


def _all_ranks_equal(tensors):
    """Every rank holds the same bits (a property at any size)."""
    ref = tensors[0].view(torch.int32)
    for t in tensors[1:]:
        assert torch.equal(t.view(torch.int32), ref)


def _check_sampled_fold(host, dev, op, seed=0, k=200000):
    n, count = len(host), host[0].size
    idx = _sample_idx(count, n, k, seed)
    C = -(-count // n)
    vals = np.stack([a[idx] for a in host])
    want = oracle.fold_samples(vals, (idx // C).astype(np.int32), op)
    got = _gather(dev, idx)
    for r in range(n):
        assert_bits_equal([got[r]], [want], f"sampled rank {r}")


# ------------------------------------------------------------ workload 1 --

def test_small_ring_4x4096():
    """4 ranks x 4096 fp32, uniform[-1, 1), SUM, ring: every element and the
    bytes each rank sent (2(N-1)/N x 16 KiB = 24 KiB)."""
    x = synth.ranks(0, 4, 4096, "uniform")
    want = [a.copy() for a in x]
    sent = oracle.ring_allreduce(want, "sum")
    d = to_dev(x)
    rrv.all_reduce(d, "sum", "ring")
    assert_bits_equal(to_host(d), want)
    st = rrv.last_stats()
    assert st["bytes_sent_max"] == int(sent.max()) == 24576 and st["steps"] == 6


# ------------------------------------------------------------ workload 2 --

@pytest.fixture(scope="module")
def inputs_8x256m():
    return synth.ranks(0, 8, 1 << 26, "normal")


@pytest.mark.parametrize("op,algo", [("avg", "auto"), ("sum", "oneshot"), ("sum", "ring"), ("avg", "ring")])
def test_8x256MiB_every_element(inputs_8x256m, op, algo):
    """8 ranks x 64 Mi fp32 (256 MiB each), normal(0, 1e-3), in place: every
    element of every rank equals the oracle (ring steps for RING, the
    ring-order definition otherwise)."""
    x = inputs_8x256m
    d = to_dev(x)
    rrv.all_reduce(d, op, algo)
    want = [a.copy() for a in x]
    (oracle.ring_allreduce if algo == "ring" else oracle.fold_ring_order)(want, op)
    assert_bits_equal(to_host(d), want, f"{op} {algo}")


# ------------------------------------------------------------ workload 3 --

def _grads_worker(args):
    seed, rank, numels = args
    return synth.rank_grads(seed, rank, numels, "normal", "bf16")


@pytest.fixture(scope="module")
def gpt_grads():
    tensors = synth.grad_ready_order(synth.gpt_grad_tensors())
    numels = [m for _, m in tensors]
    ctx = mproc.get_context("spawn")
    with ctx.Pool(8) as pool:
        host = pool.map(_grads_worker, [(0, r, numels) for r in range(8)])
    return numels, host


def _bucket_expect(host, numels, plan, b, pos, n):
    """Oracle values of sampled flat positions of bucket b: ring-order fp32
    fold of the widened gradients, AVG's division, one rounding to bf16."""
    first, cnt, numel = plan.info(b)
    starts = np.cumsum([0] + [numels[t] for t in range(first, first + cnt)])
    tens = np.searchsorted(starts, pos, side="right") - 1
    bits = np.array([[host[r][first + t][p - starts[t]] for t, p in zip(tens, pos)] for r in range(n)],
                    dtype=np.uint16)
    vals = oracle.bf16_to_f32(bits)
    C = -(-numel // n)
    f = oracle.fold_samples(vals, (pos // C).astype(np.int32), "avg")
    return oracle.f32_to_bf16(f), tens, starts


@pytest.mark.parametrize("path", ["fused", "fused_range", "staged"])
def test_gpt_like_bucketed_sync(gpt_grads, path):
    """293 bf16 gradient tensors (1.34 B parameters per rank), 8 ranks, 25 MiB
    buckets in gradient-ready order, AVG with fp32 accumulation: sampled
    positions of every bucket against the oracle, all ranks identical, and
    the bf16 result within abs/rel 1e-2 of the fp64 mean."""
    numels, host = gpt_grads
    n = 8
    plan = rrv.BucketPlan(numels, "bf16", synth.BUCKET_CAP_BYTES)
    grads = [to_dev(rank) for rank in host]
    if path == "fused":
        for b in range(plan.num_buckets):
            plan.all_reduce(b, grads, "avg")
    elif path == "fused_range":
        plan.all_reduce_range(0, plan.num_buckets, grads, "avg")
        assert rrv.last_stats()["launches"] < plan.num_buckets
    else:
        biggest = max(plan.info(b)[2] for b in range(plan.num_buckets))
        buckets = [torch.empty(biggest, dtype=torch.float32, device="cuda") for _ in range(n)]
        for b in range(plan.num_buckets):
            numel = plan.info(b)[2]
            plan.pack(b, grads, buckets)
            rrv.all_reduce([t[:numel] for t in buckets], "sum", "auto")
            plan.unpack(b, buckets, grads, "avg")
    torch.cuda.synchronize()
    rng = np.random.default_rng(1)
    for b in range(plan.num_buckets):
        first, cnt, numel = plan.info(b)
        C = -(-numel // n)
        pos = np.unique(np.concatenate([rng.integers(0, numel, size=64),
                                        np.clip(np.arange(n) * C, 0, numel - 1), [numel - 1]]))
        want, tens, starts = _bucket_expect(host, numels, plan, b, pos, n)
        for r in (0, 3, 7):
            got = np.array([grads[r][first + t][p - starts[t]].view(torch.int16).item() for t, p in
                            zip(tens, pos)], dtype=np.int64).astype(np.uint16)
            assert np.array_equal(got, want), f"bucket {b} rank {r}"
        for t in range(first, first + cnt):
            for r in range(1, n):
                assert torch.equal(grads[r][t].view(torch.int16), grads[0][t].view(torch.int16))
    # tolerance of the bf16 result against the fp64 mean, on one large tensor
    t = max(range(len(numels)), key=lambda i: numels[i])
    mean = np.mean([oracle.bf16_to_f32(host[r][t][:100000]).astype(np.float64) for r in range(n)], axis=0)
    got = oracle.bf16_to_f32(to_host([grads[0][t][:100000]])[0])
    assert np.allclose(got, mean, atol=1e-2, rtol=1e-2)


# ------------------------------------------------------------ workload 4 --

SWEEP_ALGOS = ("ring", "oneshot", "two_shot", "tree", "tree_oneshot", "double_ring")
SWEEP_ORACLE = {  # fp32: the stepping schedules give their definitions' bits (pinned on the CPU)
    "ring": oracle.fold_ring_order, "oneshot": oracle.fold_ring_order, "two_shot": oracle.fold_ring_order,
    "tree": oracle.tree_schedule, "tree_oneshot": oracle.tree_fold, "double_ring": oracle.fold_double_ring,
}


def _check_sampled_tree(host, dev, seed):
    """The tree order is element-wise: the oracle's tree fold of the sampled
    [N, m] rows is the result at those elements."""
    n, count = len(host), host[0].size
    idx = _sample_idx(count, n, 20000, seed)
    rows = [np.ascontiguousarray(a[idx]) for a in host]
    oracle.tree_fold(rows, "sum")
    got = _gather(dev, idx)
    for r in range(n):
        assert_bits_equal([got[r]], [rows[0]], f"sampled tree rank {r}")


def _check_sampled_double_ring(host, dev, seed):
    """The double ring (reading 13): element i < H = ceil(count/2) is chunk
    i // ceil(H/N) of the clockwise ring, folded upwards from that rank;
    element i >= H is chunk c = (i - H) // ceil((count - H)/N) of the mirror
    ring, folded downwards c, c-1, ..., c+1 -- the upward fold of the
    rank-reversed rows from N-1-c.  Both through the oracle's sampled fold."""
    n, count = len(host), host[0].size
    H = (count + 1) // 2
    CA, CB = -(-H // n), -(-(count - H) // n)
    idx = _sample_idx(count, n, 20000, seed)
    idx = np.unique(np.concatenate([idx, [H - 1, H, H + 1]]))
    idx = idx[(idx >= 0) & (idx < count)]
    a, b = idx[idx < H], idx[idx >= H]
    want = np.empty(idx.size, dtype=np.float32)
    want[idx < H] = oracle.fold_samples(np.stack([x[a] for x in host]), (a // CA).astype(np.int32), "sum")
    rev = np.stack([x[b] for x in host][::-1])
    want[idx >= H] = oracle.fold_samples(rev, (n - 1 - (b - H) // CB).astype(np.int32), "sum")
    got = _gather(dev, idx)
    for r in range(n):
        assert_bits_equal([got[r]], [want], f"sampled double ring rank {r}")


@pytest.mark.parametrize("n", [2, 4, 8, 16])
@pytest.mark.parametrize("nbytes", [1 << 10, 1 << 20, 1 << 26, 1 << 30])
def test_size_sweep_points(n, nbytes):
    """Sweep points (1 KiB .. 1 GiB per rank, fp32 SUM) for every schedule:
    ring, one-shot and two-shot (ring order), the tree schedule and the
    tree-order one-shot, and the double ring, against the oracle -- every
    element up to 64 MiB, sampled elements (chunk boundaries included) at
    1 GiB -- with all ranks identical, and the ring-order ones equal to each
    other bit for bit."""
    count = nbytes // 4
    # normal(0, 1e-3): full mantissas, so every fold order gives its own bits
    # (uniform[-1, 1) draws are multiples of 2^-23, whose short sums are exact)
    x = synth.ranks(4, n, count, "normal")
    pristine = to_dev(x)
    ring_sample = None
    for algo in SWEEP_ALGOS:
        d = [t.clone() for t in pristine]
        rrv.all_reduce(d, "sum", algo)
        if nbytes <= 1 << 26:
            want = [a.copy() for a in x]
            SWEEP_ORACLE[algo](want, "sum")
            assert_bits_equal(to_host(d), want, algo)
        elif algo in ("ring", "oneshot", "two_shot"):
            _check_sampled_fold(x, d, "sum", seed=n, k=20000)
        elif algo in ("tree", "tree_oneshot"):
            _check_sampled_tree(x, d, seed=n + 1)
        else:
            _check_sampled_double_ring(x, d, seed=n + 2)
        _all_ranks_equal(d)
        if algo in ("ring", "oneshot", "two_shot"):  # one ring order: the same bits
            first = d[0][: min(count, 1 << 22)].clone()
            if ring_sample is None:
                ring_sample = first
            else:
                assert torch.equal(first.view(torch.int32), ring_sample.view(torch.int32)), algo
        del d
    del pristine
    torch.cuda.empty_cache()


# ------------------------------------------------------------ workload 5 --

@pytest.fixture(scope="module")
def inputs_64x256m():
    return synth.ranks(0, 64, 1 << 26, "uniform")


@pytest.mark.parametrize("op", ["sum", "max", "min", "prod"])
def test_64x256MiB_allreduce(inputs_64x256m, op):
    """64 ranks x 64 Mi fp32 (16 GiB): SUM/MAX/MIN on uniform[-1, 1), PROD on
    uniform[0.99, 1.01); sampled elements against the oracle, all ranks
    identical."""
    x = synth.ranks(1, 64, 1 << 26, "prod") if op == "prod" else inputs_64x256m
    d = to_dev(x)
    rrv.all_reduce(d, op, "auto")
    torch.cuda.synchronize()
    _check_sampled_fold(x, d, op, seed=5, k=50000)
    _all_ranks_equal(d)
    del d
    torch.cuda.empty_cache()


def test_64x256MiB_rs_ag_a2a(inputs_64x256m):
    """Reduce-scatter, all-gather and all-to-all at 64 ranks x 64 Mi fp32,
    sampled against the oracle's definitions."""
    x = inputs_64x256m
    n, count = 64, 1 << 26
    per = count // n
    d = to_dev(x)
    rs = [torch.empty(per, dtype=torch.float32, device="cuda") for _ in range(n)]
    rrv.reduce_scatter(d, rs, "sum")
    rng = np.random.default_rng(9)
    j = np.unique(np.concatenate([rng.integers(0, per, 4000), [0, per - 1]]))
    rs_h = to_host(rs)
    for r in (0, 17, 63):  # part r = the ring-order fold of chunk r, starting on rank r
        vals = np.stack([a[r * per + j] for a in x])
        want = oracle.fold_samples(vals, np.full(j.size, r, np.int32), "sum")
        assert np.array_equal(rs_h[r][j].view(np.uint32), want.view(np.uint32))
    ag = [torch.empty(count, dtype=torch.float32, device="cuda") for _ in range(n)]
    rrv.all_gather(rs, ag)
    for r in (0, 40):
        got = to_host([ag[r]])[0]
        assert np.array_equal(got.view(np.uint32), np.concatenate(rs_h).view(np.uint32))
    del ag
    a2a = [torch.empty(count, dtype=torch.float32, device="cuda") for _ in range(n)]
    rrv.all_to_all(d, a2a)
    for r in (0, 5, 63):
        got = to_host([a2a[r]])[0]
        for p in (0, 31, 63):
            assert np.array_equal(got[p * per:(p + 1) * per], x[p][r * per:(r + 1) * per])
    del a2a, d, rs
    torch.cuda.empty_cache()
