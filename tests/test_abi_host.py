"""Host-side checks of the C ABI that need no GPU.

The library must load and export every function ``include/rr.h`` declares.
Its host logic (ring schedule, bucket plan, cost model, picker, argument
checks) is compared with the oracle and the pages' figures.  No call here
launches a kernel: every call either computes on the host only or fails
argument checks before anything is enqueued.
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
import ring_all_reduce_virtual_b200 as rrv
from conftest import ROOT, golden_lines, picker_table
from ring_all_reduce_virtual_b200 import _lib, synth
from ring_all_reduce_virtual_b200.build import build


@pytest.fixture(scope="module", autouse=True)
def _built():
    build()


def _declared():
    src = open(os.path.join(ROOT, "include", "rr.h"), encoding="utf-8").read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rr_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("rr_allreduce", "rr_reduce_scatter", "rr_all_gather", "rr_all_to_all", "rr_bucket_plan",
              "rr_bucket_pack", "rr_bucket_unpack", "rr_bucket_plan_free", "rr_get_stats",
              "rr_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = _lib.lib()
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (rr_\w+)", out))
    for name in _declared():
        assert name in exported, name
        assert hasattr(lib, name)


def test_version_and_status_strings():
    lib = _lib.lib()
    assert lib.rr_version() == 1
    assert lib.rr_status_string(0) == b"ok"
    assert lib.rr_status_string(1) == b"invalid argument"


# ------------------------------------------------------- ring schedule --

@pytest.mark.parametrize("n,count", [(1, 7), (2, 2), (4, 4096), (4, 1024), (3, 10), (8, 3), (16, 1000), (64, 130)])
def test_ring_schedule_equals_oracle_trace(n, count):
    x = synth.ranks(0, n, count, "uniform")
    sent, trace = oracle.ring_allreduce(x, trace=True)
    ours = rrv.ring_schedule(n, count, "f32")
    assert ours == trace
    per_rank = np.zeros(n, dtype=np.uint64)
    for e in ours:
        per_rank[e["rank"]] += e["bytes"]
    assert np.array_equal(per_rank, sent)


def test_ring_schedule_bytes_golden():
    g = dict(ln.split(":", 1) for ln in golden_lines("ring_bytes_4rank.txt"))
    n, m = int(g["ranks"]), int(g["elements_per_rank"])
    ev = rrv.ring_schedule(n, m, "f32")
    sent = [sum(e["bytes"] for e in ev if e["rank"] == r) for r in range(n)]
    assert sent == [int(v) for v in g["sent"].split()]


# --------------------------------------------------------- bucket plan --

@pytest.mark.parametrize("cap", [0, 1, 700, 25 * (1 << 20)])
def test_bucket_plan_equals_oracle(cap):
    if cap == 25 * (1 << 20):
        numels = [m for _, m in synth.grad_ready_order(synth.gpt_grad_tensors())]
    else:
        numels = np.random.default_rng(cap).integers(0, 400, size=50).tolist()
    b, off, nb = oracle.bucket_plan(numels, 2, cap)
    plan = rrv.BucketPlan(numels, "bf16", cap)
    assert plan.num_buckets == nb
    for t in range(len(numels)):
        assert plan.tensor(t) == (int(b[t]), int(off[t]))
    for k in range(nb):
        first, cnt, numel = plan.info(k)
        members = [t for t in range(len(numels)) if b[t] == k]
        assert (first, cnt) == (members[0], len(members))
        assert numel == sum(numels[t] for t in members)


# ---------------------------------------------------------- cost model --

def _parse_ab(line):
    name, rest = line.split(":", 1)
    lhs, rhs = rest.split("->")
    args = dict(kv.split("=") for kv in lhs.split())
    val, tol = rhs.split()
    return name, {k: float(v) for k, v in args.items()}, float(val), float(tol.split("=")[1])


def test_cost_model_matches_the_pages():
    for line in golden_lines("alpha_beta.txt"):
        name, a, want, rel = _parse_ab(line)
        n = int(a["N"])
        if name == "volume":
            got = rrv.cost_model("ring", n, a["M"], 0.0, 1.0)["bytes_sent"]
        elif name == "latency_term":
            got = rrv.cost_model("ring", n, 1.0, a["alpha"], 1.0)["latency_s"]
        elif name == "bandwidth_term":
            got = rrv.cost_model("ring", n, a["M"], 0.0, a["beta"])["bandwidth_s"]
        elif name == "ring_time":
            got = rrv.cost_model("ring", n, a["M"], a["alpha"], a["beta"])["total_s"]
        elif name == "ps_centre":
            # the parameter server's centre receives and sends (N-1) M each
            got = 2 * (n - 1) * a["M"]
        elif name == "ps_time":
            got = 2 * (n - 1) * a["M"] / a["beta"]
        else:
            raise AssertionError(name)
        assert abs(got - want) <= rel * want, (line, got)


def test_cost_model_tree_and_oneshot_steps():
    # [P3] section 6 table: the tree takes 2 log2 N steps, the ring 2(N-1)
    for n in (2, 4, 8, 16, 64):
        assert rrv.cost_model("tree", n, 1.0, 1.0, 1.0)["steps"] == 2 * np.log2(n)
        assert rrv.cost_model("ring", n, 1.0, 1.0, 1.0)["steps"] == 2 * (n - 1)
        assert rrv.cost_model("oneshot", n, 1.0, 1.0, 1.0)["steps"] == 1
        # two-shot: the ring's per-rank volume in two steps
        two = rrv.cost_model("two_shot", n, 1.0, 1.0, 1.0)
        assert two["steps"] == 2 and two["bytes_sent"] == rrv.cost_model("ring", n, 1.0, 1.0, 1.0)["bytes_sent"]
        # [P3] section 6: the double ring halves the bytes on each link
        dbl = rrv.cost_model("double_ring", n, 1.0, 1.0, 1.0)
        assert dbl["steps"] == 2 * (n - 1)
        assert dbl["bytes_sent"] == rrv.cost_model("ring", n, 1.0, 1.0, 1.0)["bytes_sent"] / 2


def test_picker_table_is_what_the_committed_sweep_record_gives():
    # the header is generated, never edited: regenerating it from the record
    # it names gives the same text
    from ring_all_reduce_virtual_b200.picker import gen_table

    text, rows, src = picker_table()
    assert rows and os.path.exists(os.path.join(ROOT, src)), src
    points, fit = gen_table.load(os.path.join(ROOT, src))
    assert gen_table.render(gen_table.table(points), fit, src) == text


def test_picker_follows_the_measured_table():
    _, rows, _ = picker_table()
    aligned = [r for r in rows if r[2] == 0]
    for n, lb, _, algo, _ in aligned:
        assert rrv.pick_algo(n, (1 << lb) // 4, "f32") == algo, (n, lb)
        # 16-bit gradients never take the ring, whose partials round at every hop
        assert rrv.pick_algo(n, (1 << lb) // 2, "bf16") == ("oneshot" if algo == "ring" else algo), (n, lb)
    # where the winner changes between adjacent measured sizes, each side keeps its own
    by_n = {}
    for n, lb, _, algo, _ in aligned:
        by_n.setdefault(n, {})[lb] = algo
    for n, sizes in by_n.items():
        lbs = sorted(sizes)
        for a, b in zip(lbs, lbs[1:]):
            if sizes[a] != sizes[b]:
                assert rrv.pick_algo(n, (1 << a) // 4, "f32") == sizes[a]
                assert rrv.pick_algo(n, (1 << b) // 4, "f32") == sizes[b]
    # an unmeasured rank count takes the nearest measured one (log2 ratio)
    ns = sorted(by_n)
    for n in range(2, 65):
        if n in by_n:
            continue
        near = min(ns, key=lambda m: (abs(np.log2(m / n)), m))
        lb = 20
        want = by_n[near][min(by_n[near], key=lambda x: (abs(x - lb), x))]
        assert rrv.pick_algo(n, (1 << lb) // 4, "f32") == want, n


def test_picker_params_switch_to_the_model_and_back():
    _, rows, _ = picker_table()
    try:
        # the alpha-beta model of one GPU: the one-shot has both the fewest
        # launches and the fewest HBM bytes, so it wins at every size
        rrv.set_picker_params(4e-6, 6.5e12)
        for n in (2, 3, 8, 64):
            for e in (10, 20, 30):
                assert rrv.pick_algo(n, (1 << e) // 4, "f32") == "oneshot"
    finally:
        rrv.set_picker_params(0.0, 0.0)  # back to the measured table
    n, lb, _, algo, _ = next(r for r in rows if r[2] == 0)
    assert rrv.pick_algo(n, (1 << lb) // 4, "f32") == algo
    with pytest.raises(rrv.RRError):
        rrv.set_picker_params(-1.0, 1e12)


# -------------------------------------------------- argument checking --

def _fake(n, stride=1 << 20, base=1 << 40):
    arr = (ctypes.c_void_p * n)()
    for i in range(n):
        arr[i] = base + i * stride
    return arr


def test_argument_errors_return_before_any_launch():
    lib = _lib.lib()
    s = ctypes.c_void_p(0)
    assert lib.rr_allreduce(_fake(4), 0, 16, 0, 0, 0, s) == _lib.RR_ERR_INVALID_ARG
    assert lib.rr_allreduce(_fake(4), 65, 16, 0, 0, 0, s) == _lib.RR_ERR_INVALID_ARG
    assert lib.rr_allreduce(_fake(4), 4, 16, 7, 0, 0, s) == _lib.RR_ERR_INVALID_ARG
    assert lib.rr_allreduce(_fake(4), 4, 16, 0, 9, 0, s) == _lib.RR_ERR_INVALID_ARG
    assert lib.rr_allreduce(_fake(4), 4, 16, 0, 0, 9, s) == _lib.RR_ERR_INVALID_ARG
    assert lib.rr_allreduce(_fake(4), 4, 16, 0, 0, 7, s) == _lib.RR_ERR_INVALID_ARG
    assert lib.rr_allreduce(_fake(4), 4, 16, 2, 1, 0, s) == _lib.RR_ERR_UNSUPPORTED  # int32 AVG
    assert lib.rr_allreduce(None, 4, 16, 0, 0, 0, s) == _lib.RR_ERR_INVALID_ARG
    overlapping = _fake(4, stride=32)  # 16 fp32 = 64 bytes apart by 32
    assert lib.rr_allreduce(overlapping, 4, 16, 0, 0, 0, s) == _lib.RR_ERR_INVALID_ARG
    assert b"overlap" in lib.rr_last_error()
    repeated = _fake(4, stride=0)
    assert lib.rr_allreduce(repeated, 4, 16, 0, 0, 0, s) == _lib.RR_ERR_INVALID_ARG
    nulls = (ctypes.c_void_p * 2)(None, None)
    assert lib.rr_allreduce(nulls, 2, 16, 0, 0, 0, s) == _lib.RR_ERR_INVALID_ARG
    # fp32 buffers 2 bytes off an element boundary: no element there can be read
    odd = _fake(4, base=(1 << 40) + 2)
    assert lib.rr_allreduce(odd, 4, 16, 0, 0, 0, s) == _lib.RR_ERR_INVALID_ARG
    assert b"element size" in lib.rr_last_error()
    assert lib.rr_ring_step(odd, 4, 16, 0, 0, 0, 0, s) == _lib.RR_ERR_INVALID_ARG
    assert lib.rr_all_to_all(odd, _fake(4, base=1 << 41), 4, 4, 0, s) == _lib.RR_ERR_INVALID_ARG
    # bad ring steps
    assert lib.rr_ring_step(_fake(4), 4, 16, 0, 0, 0, 3, s) == _lib.RR_ERR_INVALID_ARG
    assert lib.rr_ring_step(_fake(4), 4, 16, 0, 0, 2, 0, s) == _lib.RR_ERR_INVALID_ARG
    # reduce-scatter output overlapping an input
    send, recv = _fake(2), _fake(2, base=(1 << 40) + 8)
    assert lib.rr_reduce_scatter(send, recv, 2, 4, 0, 0, 0, s) == _lib.RR_ERR_INVALID_ARG
    assert lib.rr_reduce_scatter(_fake(2), _fake(2, base=1 << 41), 2, 4, 0, 0, 1, s) == _lib.RR_ERR_UNSUPPORTED


def test_reducer_argument_errors():
    lib = _lib.lib()
    out = ctypes.c_void_p()
    assert lib.rr_reducer_create(None, _fake(2), 2, 1, None, 0, ctypes.byref(out)) == _lib.RR_ERR_INVALID_ARG
    plan = rrv.BucketPlan([10, 20], "bf16", 100)
    assert lib.rr_reducer_create(plan._h, _fake(4), 2, 2, None, 0, ctypes.byref(out)) == _lib.RR_ERR_UNSUPPORTED
    assert lib.rr_reducer_create(plan._h, _fake(4), 0, 1, None, 0, ctypes.byref(out)) == _lib.RR_ERR_INVALID_ARG
    # gradients are checked at creation: a repeated pointer is refused there
    assert lib.rr_reducer_create(plan._h, _fake(4, stride=0), 2, 1, None, 0, ctypes.byref(out)) == \
        _lib.RR_ERR_INVALID_ARG
    assert b"overlap" in lib.rr_last_error()
    assert lib.rr_reducer_ready(None, 0, None) == _lib.RR_ERR_INVALID_ARG
    assert lib.rr_reducer_finish(None, None) == _lib.RR_ERR_INVALID_ARG


def test_trivial_calls_enqueue_nothing():
    lib = _lib.lib()
    s = ctypes.c_void_p(0)
    assert lib.rr_allreduce(_fake(4), 4, 0, 0, 0, 0, s) == 0  # count == 0
    assert rrv.last_stats()["launches"] == 0
    assert lib.rr_allreduce(_fake(1), 1, 1000, 0, 1, 0, s) == 0  # one rank: identity
    assert rrv.last_stats()["launches"] == 0


def test_bucket_plan_rejects_bad_dtype():
    with pytest.raises(rrv.RRError):
        rrv.BucketPlan([1, 2, 3], "i32", 100)


def test_rank_set_checks_its_tensors_once():
    """RankSet applies the same checks as the list form, at construction."""
    import torch

    with pytest.raises(ValueError):
        rrv.RankSet([])
    with pytest.raises(ValueError):
        rrv.RankSet([torch.zeros(4), torch.zeros(4)])  # not CUDA tensors
    with pytest.raises(ValueError):
        rrv.RankSet([torch.zeros(4)] * (rrv.MAX_RANKS + 1))


def test_bucket_range_argument_errors():
    """rr_bucket_allreduce_range checks the range and the gradients before any
    launch; a single rank or empty buckets enqueue nothing."""
    lib = _lib.lib()
    s = ctypes.c_void_p(0)
    plan = rrv.BucketPlan([10, 20, 30, 40], "bf16", 60)  # buckets [10, 20] (60 B), [30], [40]
    assert plan.num_buckets == 3
    grads = _fake(8, stride=1 << 20)  # 2 ranks x 4 tensors, disjoint
    for first, count in ((-1, 1), (0, 0), (0, 4), (3, 1), (2, 2)):
        assert lib.rr_bucket_allreduce_range(plan._h, first, count, grads, 2, 1, s) == _lib.RR_ERR_INVALID_ARG
    assert lib.rr_bucket_allreduce_range(plan._h, 0, 3, grads, 2, 2, s) == _lib.RR_ERR_UNSUPPORTED  # MAX
    assert lib.rr_bucket_allreduce_range(None, 0, 1, grads, 2, 1, s) == _lib.RR_ERR_INVALID_ARG
    assert lib.rr_bucket_allreduce_range(plan._h, 0, 2, None, 2, 1, s) == _lib.RR_ERR_INVALID_ARG
    repeated = _fake(8, stride=0)
    assert lib.rr_bucket_allreduce_range(plan._h, 0, 3, repeated, 2, 1, s) == _lib.RR_ERR_INVALID_ARG
    assert lib.rr_bucket_allreduce_range(plan._h, 0, 3, grads, 1, 1, s) == 0  # one rank: identity
    assert rrv.last_stats()["launches"] == 0


def test_element_counts_above_2_pow_48_are_refused():
    """A count whose byte range could wrap is refused before any launch."""
    lib = _lib.lib()
    s = ctypes.c_void_p(0)
    huge = (1 << 48) + 1
    assert lib.rr_allreduce(_fake(4), 4, huge, 0, 0, 2, s) == _lib.RR_ERR_INVALID_ARG
    assert lib.rr_allreduce(_fake(4), 4, 1 << 62, 0, 0, 2, s) == _lib.RR_ERR_INVALID_ARG
    assert b"2^48" in lib.rr_last_error()
    assert lib.rr_reduce_scatter(_fake(2), _fake(2, base=1 << 41), 2, huge, 0, 0, 0, s) == _lib.RR_ERR_INVALID_ARG
    assert lib.rr_all_gather(_fake(2), _fake(2, base=1 << 41), 2, huge, 0, 0, s) == _lib.RR_ERR_INVALID_ARG
    assert lib.rr_all_to_all(_fake(2), _fake(2, base=1 << 41), 2, huge, 0, s) == _lib.RR_ERR_INVALID_ARG
    with pytest.raises(rrv.RRError):
        rrv.BucketPlan([10, huge], "bf16", 100)


def test_host_buffer_allreduce_checks_every_buffer():
    """rr_allreduce_host refuses overlapping device buffers, overlapping host
    buffers and a host buffer that overlaps a device one, before any copy."""
    lib = _lib.lib()
    s = ctypes.c_void_p(0)
    dev, host = _fake(2), _fake(2, base=1 << 42)
    assert lib.rr_allreduce_host(host, _fake(2, stride=0), 2, 16, 0, 0, 2, s) == _lib.RR_ERR_INVALID_ARG
    assert lib.rr_allreduce_host(_fake(2, base=1 << 42, stride=8), dev, 2, 16, 0, 0, 2, s) == \
        _lib.RR_ERR_INVALID_ARG
    assert lib.rr_allreduce_host(dev, dev, 2, 16, 0, 0, 2, s) == _lib.RR_ERR_INVALID_ARG
    nulls = (ctypes.c_void_p * 2)(None, None)
    assert lib.rr_allreduce_host(nulls, dev, 2, 16, 0, 0, 2, s) == _lib.RR_ERR_INVALID_ARG


def test_grad_set_checks_its_tensors():
    import torch

    with pytest.raises(ValueError):
        rrv.GradSet([])
    with pytest.raises(ValueError):
        rrv.GradSet([[]])
    with pytest.raises(ValueError):
        rrv.GradSet([[torch.zeros(4)], [torch.zeros(4)]])  # not CUDA tensors


# ------------------------------------------- AVG's division, in numbers --

def test_avg_quotient_through_fp64_equals_ieee_division():
    """The kernels compute a / N for a rank count N that is not a power of
    two as the fp64 product of a and the fp64 reciprocal of N, rounded once
    to fp32.  That is IEEE a / N in fp32 for every a (the argument: the
    product's error is far below the quotient's distance to a rounding
    boundary).  Checked here with numpy's IEEE arithmetic on random bit
    patterns of every binade, on the values nearest to N times a rounding
    midpoint (the hardest cases), and on zeros, subnormals and infinities."""
    rng = np.random.default_rng(20261203)
    bits = rng.integers(0, 0x7F800000, size=1 << 16, dtype=np.uint32)
    bits = np.concatenate([bits, bits | np.uint32(0x80000000)])  # both signs, every finite binade
    x = bits.view(np.float32)
    special = np.array([0.0, -0.0, np.inf, -np.inf, 1e-45, -1e-45, 1.1754942e-38, 3.4028235e38, 1.0, 3.0],
                       dtype=np.float32)
    for n in [k for k in range(3, 65) if k & (k - 1)]:
        # fp32 values next to n * m, m a midpoint between neighbouring fp32 values
        m_lo = rng.integers(1 << 23, 1 << 24, size=1 << 13).astype(np.float64)
        e = rng.integers(-140, 100, size=m_lo.size)
        m = (m_lo + 0.5) * np.exp2(e - 23.0)
        near = (m * n).astype(np.float32)
        near = np.concatenate([near, np.nextafter(near, np.float32(np.inf)), np.nextafter(near, np.float32(0))])
        a = np.concatenate([x, special, near[np.isfinite(near)]])
        want = a / np.float32(n)
        got = (a.astype(np.float64) * (1.0 / n)).astype(np.float32)
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), n


# ----------------------------------------------- the boundary from plain C --

C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "rr.h"

int main(void)
{
    /* host-only entry points of the C ABI, called from C99/C11 code */
    if (rr_version() != RR_VERSION) return 1;
    if (strcmp(rr_status_string(RR_OK), "ok") != 0) return 2;
    rr_ring_event_t ev[64];
    size_t nev = 0;
    if (rr_ring_schedule(4, 4096, RR_F32, ev, 64, &nev) != RR_OK || nev != 2 * 3 * 4) return 3;
    size_t sent = 0;  /* the pages' 4-rank example: 2(N-1)/N of 16 KiB per rank */
    for (size_t i = 0; i < nev; ++i)
        if (ev[i].rank == 0) sent += ev[i].bytes;
    if (sent != 24576) return 4;
    rr_cost_t cost;
    if (rr_cost_model(RR_ALGO_RING, 8, 1.0e9, 1.0e-6, 1.0e11, &cost) != RR_OK || cost.steps != 14.0) return 5;
    const size_t numels[4] = {100, 5000, 3, 777};
    rr_bucket_plan_t* plan = NULL;
    if (rr_bucket_plan(numels, 4, RR_BF16, 4096, &plan) != RR_OK || plan == NULL) return 6;
    int first = -1, nt = -1;
    size_t numel = 0;
    if (rr_bucket_count(plan) < 1 || rr_bucket_info(plan, 0, &first, &nt, &numel) != RR_OK || first != 0) return 7;
    rr_bucket_plan_free(plan);
    if (rr_allreduce(NULL, 4, 16, RR_F32, RR_SUM, RR_ALGO_AUTO, 0) != RR_ERR_INVALID_ARG) return 8;
    printf("c client ok\n");
    return 0;
}
"""


def test_c_client_compiles_links_and_runs_host_calls(tmp_path):
    """The boundary is plain C: a C11 program including rr.h compiles with
    warnings as errors, links against the library and runs the host-only
    calls (schedule, cost model, bucket plan, argument errors)."""
    import shutil

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    cuda_inc, cuda_lib = "/usr/local/cuda/include", "/usr/local/cuda/lib64"
    lib_dir = os.path.dirname(_lib.LIB_PATH)
    cmd = [gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           "-I", cuda_inc, str(src), "-o", str(exe), "-L", lib_dir, "-lrr_virtual", "-L", cuda_lib, "-lcudart",
           f"-Wl,-rpath,{lib_dir}", f"-Wl,-rpath,{cuda_lib}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and "c client ok" in run.stdout, (run.returncode, run.stderr)
