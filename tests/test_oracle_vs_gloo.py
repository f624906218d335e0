"""Pin the oracle's collectives to PyTorch's own, run the way the pages run
them: 4 CPU processes over the gloo backend ([P4] "Collective communication
primitives", section "The five primitives").

On integer-valued inputs every reduction order gives the same exact result,
so the oracle must match the library bit for bit; on random fp32 inputs it
must match within the page's ``allclose(atol=1e-5)``.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from ring_all_reduce_virtual_b200 import synth

N = 4
PER = 6  # elements per rank block; count = N * PER


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, port, outdir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=N)
    try:
        res = {}
        ints = torch.from_numpy(synth.rank_values(3, rank, N * PER, "int", "f32"))
        small = torch.from_numpy(synth.cast(np.random.default_rng([4, rank]).integers(-3, 4, N * PER), "f32"))
        rnd = torch.from_numpy(synth.rank_values(5, rank, N * PER, "uniform", "f32"))
        for name, x in (("int", ints), ("small", small), ("rnd", rnd)):
            for op_name, op in (("sum", dist.ReduceOp.SUM), ("max", dist.ReduceOp.MAX),
                                ("min", dist.ReduceOp.MIN), ("prod", dist.ReduceOp.PRODUCT)):
                y = x.clone()
                dist.all_reduce(y, op=op)
                res[f"ar_{name}_{op_name}"] = y.numpy()
            chunk = torch.empty(PER)
            dist.reduce_scatter_tensor(chunk, x.clone())
            res[f"rs_{name}"] = chunk.numpy()
            gathered = torch.empty(N * PER)
            dist.all_gather_into_tensor(gathered, chunk)
            res[f"ag_{name}"] = gathered.numpy()
            out = torch.empty(N * PER)
            dist.all_to_all_single(out, x.clone())
            res[f"a2a_{name}"] = out.numpy()
        np.savez(os.path.join(outdir, f"rank{rank}.npz"), **res)
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def gloo_results(tmp_path_factory):
    outdir = str(tmp_path_factory.mktemp("gloo"))
    mp.spawn(_worker, args=(_free_port(), outdir), nprocs=N, join=True)
    return [dict(np.load(os.path.join(outdir, f"rank{r}.npz"))) for r in range(N)]


def _inputs(name):
    if name == "int":
        return [synth.rank_values(3, r, N * PER, "int", "f32") for r in range(N)]
    if name == "small":
        return [synth.cast(np.random.default_rng([4, r]).integers(-3, 4, N * PER), "f32") for r in range(N)]
    return [synth.rank_values(5, r, N * PER, "uniform", "f32") for r in range(N)]


@pytest.mark.parametrize("name,op", [("int", "sum"), ("int", "max"), ("int", "min"), ("small", "prod"),
                                     ("small", "sum")])
def test_allreduce_matches_gloo_exactly(gloo_results, name, op):
    for path in (oracle.ring_allreduce, oracle.fold_ring_order, oracle.tree_schedule):
        x = _inputs(name)
        path(x, op)
        for r in range(N):
            assert np.array_equal(x[r], gloo_results[r][f"ar_{name}_{op}"]), (path.__name__, r)


@pytest.mark.parametrize("name", ["int", "small"])
def test_rs_ag_a2a_match_gloo_exactly(gloo_results, name):
    x = _inputs(name)
    rs = oracle.reduce_scatter(x, "sum")
    ag = oracle.all_gather(rs)
    a2a = oracle.all_to_all(x)
    for r in range(N):
        assert np.array_equal(rs[r], gloo_results[r][f"rs_{name}"])
        assert np.array_equal(ag[r], gloo_results[r][f"ag_{name}"])
        assert np.array_equal(a2a[r], gloo_results[r][f"a2a_{name}"])


def test_random_fp32_within_page_tolerance(gloo_results):
    x = _inputs("rnd")
    oracle.ring_allreduce(x, "sum")
    for r in range(N):
        assert np.allclose(x[r], gloo_results[r]["ar_rnd_sum"], atol=1e-5)
    # max/min/a2a/ag involve no rounding: exact even on random data
    for op in ("max", "min"):
        y = _inputs("rnd")
        oracle.ring_allreduce(y, op)
        assert np.array_equal(y[2], gloo_results[2][f"ar_rnd_{op}"])
    a2a = oracle.all_to_all(_inputs("rnd"))
    assert np.array_equal(a2a[1], gloo_results[1]["a2a_rnd"])
