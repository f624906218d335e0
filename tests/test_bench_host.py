"""Host-side logic of bench.py, without a GPU: the multi-rank barrier and
max-over-ranks timing on 2 gloo processes, the clock-record parser, and the
reference arm (the CPU oracle) end to end."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    got = d.max(1.5 + rank, "cpu")  # each rank's "time"; every rank must see the max
    d.barrier()
    d.close()
    with open(os.path.join(out, f"r{rank}"), "w") as f:
        f.write(repr(got))


def test_max_over_ranks_on_two_gloo_ranks(tmp_path):
    mp.spawn(_rank_main, args=(_port(), str(tmp_path)), nprocs=2, join=True)
    assert [float(open(tmp_path / f"r{r}").read()) for r in range(2)] == [2.5, 2.5]


def test_clock_record_parser():
    u = "GPU-17731243-e024-de5d-5bb2-56de629d4926"
    lines = [f"{u}, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active\n",
             f"{u}, 1875, 1965, 990.2, 0x4, Not Active, Not Active, Not Active, Active\n",
             "GPU-other, 100, 1965, 1, 0x0, Active, Not Active, Not Active, Not Active\n", "garbage\n"]
    got = bench.Clocks.parse(lines, bench.Clocks._norm(u[4:]))
    assert got == {"sm_mhz": 1920.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 2}


def test_reference_arm_prints_one_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "1", "--ref-seconds", "1"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["metric"] == bench.METRIC and j["value"] > 0
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["cpu_baseline"]["kind"] == "oracle"
    assert j["higher_is_better"] is True and j["unit"] == "GB/s"


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2"],
                       capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_alpha_beta_fit_recovers_known_terms(capsys):
    """The sweep's least-squares fit of time = launches * alpha + bytes / beta
    returns the alpha and beta that generated exact points."""
    rows = [(k, b, k * 3e-6 + b / 7e12, (k * 1.5e-6 + b / 7e12) if b < 1e7 else None, False)
            for k in (1, 6, 14, 30) for b in (1e4, 1e6, 1e8, 1e10)]
    # L2-resident points above 4 MiB would pull beta up: they are left out
    rows += [(1, 5e7, 1e-6, None, True), (2, 9e7, 2e-6, None, True)]
    bench.fit_alpha_beta(rows)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["per_call"]["alpha_us"] == pytest.approx(3.0, rel=1e-6)
    assert line["per_call"]["beta_gbs"] == pytest.approx(7000.0, rel=1e-6)
    assert line["in_graph"]["alpha_us"] == pytest.approx(1.5, rel=1e-6)
    assert line["per_call"]["rel_residual_max"] < 1e-6
