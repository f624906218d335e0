#!/usr/bin/env python3
"""Benchmark: all-reduce algbw / busbw and % of the HBM roofline for 8
virtual ranks x 256 MiB fp32 on one B200 (per GPU; N GPUs run N independent
copies of the workload, weak scaling).

One step = one ``all_reduce`` call through the library's public API (algo
AUTO, op AVG, in place) on 8 rank buffers of 64 Mi fp32 each: the chunk
partition, the ring-order fold with AVG's division, and the store of the
result to all 8 buffers.  Prints one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

``--impl reference`` times the CPU oracle (the plain ring all-reduce written
from the pages) on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "all-reduce algbw/busbw GB/s and % of HBM peak, 8 virtual ranks x 256 MB fp32"
WORKLOAD = "allreduce-8x256MiB-f32"
NRANKS = 8
COUNT = 1 << 26  # fp32 elements per rank: 256 MiB
ELEM = 4
SEED = 0
FALLBACK_HBM_GBS = 6650.0

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# the dominant kernel at the full 8 x 256 MiB size, from one ncu capture of
# that launch in steady state:
#   ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum
#       --clock-control none -k regex:bulk_fold_kernel -s 5 -c 1
#       python bench.py --steps 3 --warmup 5 --no-extra --no-e2e --no-cpu
# with the hash of the kernel's source files it was taken on (the bench
# reports null once they change).
NCU_TRAFFIC = {"bytes_per_launch": 2147919104 + 2091206912, "sources_sha1": "a19439deaae00055e91be891d75504bac94abc5b"}


# The files that hold the dominant kernel's device code (bulk_fold_kernel in
# ring order and the element types, operators and helpers it uses).
KERNEL_SOURCES = ("rr_device.cuh", "rr_bulk.cuh")


def sources_sha1() -> str:
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "ring_all_reduce_virtual_b200", "csrc")
    for name in KERNEL_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--cpu-seconds", type=float, default=8.0, help="CPU-baseline sample budget")
    ap.add_argument("--ref-seconds", type=float, default=90.0, help="reference-arm time budget")
    ap.add_argument("--no-extra", action="store_true", help="skip the per-algorithm extra timings")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end host-buffer timing")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline")
    ap.add_argument("--workload", choices=[WORKLOAD, "sweep", "gpt-buckets", "64x256MiB", "kernels", "overlap"],
                    default=WORKLOAD,
                    help="the headline workload (default), the message-size sweep, or the bucketed "
                         "gradient sync of a GPT-like model; the last two print one JSON line per point")
    ap.add_argument("--nranks", type=int, default=NRANKS, help="virtual ranks of --workload kernels")
    ap.add_argument("--reps", type=int, default=5, help="timed calls per kernel family of --workload kernels")
    ap.add_argument("--tokens", type=int, default=1024, help="tokens of the synthetic backward of --workload overlap")
    ap.add_argument("--odd", action="store_true",
                    help="--workload kernels: odd bucket tensor sizes, so later tensors sit out of phase with "
                         "their gradients in the fp32 bucket")
    ap.add_argument("--mixed", action="store_true",
                    help="--workload kernels: rank buffers of the all-reduces at different 16-byte phases "
                         "(rank r starts (3r + 1) mod 4 elements past a boundary)")
    ap.add_argument("--count", type=int, default=COUNT,
                    help="fp32 elements per virtual rank (default 2^26 = 256 MiB); smaller for profiling")
    return ap.parse_args()


# ------------------------------------------------------------- plumbing --

class Dist:
    """Rank/world from the launcher's environment; NCCL only for the
    barrier and the max over ranks of the measured time."""

    def __init__(self):
        self.rank = int(os.environ.get("RANK", "0"))
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False

    def init(self, backend: str):
        import torch.distributed as dist

        if self.world > 1 and not self.pg:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as dist

            dist.barrier()

    def max(self, x: float, device) -> float:
        if not self.pg:
            return x
        import torch
        import torch.distributed as dist

        t = torch.tensor([x], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist

            dist.destroy_process_group()
            self.pg = False


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed
    region."""

    FIELDS = ["uuid", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, uuid: str | None):
        self.uuid = self._norm(uuid)
        self.proc = None
        self.path = None

    @staticmethod
    def _norm(u) -> str:
        u = str(u or "").lower()
        return u[4:].replace("-", "") if u.startswith("gpu-") else u.replace("-", "")

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="rr_clocks_", suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS), "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return self.parse(lines, self.uuid)

    @classmethod
    def parse(cls, lines, uuid: str = ""):
        """Median SM clock, max clock and the throttle reasons seen."""
        rows = []
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(cls.FIELDS):
                continue
            if uuid and cls._norm(parts[0]) != uuid:
                continue
            rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- inputs --

def host_inputs(rank_offset: int, count: int):
    from ring_all_reduce_virtual_b200 import synth

    return [synth.rank_values(SEED + rank_offset, r, count, "normal", "f32") for r in range(NRANKS)]


# ------------------------------------------------------------ cpu oracle --

def cpu_baseline(budget_s: float):
    """The oracle's ring all-reduce on a bounded sample (8 ranks x m fp32),
    single-threaded and with each step's transfers on all host cores."""
    import oracle
    from ring_all_reduce_virtual_b200 import synth

    m = 1 << 20
    x = synth.ranks(SEED, NRANKS, m, "normal", "f32")
    t0 = time.perf_counter()
    oracle.ring_allreduce(x, "avg")
    one = time.perf_counter() - t0
    reps = max(1, int(budget_s / 2 / max(one, 1e-6)))
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.ring_allreduce(x, "avg")
    t1 = (time.perf_counter() - t0) / reps
    cores = os.cpu_count() or 1
    oracle.ring_allreduce_omp(x, "avg", cores)
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.ring_allreduce_omp(x, "avg", cores)
    tp = (time.perf_counter() - t0) / reps
    S = m * ELEM
    return {
        "value": round(S / t1 / 1e9, 4), "unit": "GB/s (algbw)", "cores": 1, "kind": "oracle",
        "sample": f"{reps} ring all-reduce calls (AVG) of {NRANKS} ranks x {m} fp32 ({S >> 20} MiB per rank), "
                  f"single-threaded C oracle",
        "parallel": {"value": round(S / tp / 1e9, 4), "cores": cores,
                     "kind": "oracle, each step's N transfers on host threads (OpenMP)"},
        "cpu_model": _cpu_model(),
    }


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def run_reference(args, d: Dist):
    """The reference arm: the CPU oracle, as it stands, on a bounded sample
    of this workload per step (rank 0 only)."""
    if d.rank != 0:
        return
    import oracle
    from ring_all_reduce_virtual_b200 import synth

    steps, warm = args.steps, args.warmup
    m = 1 << 16
    x = synth.ranks(SEED, NRANKS, m, "normal", "f32")
    t0 = time.perf_counter()
    oracle.ring_allreduce(x, "avg")
    one = max(time.perf_counter() - t0, 1e-6)
    budget = 0.5 * args.ref_seconds / max(steps + warm, 1)  # whole run within the budget (time grows faster than m)
    m = int(min(COUNT, max(4096, m * budget / one)))
    m -= m % NRANKS
    x = synth.ranks(SEED, NRANKS, m, "normal", "f32")
    for _ in range(warm):
        oracle.ring_allreduce(x, "avg")
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle.ring_allreduce(x, "avg")
    dt = (time.perf_counter() - t0) / max(steps, 1)
    S = m * ELEM
    algbw = S / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(algbw, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": warm, "ms_per_step": round(dt * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic: normal(0, 1e-3) fp32 from numpy default_rng([seed, rank])",
        "config": {"workload": WORKLOAD, "nranks_virtual": NRANKS, "count_per_rank": m,
                   "sample_of_count_per_rank": COUNT, "op": "avg", "algo": "ring (CPU oracle)"},
        "busbw": round(algbw * 2 * (NRANKS - 1) / NRANKS, 4),
        "cpu_baseline": {"value": round(algbw, 4), "unit": "GB/s (algbw)", "cores": 1, "kind": "oracle",
                         "sample": f"each step: ring all-reduce (AVG) of {NRANKS} ranks x {m} fp32, "
                                   f"single-threaded C oracle", "cpu_model": _cpu_model()},
        "e2e": {"value": round(algbw, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ ours --

def run_ours(args, d: Dist):
    import torch

    import ring_all_reduce_virtual_b200 as rrv
    from ring_all_reduce_virtual_b200.build import build

    torch.cuda.set_device(d.local_rank)
    dev = torch.device("cuda", d.local_rank)
    d.init("nccl")
    if d.rank == 0:
        build()  # no-op when the library is up to date
    d.barrier()  # the other ranks load the library only once it is built
    stream = torch.cuda.current_stream(dev)

    count = args.count
    host = host_inputs(d.rank * NRANKS, count)
    bufs = [torch.from_numpy(a).to(dev) for a in host]
    S = count * ELEM
    alg_bytes = 2 * NRANKS * S  # one-shot: read N*S, write N*S

    def step():
        rrv.all_reduce(bufs, "avg", "auto", stream)

    # warm-up, then exactly K timed steps between barriers and syncs
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    picked = rrv.last_stats()
    clocks = Clocks(getattr(torch.cuda.get_device_properties(dev), "uuid", None))
    clocks.start()
    d.barrier()
    torch.cuda.synchronize(dev)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    d.barrier()
    clk = clocks.stop()
    ms_local = ev0.elapsed_time(ev1) / max(args.steps, 1)
    ms = d.max(ms_local, dev)
    t = ms / 1e3
    algbw = S / t / 1e9  # per GPU
    value = algbw * d.world  # whole job: every GPU reduces its own 8 x 256 MiB
    busbw = algbw * 2 * (NRANKS - 1) / NRANKS
    achieved = alg_bytes / t / 1e9
    peak, peak_kind = hbm_peak()
    traffic = None
    if NCU_TRAFFIC["bytes_per_launch"] and NCU_TRAFFIC["sources_sha1"] == sources_sha1() and count == COUNT:
        traffic = int(NCU_TRAFFIC["bytes_per_launch"])

    copy_gbs = None if args.no_extra else time_copy_ceiling(dev, stream, NRANKS * S)
    # end to end through the public API with host buffers: H2D + all-reduce + D2H
    e2e = None
    if not args.no_e2e:
        e2e = time_e2e(args, d, dev, stream, host, bufs, S)
    extra = {} if args.no_extra else time_extra(dev, stream, host, S, hbm_peak()[0])
    cpu = cpu_baseline(args.cpu_seconds) if (d.rank == 0 and d.world == 1 and not args.no_cpu) else None
    if d.rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": d.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32",
            "data": "synthetic: normal(0, 1e-3) fp32 from numpy default_rng([seed, rank]), generated on the host",
            "config": {"workload": WORKLOAD if count == COUNT else f"allreduce-8x{count}-f32", "nranks_virtual": NRANKS,
                       "count_per_rank": count, "bytes_per_rank": S, "op": "avg",
                       "algo": "auto -> " + str(picked["algo"]), "in_place": True,
                       "value_is": "algbw = S / T summed over GPUs",
                       "l2": f"inputs {NRANKS * S / 2**30:.2f} GiB per GPU vs 126 MB L2; no flush between steps"},
            "algbw_per_gpu": round(algbw, 3), "busbw": round(busbw, 3),
            "hbm_gbs": round(achieved, 1), "hbm_frac": round(achieved / peak, 4),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic,
                         "kernel": "bulk_fold_kernel<F32T, AVG, N 8, ring order> (bulk-copy tiles, 2 KB per rank)",
                         "algorithmic_bytes_per_launch": alg_bytes, "peak_kind": peak_kind + " (burst copy)"},
            "copy_ceiling": None if copy_gbs is None else {
                "copy_gbs": round(copy_gbs[0], 1), "frac_of_copy": round(achieved / copy_gbs[0], 4),
                "own_copy_gbs": round(copy_gbs[1], 1), "frac_of_own_copy": round(achieved / copy_gbs[1], 4),
                "what": "copies of the same 2 GiB (read + write), timed in this run like the headline: torch "
                        "copy_, and the library's own copy kernel (all-to-all of one rank)"},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": int(picked["launches"]) * args.steps,
            "clocks": clk,
            "extra": extra,
        }
        print(json.dumps(line), flush=True)
    d.close()


def time_copy_ceiling(dev, stream, nbytes):
    """GB/s (read + write) of plain device-to-device copies of nbytes, the
    same traffic as one headline call, with CUDA events on the stream: torch's
    copy_, and the library's own copy kernel (an all-to-all of one rank, which
    copies its buffer)."""
    import torch

    import ring_all_reduce_virtual_b200 as rrv

    src = torch.empty(nbytes // 4, dtype=torch.float32, device=dev).normal_()
    dst = torch.empty_like(src)

    def rate(fn):
        with torch.cuda.stream(stream):
            for _ in range(5):
                fn()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(50):
                fn()
            b.record(stream)
        torch.cuda.synchronize(dev)
        return 2 * nbytes / (a.elapsed_time(b) / 50 / 1e3) / 1e9

    torch_gbs = rate(lambda: dst.copy_(src))
    own_gbs = rate(lambda: rrv.all_to_all([src], [dst], stream))
    del src, dst
    return torch_gbs, own_gbs


def time_e2e(args, d, dev, stream, host, bufs, S):
    import torch

    import ring_all_reduce_virtual_b200 as rrv

    pinned = [torch.from_numpy(a).pin_memory() for a in host]
    for _ in range(2):
        rrv.all_reduce_host(pinned, bufs, "avg", "auto", stream)
    torch.cuda.synchronize(dev)
    d.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        rrv.all_reduce_host(pinned, bufs, "avg", "auto", stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    d.barrier()
    e2e_ms = d.max(e0.elapsed_time(e1) / max(args.e2e_steps, 1), dev)
    return {"value": round(S / (e2e_ms / 1e3) / 1e9 * d.world, 3), "unit": "GB/s",
            "h2d_bytes_per_step": NRANKS * S, "d2h_bytes_per_step": NRANKS * S,
            "ms_per_step": round(e2e_ms, 3), "host_memory": "pinned"}


def time_extra(dev, stream, host, S, peak):
    """The other algorithms on the same workload (a few calls each)."""
    import torch

    import ring_all_reduce_virtual_b200 as rrv

    extra = {}
    for name, op, algo, reps in (("oneshot_sum", "sum", "oneshot", 20), ("ring_sum", "sum", "ring", 10),
                                 ("tree_oneshot_sum", "sum", "tree_oneshot", 10), ("tree_sum", "sum", "tree", 10)):
        fresh = [torch.from_numpy(a).to(dev) for a in host]
        rrv.all_reduce(fresh, op, algo, stream)
        st = rrv.last_stats()
        torch.cuda.synchronize(dev)
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(reps):
            rrv.all_reduce(fresh, op, algo, stream)
        a1.record(stream)
        torch.cuda.synchronize(dev)
        tm = a0.elapsed_time(a1) / reps / 1e3
        extra[name] = {"ms": round(tm * 1e3, 4), "algbw_gbs": round(S / tm / 1e9, 2),
                       "hbm_gbs": round(st["hbm_bytes"] / tm / 1e9, 1),
                       "hbm_frac": round(st["hbm_bytes"] / tm / 1e9 / peak, 4), "launches": st["launches"]}
        del fresh
    # bf16 and fp16 gradients (fp32 accumulation, one rounding): the same 256 MiB per rank
    gen = torch.Generator(device=dev).manual_seed(SEED)
    for name, dt in (("oneshot_bf16_avg", torch.bfloat16), ("oneshot_f16_avg", torch.float16)):
        g16 = [(torch.randn(2 * len(h), device=dev, generator=gen) * 1e-3).to(dt) for h in host]
        rrv.all_reduce(g16, "avg", "auto", stream)
        st = rrv.last_stats()
        torch.cuda.synchronize(dev)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(20):
            rrv.all_reduce(g16, "avg", "auto", stream)
        a1.record(stream)
        torch.cuda.synchronize(dev)
        tm = a0.elapsed_time(a1) / 20 / 1e3
        extra[name] = {"ms": round(tm * 1e3, 4), "algbw_gbs": round(S / tm / 1e9, 2),
                       "hbm_gbs": round(st["hbm_bytes"] / tm / 1e9, 1),
                       "hbm_frac": round(st["hbm_bytes"] / tm / 1e9 / peak, 4), "launches": st["launches"]}
        del g16
    return extra


def fit_alpha_beta(rows):
    """Fit of the alpha-beta model to the sweep ([P3] section 4: time =
    steps * alpha + bytes / beta; on one GPU a step is a launch and the bytes
    are HBM bytes), per call from Python and per call inside a CUDA graph
    (small sizes).  rows: (launches, HBM bytes, seconds per call, seconds per
    call in a graph or None, L2-resident).  Each point is weighted by 1 / its
    time, so the fit minimises relative error and the small sizes that fix
    alpha count as much as the large ones that fix beta; points whose bytes
    are L2-resident and not negligible (above 4 MiB) are left out, since L2
    is faster than the HBM beta describes.  Prints one JSON line with the pair
    and the fit's relative residuals; rr_set_picker_params takes such a pair."""
    import numpy as np

    out = {"workload": "size-sweep-f32-sum",
           "fit": "alpha-beta, least squares weighted by 1/time (relative error), over launch-bound points "
                  "and HBM-resident points (L2-resident points above 4 MiB left out)"}
    for key, idx in (("per_call", 2), ("in_graph", 3)):
        pts = [(r[0], r[1], r[idx]) for r in rows
               if r[idx] is not None and r[idx] > 0 and (r[1] <= 4 << 20 or not (len(r) > 4 and r[4]))]
        if len(pts) < 3:
            continue
        a = np.array([[p[0], p[1]] for p in pts], dtype=float)
        y = np.array([p[2] for p in pts], dtype=float)
        w = 1.0 / y
        sol = np.linalg.lstsq(a * w[:, None], y * w, rcond=None)[0]
        if sol[1] > 0 and sol[0] > 0:
            rel = (a @ sol - y) / y
            out[key] = {"alpha_us": round(sol[0] * 1e6, 3), "beta_gbs": round(1 / sol[1] / 1e9, 1), "points": len(pts),
                        "rel_residual_rms": round(float(np.sqrt(np.mean(rel ** 2))), 4),
                        "rel_residual_max": round(float(np.max(np.abs(rel))), 4)}
    print(json.dumps(out), flush=True)


SWEEP_NS = (2, 4, 8, 16)  # the size sweep's rank counts
SWEEP_ALGOS = ("ring", "oneshot", "two_shot", "tree", "tree_oneshot", "double_ring", "ring_steps")
PICKER_NS = (3, 5, 6, 7, 12, 24, 32, 48, 64)  # further rank counts the picker's table covers
PICKER_ALGOS = ("ring", "oneshot", "two_shot")  # AUTO's candidates (the ring's bits)
PICKER_SIZES = (10, 16, 20, 24, 28, 30)  # log2 bytes per rank
ALIGN_NS = (4, 5, 8)
ALIGN_SIZES = (16, 24, 28)


def _offsets(kind: str, n: int):
    """Element offsets of each rank's buffer from a 16-byte boundary: aligned,
    all ranks one fp32 element past it (a shared phase), or phases that
    differ between ranks (the scalar path)."""
    if kind == "aligned":
        return [0] * n
    if kind == "shared":
        return [1] * n
    return [r % 4 for r in range(n)]


def run_sweep(args):
    """Message-size sweep: 1 KiB .. 1 GiB per rank, N in {2, 4, 8, 16}, fp32
    SUM, every algorithm (ring, one-shot, two-shot, tree schedule, tree-order
    one-shot, double ring); then AUTO's candidates at further rank counts
    (3 .. 64) and sizes, and with misaligned buffers.  Per point: median
    per-call device time over 20 calls after 5 warm-ups, the library's own
    host time per call (rr_get_stats host_ns, and launch_ns spent in the
    launch calls), and for sizes up to 1 MiB the per-call time through a
    RankSet (pointers marshalled once) and inside a CUDA graph of 100 calls.
    Points whose 2 N S bytes fit in L2 are flagged.  The last line is the
    alpha-beta fit of the first part's points."""
    import torch

    import ring_all_reduce_virtual_b200 as rrv
    from ring_all_reduce_virtual_b200.build import build

    build()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.Stream(dev)
    peak, _ = hbm_peak()
    fit_rows = []  # (launches, HBM bytes, s per call, s per call in a graph, L2-resident)

    def call_of(algo, bufs, n):
        """One all-reduce as a callable; "ring_steps" is the ring schedule as
        2(N-1) rr_ring_step launches.  stats_of() then gives its statistics
        (summed over the steps)."""
        if algo != "ring_steps":
            return (lambda: rrv.all_reduce(bufs, "sum", algo, stream)), rrv.last_stats
        step_stats = []

        def steps():
            step_stats.clear()
            for phase in ("reduce_scatter", "all_gather"):
                for s_ in range(n - 1):
                    rrv.ring_step(bufs, "sum", phase, s_, stream)
                    step_stats.append(rrv.last_stats())

        def stats_of():
            tot = dict(step_stats[0])
            for st_ in step_stats[1:]:
                for key in ("launches", "hbm_bytes", "host_ns", "launch_ns"):
                    tot[key] += st_[key]
            return tot
        return steps, stats_of

    def point(n, nbytes, algo, bufs, align, part):
        run, stats_of = call_of(algo, bufs, n)
        with torch.cuda.stream(stream):
            for _ in range(5):
                run()
            st = stats_of()
            times, host_ns, launch_ns = [], [], []
            for _ in range(20):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                run()
                b.record(stream)
                s2 = stats_of()
                host_ns.append(s2["host_ns"])
                launch_ns.append(s2["launch_ns"])
                times.append((a, b))
            stream.synchronize()
            t = statistics.median(x.elapsed_time(y) for x, y in times) / 1e3
            graph_us = rankset_us = bound_us = loop_us = None
            if nbytes <= 16 << 20 and algo != "ring_steps":
                # per call inside a CUDA graph of 100 calls: device time plus launch, no Python
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for _ in range(100):
                        rrv.all_reduce(bufs, "sum", algo, stream)
                g.replay()
                stream.synchronize()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for _ in range(5):
                    g.replay()
                b.record(stream)
                stream.synchronize()
                graph_us = a.elapsed_time(b) * 1e3 / 500
                del g
            if nbytes <= 1 << 20 and algo != "ring_steps":
                rs = rrv.RankSet(bufs)
                bound = rs.bind("sum", algo, stream)  # arguments converted once
                for label, fn in (("rankset", lambda: rrv.all_reduce(rs, "sum", algo, stream)), ("bound", bound)):
                    times = []
                    for _ in range(20):
                        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                        a.record(stream)
                        fn()
                        b.record(stream)
                        times.append((a, b))
                    stream.synchronize()
                    us = statistics.median(x.elapsed_time(y) for x, y in times) * 1e3
                    if label == "rankset":
                        rankset_us = us
                    else:
                        bound_us = us
                # host-bound loop: 200 bound calls back to back, wall time per call
                stream.synchronize()
                t0 = time.perf_counter()
                for _ in range(200):
                    bound()
                loop_us = (time.perf_counter() - t0) / 200 * 1e6
                stream.synchronize()
        algbw = nbytes / t / 1e9
        l2 = 2 * n * nbytes <= 126 * 10**6
        if part == "sizes" and algo in ("oneshot", "two_shot", "tree_oneshot", "ring_steps"):
            # the algorithms whose algorithmic bytes are the DRAM bytes (the
            # one-launch schedules serve most of theirs from L2)
            fit_rows.append((st["launches"], st["hbm_bytes"], t, None if graph_us is None else graph_us * 1e-6, l2))
        print(json.dumps({
            "workload": "size-sweep-f32-sum", "part": part, "nranks_virtual": n, "bytes_per_rank": nbytes,
            "algo": algo, "align": align, "latency_us": round(t * 1e6, 3),
            "host_us": round(statistics.median(host_ns) / 1e3, 3),
            "launch_call_us": round(statistics.median(launch_ns) / 1e3, 3),
            "graph_latency_us": None if graph_us is None else round(graph_us, 3),
            "rankset_latency_us": None if rankset_us is None else round(rankset_us, 3),
            "bound_latency_us": None if bound_us is None else round(bound_us, 3),
            "bound_loop_us": None if loop_us is None else round(loop_us, 3),
            "algbw_gbs": round(algbw, 3), "busbw_gbs": round(algbw * 2 * (n - 1) / n, 3),
            "hbm_gbs": round(st["hbm_bytes"] / t / 1e9, 1), "hbm_frac": round(st["hbm_bytes"] / t / 1e9 / peak, 4),
            "launches": st["launches"], "l2_resident": l2}), flush=True)

    def ranks(n, count, align):
        offs = _offsets(align, n)
        if align == "aligned":
            return [torch.randn(count, device=dev) for _ in range(n)]
        return [torch.randn(count + 4, device=dev)[o:o + count] for o in offs]

    for n in SWEEP_NS:
        for e in range(10, 31):
            bufs = ranks(n, (1 << e) // ELEM, "aligned")
            for algo in SWEEP_ALGOS:
                point(n, 1 << e, algo, bufs, "aligned", "sizes")
            del bufs
            torch.cuda.empty_cache()
    fit_alpha_beta(fit_rows)
    for n in PICKER_NS:
        for e in PICKER_SIZES:
            count = (1 << e) // ELEM
            bufs = ranks(n, count, "aligned")
            for algo in PICKER_ALGOS:
                point(n, count * ELEM, algo, bufs, "aligned", "ranks")
            del bufs
            torch.cuda.empty_cache()
    for align in ("shared", "mixed"):
        for n in ALIGN_NS:
            for e in ALIGN_SIZES:
                count = (1 << e) // ELEM
                bufs = ranks(n, count, align)
                for algo in PICKER_ALGOS:
                    point(n, count * ELEM, algo, bufs, align, "align")
                del bufs
                torch.cuda.empty_cache()


def run_gpt_buckets(args):
    """Bucketed gradient sync of a GPT-like model (24 layers, d_model 2048,
    4x MLP, 32k vocab: 293 bf16 tensors, 1.34 B parameters per rank) over 8
    virtual ranks with 25 MiB buckets and AVG: the fused path (4 bytes per
    parameter per rank) one bucket per call and all buckets in one range call,
    and the staged pack -> all-reduce -> unpack path (20 bytes).  Gradients are normal(0, 1e-3) drawn on the device (timing does
    not depend on the values)."""
    import torch

    import ring_all_reduce_virtual_b200 as rrv
    from ring_all_reduce_virtual_b200 import synth
    from ring_all_reduce_virtual_b200.build import build

    build()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    n = 8
    numels = [m for _, m in synth.grad_ready_order(synth.gpt_grad_tensors())]
    params = sum(numels)
    gen = torch.Generator(device=dev).manual_seed(SEED)
    grads = [[(torch.randn(m, device=dev, generator=gen) * 1e-3).to(torch.bfloat16) for m in numels]
             for _ in range(n)]
    plan = rrv.BucketPlan(numels, "bf16", synth.BUCKET_CAP_BYTES)
    gset = rrv.GradSet(grads)  # pointers marshalled once, as a DDP step would
    nb = plan.num_buckets
    biggest = max(plan.info(b)[2] for b in range(nb))
    buckets = [torch.empty(biggest, dtype=torch.float32, device=dev) for _ in range(n)]
    peak, _ = hbm_peak()

    views = [[t[:plan.info(b)[2]] for t in buckets] for b in range(nb)]

    def launches(call):  # run one library call and return how many kernels it launched
        call()
        return rrv.last_stats()["launches"]

    def fused():  # one fused sync per bucket, as each bucket becomes ready
        return sum(launches(lambda: plan.all_reduce(b, gset, "avg", stream)) for b in range(nb))

    def fused_range():  # every bucket at once: the buckets share launches
        return launches(lambda: plan.all_reduce_range(0, nb, gset, "avg", stream))

    def staged():
        k = 0
        for b in range(nb):
            k += launches(lambda: plan.pack(b, gset, buckets, stream))
            k += launches(lambda: rrv.all_reduce(views[b], "sum", "auto", stream))
            k += launches(lambda: plan.unpack(b, buckets, gset, "avg", stream))
        return k

    for name, fn, bpp in (("fused", fused, 4), ("fused_range", fused_range, 4), ("staged", staged, 20)):
        nl = fn()
        for _ in range(max(args.warmup, 3) - 1):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 10
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        t = a.elapsed_time(b) / reps / 1e3
        hbm = n * params * bpp
        print(json.dumps({
            "workload": "gpt-24x2048-buckets-bf16-avg", "path": name, "nranks_virtual": n, "params_per_rank": params,
            "tensors": len(numels), "buckets": nb, "bucket_cap_bytes": synth.BUCKET_CAP_BYTES,
            "ms_per_sync": round(t * 1e3, 3), "grad_bytes_per_rank": params * 2,
            "algbw_gbs": round(params * 2 / t / 1e9, 2), "hbm_bytes_per_param_per_rank": bpp,
            "hbm_gbs": round(hbm / t / 1e9, 1), "hbm_frac": round(hbm / t / 1e9 / peak, 4),
            "launches_per_sync": nl}), flush=True)


def run_64_ranks(args):
    """64 virtual ranks x 64 Mi fp32 (16 GiB): all-reduce SUM/MAX/MIN/PROD
    (PROD on [0.99, 1.01]) and reduce-scatter, all-gather, all-to-all, each
    timed over 10 calls.  Inputs are drawn on the device (timing does not
    depend on the values)."""
    import torch

    import ring_all_reduce_virtual_b200 as rrv
    from ring_all_reduce_virtual_b200.build import build

    build()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    n, count = 64, COUNT
    S = count * ELEM
    peak, _ = hbm_peak()
    gen = torch.Generator(device=dev).manual_seed(SEED)
    x = [torch.rand(count, device=dev, generator=gen) * 2 - 1 for _ in range(n)]

    def timed(fn, reps=10):
        fn()
        st = rrv.last_stats()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / reps / 1e3, st

    def emit(what, t, st):
        print(json.dumps({"workload": "64x256MiB-f32", "call": what, "nranks_virtual": n, "bytes_per_rank": S,
                          "ms": round(t * 1e3, 3), "algbw_gbs": round(S / t / 1e9, 2),
                          "hbm_gbs": round(st["hbm_bytes"] / t / 1e9, 1),
                          "hbm_frac": round(st["hbm_bytes"] / t / 1e9 / peak, 4), "launches": st["launches"]}),
              flush=True)

    for op in ("sum", "max", "min"):
        emit(f"all_reduce {op}", *timed(lambda: rrv.all_reduce(x, op, "auto", stream)))
    for t in x:  # PROD inputs: uniform[0.99, 1.01) on every rank
        t.uniform_(0.99, 1.01, generator=gen)
    emit("all_reduce prod", *timed(lambda: rrv.all_reduce(x, "prod", "auto", stream)))
    per = count // n
    rs = [torch.empty(per, device=dev) for _ in range(n)]
    emit("reduce_scatter sum", *timed(lambda: rrv.reduce_scatter(x, rs, "sum", "auto", stream)))
    out = [torch.empty(count, device=dev) for _ in range(n)]
    emit("all_gather", *timed(lambda: rrv.all_gather(rs, out, "auto", stream)))
    emit("all_to_all", *timed(lambda: rrv.all_to_all(x, out, stream)))


def run_kernels(args):
    """Every kernel family once per call at a chosen size (--nranks, --count
    fp32 elements per rank): one-shot, two-shot, ring, tree and tree-order
    all-reduce, reduce-scatter, all-gather, all-to-all, and the bucket pack,
    unpack and fused sync on bf16 gradients of the same total size.  One JSON
    line per call with its time and HBM fraction; small sizes make this the
    target for per-kernel ncu captures."""
    import torch

    import ring_all_reduce_virtual_b200 as rrv
    from ring_all_reduce_virtual_b200.build import build

    build()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    n, count = args.nranks, args.count - args.count % args.nranks
    S = count * ELEM
    peak, _ = hbm_peak()
    gen = torch.Generator(device=dev).manual_seed(SEED)
    if args.mixed:  # views at unequal offsets: no two ranks share a 16-byte phase (up to 4 ranks)
        x = [(torch.randn(count + 4, device=dev, generator=gen) * 1e-3)[(3 * r + 1) % 4:][:count] for r in range(n)]
    else:
        x = [torch.randn(count, device=dev, generator=gen) * 1e-3 for _ in range(n)]
    per = count // n
    rs = [torch.empty(per, device=dev) for _ in range(n)]
    out = [torch.empty(count, device=dev) for _ in range(n)]
    # three tensors, two small and one large, sized in multiples of 8 elements so
    # every tensor's offset in the fp32 bucket has its gradient's 16-byte phase
    # (a model's tensors usually do); with --odd the first two sizes are odd,
    # so the next tensors start 1 and 2 elements out of phase
    small = (per // 3) & ~7
    numels = [small + 1, small + 1, count - 2 * small - 2] if args.odd else [small, small, count - 2 * small]
    grads = rrv.GradSet([[(torch.randn(m, device=dev, generator=gen) * 1e-3).to(torch.bfloat16) for m in numels]
                         for _ in range(n)])
    plan = rrv.BucketPlan(numels, "bf16", 2 * count)  # one bucket
    buckets = [torch.empty(count, device=dev) for _ in range(n)]

    def emit(what, fn):
        fn()
        st = rrv.last_stats()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        t = a.elapsed_time(b) / max(args.reps, 1) / 1e3
        print(json.dumps({"workload": f"kernels-{n}x{count}-f32" + ("-odd" if args.odd else "")
                          + ("-mixed" if args.mixed else ""), "call": what,
                          "ms": round(t * 1e3, 4),
                          "hbm_gbs": round(st["hbm_bytes"] / t / 1e9, 1),
                          "hbm_frac": round(st["hbm_bytes"] / t / 1e9 / peak, 4), "launches": st["launches"]}),
              flush=True)

    for algo in ("oneshot", "two_shot", "ring", "double_ring", "tree", "tree_oneshot"):
        emit(f"all_reduce {algo}", lambda: rrv.all_reduce(x, "sum", algo, stream))
    for algo in ("oneshot", "ring"):
        emit(f"all_reduce_wire bf16 {algo}", lambda: rrv.all_reduce_wire(x, "avg", "bf16", algo, stream))
    emit("reduce_scatter", lambda: rrv.reduce_scatter(x, rs, "sum", "auto", stream))
    emit("all_gather", lambda: rrv.all_gather(rs, out, "auto", stream))
    emit("all_to_all", lambda: rrv.all_to_all(x, out, stream))
    emit("bucket_pack", lambda: plan.pack(0, grads, buckets, stream))
    emit("bucket_unpack", lambda: plan.unpack(0, buckets, grads, "avg", stream))
    emit("bucket_allreduce", lambda: plan.all_reduce(0, grads, "avg", stream))


def run_overlap(args):
    """Bucket syncs overlapped with a synthetic backward (GPT-like model, 8
    virtual ranks, 25 MiB buckets, AVG).  The backward produces every rank's
    gradient of each tensor, in gradient-ready order, with one batched bf16
    GEMM per tensor (weight gradient = X^T dY over --tokens tokens; vectors
    as a GEMM with a ones row).  Timed: backward alone, syncs alone, backward
    then syncs, backward with the reducer launching each bucket's sync on a
    second stream as soon as it is ready, and that overlapped step captured
    in one CUDA graph; with the syncs' CTAs capped, and with cuBLAS keeping a
    number of SMs free of GEMM work (PyTorch's experimental SM carve-out) so
    that the capped syncs run beside the GEMMs.  Exposed sync time is counted
    against the backward without a carve-out."""
    import torch

    import ring_all_reduce_virtual_b200 as rrv
    from ring_all_reduce_virtual_b200 import synth
    from ring_all_reduce_virtual_b200.build import build

    build()
    dev = torch.device("cuda", 0)
    n, T = 8, args.tokens
    tensors = synth.grad_ready_order(synth.gpt_grad_tensors())
    d = 2048
    shapes = []
    for name, m in tensors:  # (rows, cols) of each gradient as a GEMM output
        rows = d if m % d == 0 and m // d > 1 else 1
        shapes.append((rows, m // rows))
    bufs = [torch.empty((n, r, c), dtype=torch.bfloat16, device=dev) for r, c in shapes]
    grads = rrv.GradSet([[bufs[t][r].view(-1) for t in range(len(tensors))] for r in range(n)])
    gen = torch.Generator(device=dev).manual_seed(SEED)
    act = {}
    for r, c in shapes:  # one activation / output-gradient pair per shape, shared by the ranks
        for k in (r, c):
            if k not in act:
                act[k] = (torch.randn((1, T, k), device=dev, generator=gen) * 1e-2).to(torch.bfloat16)
    ones = torch.ones((1, 1, T), dtype=torch.bfloat16, device=dev)
    lhs = [(ones if r == 1 else act[r].transpose(1, 2)).expand(n, r, T) for r, c in shapes]
    rhs = [act[c].expand(n, T, c) for r, c in shapes]
    plan = rrv.BucketPlan([m for _, m in tensors], "bf16", synth.BUCKET_CAP_BYTES)
    compute = torch.cuda.Stream(dev)
    red = None

    def backward(mark):
        for t in range(len(tensors)):
            torch.bmm(lhs[t], rhs[t], out=bufs[t])
            if mark:
                red.ready(t, compute)
        if mark:
            red.finish(compute)

    def syncs():
        for b in range(plan.num_buckets):
            plan.all_reduce(b, grads, "avg", compute)

    def timed(fn, reps=5):
        with torch.cuda.stream(compute):
            fn()
            compute.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(compute)
            for _ in range(reps):
                fn()
            b.record(compute)
            b.synchronize()
        return a.elapsed_time(b) / reps

    t_b0 = timed(lambda: backward(False))
    t_s = timed(syncs)
    t_serial = timed(lambda: (backward(False), syncs()))
    flops = 2.0 * T * sum(m for _, m in tensors) * n
    # (SMs kept free of GEMM work, CTAs per bucket sync): the syncs on a
    # high-priority stream, capped or not; with a carve-out the GEMMs leave
    # SMs to the capped syncs (about 2 CTAs of the fused kernel per free SM)
    for carve, ctas in ((0, 0), (0, 32), (0, 64), (0, 128), (0, 256), (8, 16), (16, 32), (32, 64)):
        torch._C._set_sm_carveout_experimental(carve or None)
        t_b = timed(lambda: backward(False)) if carve else t_b0
        red = rrv.Reducer(plan, grads, "avg", max_ctas=ctas)
        t_over = timed(lambda: backward(True))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(compute):
            backward(True)
            compute.synchronize()
        with torch.cuda.graph(g, stream=compute):
            backward(True)
        t_graph = timed(g.replay)
        del g
        print(json.dumps({
            "workload": "gpt-24x2048-overlap-bf16-avg", "nranks_virtual": n, "tokens": T, "buckets": plan.num_buckets,
            "gemm_sm_carveout": carve, "sync_ctas": ctas or "one per tile", "backward_ms": round(t_b, 3),
            "backward_tflops": round(flops / t_b / 1e9, 1), "syncs_ms": round(t_s, 3),
            "serial_ms": round(t_serial, 3), "overlapped_ms": round(t_over, 3), "overlapped_graph_ms": round(t_graph, 3),
            "exposed_sync_ms": round(t_over - t_b0, 3), "exposed_sync_graph_ms": round(t_graph - t_b0, 3),
            "graph_vs_serial": round(t_graph / t_serial, 3),
            "hidden_fraction_graph": round(1 - (t_graph - t_b0) / t_s, 3) if t_s > 0 else None}), flush=True)
    torch._C._set_sm_carveout_experimental(None)


def main():
    args = parse_args()
    d = Dist()
    if args.impl == "reference":
        run_reference(args, d)
        return
    if args.workload == "sweep":
        run_sweep(args)
        return
    if args.workload == "gpt-buckets":
        run_gpt_buckets(args)
        return
    if args.workload == "64x256MiB":
        run_64_ranks(args)
        return
    if args.workload == "kernels":
        run_kernels(args)
        return
    if args.workload == "overlap":
        run_overlap(args)
        return
    run_ours(args, d)


if __name__ == "__main__":
    main()
