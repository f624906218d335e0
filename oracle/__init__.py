"""Python face of the CPU oracle (``rr_oracle.c``), via ctypes and numpy.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  It shares
no code with the CUDA library and never imports it.

Buffers are numpy arrays, one per virtual rank: ``float32`` for fp32,
``uint16`` bit patterns for bf16, ``float16`` for fp16, ``int32`` for int32.
Functions that the C file defines "in place" modify the arrays given to them.
Each function's docstring names the passage of the pages it follows; the C
file has the full statements and the readings taken where the pages are
silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))

F32, BF16, I32, F16 = 0, 1, 2, 3
SUM, AVG, MAX, MIN, PROD = 0, 1, 2, 3, 4
PHASE_RS, PHASE_AG = 0, 1
OPS = {"sum": SUM, "avg": AVG, "max": MAX, "min": MIN, "prod": PROD}


class Event(ctypes.Structure):
    """One record of the ring schedule: who sent which chunk to whom."""

    _fields_ = [
        ("phase", ctypes.c_int32),
        ("step", ctypes.c_int32),
        ("rank", ctypes.c_int32),
        ("dst", ctypes.c_int32),
        ("send_idx", ctypes.c_int32),
        ("recv_idx", ctypes.c_int32),
        ("bytes", ctypes.c_uint64),
    ]


_lock = threading.Lock()
_libs: dict[bool, ctypes.CDLL] = {}


def build(force: bool = False) -> None:
    """Compile the oracle (and its mutant twin) with the Makefile beside it."""
    args = ["make", "-s", "-C", _HERE]
    if force:
        args.append("-B")
    subprocess.run(args, check=True)


def _load(mutant: bool = False) -> ctypes.CDLL:
    with _lock:
        if mutant in _libs:
            return _libs[mutant]
        name = "liboracle_mut.so" if mutant else "liboracle.so"
        path = os.path.join(_HERE, name)
        src = os.path.join(_HERE, "rr_oracle.c")
        if not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(src):
            build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        PP = ctypes.POINTER(ctypes.c_void_p)
        i32, sz = ctypes.c_int, ctypes.c_size_t
        lib.orc_ring_step.argtypes = [PP, i32, sz, i32, i32, i32, i32, ctypes.POINTER(Event)]
        lib.orc_ring_allreduce.argtypes = [PP, i32, sz, i32, i32, ctypes.POINTER(Event), P]
        lib.orc_ring_allreduce_omp.argtypes = [PP, i32, sz, i32, i32, i32]
        lib.orc_fold_ring_order.argtypes = [PP, i32, sz, i32, i32]
        lib.orc_ring_allreduce_wire.argtypes = [PP, i32, sz, i32]
        lib.orc_fold_wire.argtypes = [PP, i32, sz, i32]
        lib.orc_double_ring_step.argtypes = [PP, i32, sz, i32, i32, i32, i32, P]
        lib.orc_double_ring_allreduce.argtypes = [PP, i32, sz, i32, i32, P]
        lib.orc_fold_double_ring.argtypes = [PP, i32, sz, i32, i32]
        lib.orc_fold_samples.argtypes = [P, i32, sz, P, i32, i32, P]
        lib.orc_naive_allreduce.argtypes = [PP, i32, sz, i32, i32, P]
        lib.orc_tree_schedule.argtypes = [PP, i32, sz, i32, i32, P]
        lib.orc_tree_fold.argtypes = [PP, i32, sz, i32, i32]
        lib.orc_reduce_scatter.argtypes = [PP, PP, i32, sz, i32, i32]
        lib.orc_all_gather.argtypes = [PP, PP, i32, sz, i32]
        lib.orc_all_to_all.argtypes = [PP, PP, i32, sz, i32]
        lib.orc_bucket_plan.argtypes = [P, i32, ctypes.c_uint64, ctypes.c_uint64, P, P, P]
        lib.orc_bucket_pack.argtypes = [PP, P, P, P, i32, i32, i32, P]
        lib.orc_bucket_unpack.argtypes = [PP, P, P, P, i32, i32, i32, P, i32, i32]
        lib.orc_f32_to_bf16_array.argtypes = [P, P, sz]
        lib.orc_bf16_to_f32_array.argtypes = [P, P, sz]
        lib.orc_f32_to_f16_array.argtypes = [P, P, sz]
        lib.orc_f16_to_f32_array.argtypes = [P, P, sz]
        lib.orc_chunk_size.argtypes = [sz, i32]
        lib.orc_chunk_size.restype = sz
        lib.orc_chunk_len.argtypes = [sz, i32, i32]
        lib.orc_chunk_len.restype = sz
        if mutant:
            lib.orc_set_mutant.argtypes = [i32]
        _libs[mutant] = lib
        return lib


class _Mutant:
    """Context manager that switches on one planted mistake (tests only)."""

    def __init__(self, kind: int):
        self.kind = kind

    def __enter__(self):
        _load(True).orc_set_mutant(self.kind)
        _state.mutant = True
        return self

    def __exit__(self, *exc):
        _load(True).orc_set_mutant(0)
        _state.mutant = False
        return False


class _State(threading.local):
    mutant = False


_state = _State()


def mutant(kind: int) -> _Mutant:
    """Run the oracle with planted mistake ``kind`` (see rr_oracle.c)."""
    return _Mutant(kind)


def _lib() -> ctypes.CDLL:
    return _load(_state.mutant)


# --------------------------------------------------------------- helpers --

def dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.int32:
        return I32
    if a.dtype == np.float16:
        return F16
    raise TypeError(f"oracle buffers are float32, uint16 (bf16 bits), float16 or int32, not {a.dtype}")


def _op(op) -> int:
    return OPS[op] if isinstance(op, str) else int(op)


def _ptrs(bufs) -> ctypes.Array:
    arr = (ctypes.c_void_p * max(len(bufs), 1))()
    for i, b in enumerate(bufs):
        if not (isinstance(b, np.ndarray) and b.flags.c_contiguous):
            raise TypeError("oracle buffers must be C-contiguous numpy arrays")
        arr[i] = b.ctypes.data
    return arr


def _same(bufs) -> tuple[int, int]:
    if not bufs:
        raise ValueError("need at least one rank")
    d = dtype_code(bufs[0])
    n0 = bufs[0].size
    for b in bufs:
        if dtype_code(b) != d or b.size != n0:
            raise ValueError("all ranks need the same dtype and size")
    return d, n0


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


def chunk_size(count: int, n: int) -> int:
    """C = ceil(count / N) ([P4] ring_allreduce.py splits with tensor.chunk)."""
    return int(_lib().orc_chunk_size(count, n))


def chunk_len(count: int, n: int, k: int) -> int:
    return int(_lib().orc_chunk_len(count, n, k))


# ----------------------------------------------------------- collectives --

def ring_step(bufs, op, phase: int, step: int):
    """One ring step for all ranks at once, in place; returns N events.

    [P4] "Ring all-reduce and communication volume"; [P3] section 3."""
    d, count = _same(bufs)
    n = len(bufs)
    ev = (Event * n)()
    _check(_lib().orc_ring_step(_ptrs(bufs), n, count, d, _op(op), phase, step, ev), "ring_step")
    return [_event_dict(e) for e in ev]


def _event_dict(e: Event) -> dict:
    return {k: int(getattr(e, k)) for k, _ in Event._fields_}


def ring_allreduce(bufs, op="sum", trace: bool = False):
    """The ring all-reduce, in place: N-1 reduce-scatter then N-1 all-gather
    steps.  Returns the bytes each rank sent (and the schedule if asked).

    [P4] "Ring all-reduce and communication volume"; [P3] sections 3-4."""
    d, count = _same(bufs)
    n = len(bufs)
    sent = np.zeros(n, dtype=np.uint64)
    nev = 2 * (n - 1) * n
    ev = (Event * max(nev, 1))() if trace else None
    _check(_lib().orc_ring_allreduce(_ptrs(bufs), n, count, d, _op(op), ev, sent.ctypes.data), "ring")
    if trace:
        return sent, [_event_dict(ev[i]) for i in range(nev)]
    return sent


def ring_allreduce_omp(bufs, op="sum", nthreads: int = 0) -> None:
    """The ring with each step's N transfers on several host threads (the
    timed CPU baseline); same arithmetic as ``ring_allreduce``."""
    d, count = _same(bufs)
    _check(_lib().orc_ring_allreduce_omp(_ptrs(bufs), len(bufs), count, d, _op(op), nthreads), "ring_omp")


def ring_allreduce_wire(bufs, op="sum") -> None:
    """The ring all-reduce of fp32 buffers with every transfer rounded to
    bf16 and fp32 folds, in place ([P1] s7.3: low-precision gradients on the
    wire)."""
    d, count = _same(bufs)
    if d != F32:
        raise TypeError("the bf16 wire carries fp32 buffers")
    _check(_lib().orc_ring_allreduce_wire(_ptrs(bufs), len(bufs), count, _op(op)), "ring wire")


def fold_wire(bufs, op="sum") -> None:
    """The bf16-wire all-reduce by definition (its fused one-shot form)."""
    d, count = _same(bufs)
    if d != F32:
        raise TypeError("the bf16 wire carries fp32 buffers")
    _check(_lib().orc_fold_wire(_ptrs(bufs), len(bufs), count, _op(op)), "fold wire")


def double_ring_allreduce(bufs, op="sum"):
    """The double ring ([P3] section 6): half A on the clockwise ring, half B
    on the counter-clockwise ring, in place; returns the bytes each rank
    sent."""
    d, count = _same(bufs)
    n = len(bufs)
    sent = np.zeros(n, dtype=np.uint64)
    _check(_lib().orc_double_ring_allreduce(_ptrs(bufs), n, count, d, _op(op), sent.ctypes.data), "double ring")
    return sent


def double_ring_step(bufs, op, phase: int, step: int):
    """One step of both rings, in place; returns the bytes each rank sent."""
    d, count = _same(bufs)
    n = len(bufs)
    sent = np.zeros(n, dtype=np.uint64)
    _check(_lib().orc_double_ring_step(_ptrs(bufs), n, count, d, _op(op), phase, step, sent.ctypes.data),
           "double ring step")
    return sent


def fold_double_ring(bufs, op="sum") -> None:
    """The double ring's result by definition (half B folds downwards),
    folded in fp32 and rounded once, in place."""
    d, count = _same(bufs)
    _check(_lib().orc_fold_double_ring(_ptrs(bufs), len(bufs), count, d, _op(op)), "fold double ring")


def fold_ring_order(bufs, op="sum") -> None:
    """One-shot all-reduce by its definition (ring-order fold), in place.

    [P4] "alpha-beta model" (one-shot: read every rank's buffer directly)."""
    d, count = _same(bufs)
    _check(_lib().orc_fold_ring_order(_ptrs(bufs), len(bufs), count, d, _op(op)), "fold")


def fold_samples(vals: np.ndarray, start: np.ndarray, op="sum") -> np.ndarray:
    """Ring-order fold of sampled elements: ``vals`` is [N, m] (one row per
    rank), ``start`` the chunk index (fold start rank) of each column."""
    vals = np.ascontiguousarray(vals)
    n, m = vals.shape
    start = np.ascontiguousarray(start, dtype=np.int32)
    out = np.empty(m, dtype=vals.dtype)
    _check(_lib().orc_fold_samples(vals.ctypes.data, n, m, start.ctypes.data, dtype_code(vals),
                                   _op(op), out.ctypes.data), "fold_samples")
    return out


def naive_allreduce(bufs, op="sum") -> np.ndarray:
    """Naive all-gather then local reduce in rank order, in place; returns
    the bytes each rank sent ([P1] s2.1, s3.1, s3.3)."""
    d, count = _same(bufs)
    n = len(bufs)
    sent = np.zeros(n, dtype=np.uint64)
    _check(_lib().orc_naive_allreduce(_ptrs(bufs), n, count, d, _op(op), sent.ctypes.data), "naive")
    return sent


def tree_schedule(bufs, op="sum") -> int:
    """Tree reduce then broadcast, level by level, in place; returns the
    number of steps ([P3] section 6)."""
    d, count = _same(bufs)
    steps = ctypes.c_int(0)
    _check(_lib().orc_tree_schedule(_ptrs(bufs), len(bufs), count, d, _op(op), ctypes.addressof(steps)),
           "tree")
    return steps.value


def tree_fold(bufs, op="sum") -> None:
    """Tree-order result folded in fp32 and rounded once, in place."""
    d, count = _same(bufs)
    _check(_lib().orc_tree_fold(_ptrs(bufs), len(bufs), count, d, _op(op)), "tree_fold")


def reduce_scatter(send, op="sum"):
    """Reduce-scatter; returns N arrays of count/N elements ([P4] "The five
    primitives")."""
    d, count = _same(send)
    n = len(send)
    if count % n:
        raise ValueError("reduce-scatter needs count divisible by N")
    recv = [np.empty(count // n, dtype=send[0].dtype) for _ in range(n)]
    _check(_lib().orc_reduce_scatter(_ptrs(send), _ptrs(recv), n, count // n, d, _op(op)), "rs")
    return recv


def all_gather(send):
    """All-gather; returns N arrays of N*count elements ([P4] "The five
    primitives")."""
    d, count = _same(send)
    n = len(send)
    recv = [np.empty(count * n, dtype=send[0].dtype) for _ in range(n)]
    _check(_lib().orc_all_gather(_ptrs(send), _ptrs(recv), n, count, d), "ag")
    return recv


def all_to_all(send):
    """All-to-all (a transpose of rank blocks); returns N arrays ([P4] "The
    five primitives")."""
    d, count = _same(send)
    n = len(send)
    if count % n:
        raise ValueError("all-to-all needs count divisible by N")
    recv = [np.empty(count, dtype=send[0].dtype) for _ in range(n)]
    _check(_lib().orc_all_to_all(_ptrs(send), _ptrs(recv), n, count // n, d), "a2a")
    return recv


# --------------------------------------------------------------- buckets --

def bucket_plan(numels, elem_bytes: int, cap_bytes: int):
    """Greedy bucket plan ([P2] s3.3; [P1] s5.2).  Returns (bucket_of,
    offset_of, nbuckets)."""
    numels = np.ascontiguousarray(numels, dtype=np.uint64)
    nt = numels.size
    bucket_of = np.zeros(max(nt, 1), dtype=np.int32)
    offset_of = np.zeros(max(nt, 1), dtype=np.uint64)
    nb = ctypes.c_int32(0)
    _check(_lib().orc_bucket_plan(numels.ctypes.data, nt, elem_bytes, cap_bytes, bucket_of.ctypes.data,
                                  offset_of.ctypes.data, ctypes.addressof(nb)), "bucket_plan")
    return bucket_of[:nt], offset_of[:nt], nb.value


def bucket_pack(grads, numels, bucket_of, offset_of, bucket: int, bucket_numel: int) -> np.ndarray:
    """Pack one rank's gradients of one bucket into an fp32 bucket."""
    numels = np.ascontiguousarray(numels, dtype=np.uint64)
    out = np.zeros(bucket_numel, dtype=np.float32)
    d = dtype_code(grads[0])
    _check(_lib().orc_bucket_pack(_ptrs(grads), numels.ctypes.data, bucket_of.ctypes.data,
                                  offset_of.ctypes.data, len(grads), bucket, d, out.ctypes.data), "pack")
    return out


def bucket_unpack(grads, numels, bucket_of, offset_of, bucket: int, data: np.ndarray, n: int, op="avg"):
    """Unpack one rank's reduced fp32 bucket into its gradients, in place."""
    numels = np.ascontiguousarray(numels, dtype=np.uint64)
    data = np.ascontiguousarray(data, dtype=np.float32)
    d = dtype_code(grads[0])
    _check(_lib().orc_bucket_unpack(_ptrs(grads), numels.ctypes.data, bucket_of.ctypes.data,
                                    offset_of.ctypes.data, len(grads), bucket, d, data.ctypes.data, n,
                                    _op(op)), "unpack")


def bucket_sync(grads_per_rank, cap_bytes: int, op="avg") -> None:
    """The whole bucketed gradient sync, in place on every rank's gradient
    list: plan, then per bucket pack -> ring-order SUM fold in fp32 ->
    unpack with AVG's division and one rounding ([P1] s5.1-5.3; [P2] s3.3)."""
    n = len(grads_per_rank)
    numels = np.array([g.size for g in grads_per_rank[0]], dtype=np.uint64)
    es = grads_per_rank[0][0].itemsize
    bucket_of, offset_of, nb = bucket_plan(numels, es, cap_bytes)
    for b in range(nb):
        members = np.nonzero(bucket_of == b)[0]
        numel = int(sum(int(numels[t]) for t in members))
        packed = [bucket_pack(g, numels, bucket_of, offset_of, b, numel) for g in grads_per_rank]
        fold_ring_order(packed, SUM)
        for r in range(n):
            bucket_unpack(grads_per_rank[r], numels, bucket_of, offset_of, b, packed[r], n, op)


# ------------------------------------------------------------------ bf16 --

def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (IEEE 754)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _lib().orc_f32_to_bf16_array(x.ctypes.data, out.ctypes.data, x.size)
    return out


def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32 (exact)."""
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, dtype=np.float32)
    _lib().orc_bf16_to_f32_array(h.ctypes.data, out.ctypes.data, h.size)
    return out


# ------------------------------------------------------------------ fp16 --
# fp16 rank buffers are numpy float16 arrays; the oracle reads and writes
# their bit patterns with its own conversions (IEEE 754 binary16, round to
# nearest even), not numpy's.

def f32_to_f16(x: np.ndarray) -> np.ndarray:
    """fp32 -> fp16 (as float16 whose bits the oracle computed), round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _lib().orc_f32_to_f16_array(x.ctypes.data, out.ctypes.data, x.size)
    return out.view(np.float16)


def f16_to_f32(h: np.ndarray) -> np.ndarray:
    """fp16 -> fp32 (exact), by the oracle's own widening of the bit patterns."""
    h = np.ascontiguousarray(h).view(np.uint16)
    out = np.empty(h.shape, dtype=np.float32)
    _lib().orc_f16_to_f32_array(h.ctypes.data, out.ctypes.data, h.size)
    return out
