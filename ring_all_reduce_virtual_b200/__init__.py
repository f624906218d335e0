"""Ring all-reduce over N virtual ranks on one B200: the Python binding.

Each "virtual rank" is one CUDA tensor (one buffer in the GPU's HBM).  These
functions only marshal tensors, enums and the current stream into the C ABI
of ``librr_virtual.so`` (declared in ``include/rr.h``); every step of every
collective runs in that library's CUDA kernels.  If the library is missing,
the first call raises: there is no fallback.

Sources: [P4] "Collective communication primitives" (ai-infra-handbooks);
[P3] "Training gradient sync and collective communication" (geek-doc.cn);
[P1] "How all-reduce keeps every card identical" (mhpq.cn); [P2] "AllReduce
from principle to tuning" (xxqk.cn).  ``include/rr.h`` states each call's
semantics with its passage.
"""
from __future__ import annotations

import ctypes
from typing import Sequence

from ._lib import MAX_RANKS, Cost, RingEvent, RRError, Stats, check, lib

__all__ = [
    "all_reduce", "all_reduce_wire", "all_reduce_host", "all_reduce_host_noalloc", "ring_step", "ring_schedule", "reduce_scatter", "all_gather", "all_to_all",
    "RankSet", "BucketPlan", "GradSet", "Reducer", "cost_model", "pick_algo", "set_picker_params", "last_stats",
    "check_timeouts", "RRError",
    "OPS", "ALGOS", "MAX_RANKS",
]

OPS = {"sum": 0, "avg": 1, "max": 2, "min": 3, "prod": 4}
ALGOS = {"auto": 0, "ring": 1, "oneshot": 2, "tree": 3, "tree_oneshot": 4, "two_shot": 5, "double_ring": 6}
ALGO_NAMES = {v: k for k, v in ALGOS.items()}
PHASES = {"reduce_scatter": 0, "all_gather": 1}
_DTYPE_NAMES = {"f32": 0, "bf16": 1, "i32": 2, "f16": 3}


def _dtype_code(dtype) -> int:
    import torch

    codes = {torch.float32: 0, torch.bfloat16: 1, torch.int32: 2, torch.float16: 3}
    if isinstance(dtype, str):
        return _DTYPE_NAMES[dtype]
    if dtype not in codes:
        raise TypeError(f"unsupported dtype {dtype}; use float32, bfloat16, float16 or int32")
    return codes[dtype]


def _ptr_array(tensors: Sequence) -> ctypes.Array:
    arr = (ctypes.c_void_p * max(len(tensors), 1))()
    for i, t in enumerate(tensors):
        arr[i] = t.data_ptr()
    return arr


def _ranks(tensors: Sequence, what: str):
    """Check that the rank tensors are CUDA, contiguous and alike."""
    if len(tensors) < 1 or len(tensors) > MAX_RANKS:
        raise ValueError(f"{what}: need 1..{MAX_RANKS} rank tensors, got {len(tensors)}")
    t0 = tensors[0]
    for t in tensors:
        if not t.is_cuda:
            raise ValueError(f"{what}: rank tensors must be CUDA tensors")
        if not t.is_contiguous():
            raise ValueError(f"{what}: rank tensors must be contiguous")
        if t.dtype != t0.dtype or t.numel() != t0.numel() or t.device != t0.device:
            raise ValueError(f"{what}: rank tensors must share dtype, size and device")
    return t0.numel(), _dtype_code(t0.dtype), t0.device


class RankSet:
    """The N rank tensors of an all-reduce, checked and marshalled once.

    ``all_reduce``, ``all_reduce_wire`` and ``ring_step`` accept either this
    or a list of tensors.  A list is checked (CUDA, contiguous, same dtype,
    size and device) and its pointers copied into a ctypes array on every
    call, which costs several microseconds for 8 ranks -- as much as the
    kernel of a small message.  A RankSet does that once: it keeps the tensors
    alive and stays valid while they keep their storage (in-place updates are
    fine; ``resize_`` or ``set_`` on a member is not)."""

    def __init__(self, tensors: Sequence):
        self.count, self.dtype, self.device = _ranks(tensors, "RankSet")
        self.nranks = len(tensors)
        self.ptrs = _ptr_array(tensors)
        self.tensors = list(tensors)

    def __len__(self) -> int:
        return self.nranks

    def bind(self, op="sum", algo="auto", stream=None):
        """A callable that runs ``all_reduce(self, op, algo, stream)`` with
        every argument converted to its C type once, so each call costs one
        ctypes call: for small messages, repeated from Python, whose per-call
        host cost is otherwise several microseconds of argument handling."""
        f = lib().rr_allreduce
        args = (self.ptrs, ctypes.c_int(self.nranks), ctypes.c_size_t(self.count), ctypes.c_int(self.dtype),
                ctypes.c_int(_op(op)), ctypes.c_int(_algo(algo)), _stream(stream, self.device))

        def call() -> None:
            st = f(*args)
            if st:
                check(st, "all_reduce")
        return call


def _rank_args(tensors, what: str):
    """(pointer array, nranks, count, dtype code, device) of a list or a RankSet."""
    if isinstance(tensors, RankSet):
        return tensors.ptrs, tensors.nranks, tensors.count, tensors.dtype, tensors.device
    count, d, dev = _ranks(tensors, what)
    return _ptr_array(tensors), len(tensors), count, d, dev


def _stream(stream, device):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _op(op) -> int:
    return OPS[op] if isinstance(op, str) else int(op)


def _algo(algo) -> int:
    return ALGOS[algo] if isinstance(algo, str) else int(algo)


def all_reduce(tensors, op="sum", algo="auto", stream=None) -> None:
    """In-place all-reduce over the rank tensors, a list or a ``RankSet``
    (``rr_allreduce``)."""
    ptrs, n, count, d, dev = _rank_args(tensors, "all_reduce")
    check(lib().rr_allreduce(ptrs, n, count, d, _op(op), _algo(algo), _stream(stream, dev)), "all_reduce")


def all_reduce_wire(tensors, op="sum", wire="bf16", algo="auto", stream=None) -> None:
    """In-place all-reduce of fp32 rank tensors whose transfers are rounded
    to the bf16 wire format while the folds stay fp32 (``rr_allreduce_wire``)."""
    ptrs, n, count, d, dev = _rank_args(tensors, "all_reduce_wire")
    if d != _DTYPE_NAMES["f32"]:
        raise TypeError("all_reduce_wire: the rank tensors must be float32 (the wire format is bf16)")
    check(lib().rr_allreduce_wire(ptrs, n, count, _op(op), _dtype_code(wire), _algo(algo), _stream(stream, dev)),
          "all_reduce_wire")


def all_reduce_host(host: Sequence, device: Sequence, op="sum", algo="auto", stream=None) -> None:
    """All-reduce of host tensors through device staging tensors
    (``rr_allreduce_host``): copy in, reduce, copy back, all enqueued on
    ``stream``.  ``host`` should be pinned; it holds the result once the
    stream is synchronised."""
    count, d, dev = _ranks(device, "all_reduce_host")
    if len(host) != len(device):
        raise ValueError("all_reduce_host: one host tensor per device tensor")
    for h in host:
        if h.is_cuda or not h.is_contiguous() or h.numel() != count or _dtype_code(h.dtype) != d:
            raise ValueError("all_reduce_host: host tensors must be contiguous CPU tensors like the device ones")
    check(lib().rr_allreduce_host(_ptr_array(host), _ptr_array(device), len(device), count, d, _op(op),
                                  _algo(algo), _stream(stream, dev)), "all_reduce_host")


def all_reduce_host_noalloc(host: Sequence, op="sum", algo="auto", stream=None) -> None:
    """All-reduce of host tensors for callers that cannot allocate device
    memory (``rr_allreduce_host_noalloc``): the values are staged in the
    library's static device region (``RR_NOALLOC_MAX_BYTES`` in all), so the
    call allocates nothing.  ``host`` should be pinned; it holds the result
    once the stream is synchronised."""
    import torch

    if len(host) < 1 or len(host) > MAX_RANKS:
        raise ValueError(f"all_reduce_host_noalloc: need 1..{MAX_RANKS} host tensors")
    h0 = host[0]
    for h in host:
        if h.is_cuda or not h.is_contiguous() or h.numel() != h0.numel() or h.dtype != h0.dtype:
            raise ValueError("all_reduce_host_noalloc: host tensors must be contiguous CPU tensors alike")
    dev = torch.device("cuda", torch.cuda.current_device())
    check(lib().rr_allreduce_host_noalloc(_ptr_array(host), len(host), h0.numel(), _dtype_code(h0.dtype), _op(op),
                                          _algo(algo), _stream(stream, dev)), "all_reduce_host_noalloc")


def ring_step(tensors, op, phase, step: int, stream=None) -> None:
    """One ring step for all ranks at once (``rr_ring_step``)."""
    ptrs, n, count, d, dev = _rank_args(tensors, "ring_step")
    ph = PHASES[phase] if isinstance(phase, str) else int(phase)
    check(lib().rr_ring_step(ptrs, n, count, d, _op(op), ph, step, _stream(stream, dev)), "ring_step")


def ring_schedule(nranks: int, count: int, dtype="f32") -> list[dict]:
    """The ring schedule as a list of transfers (``rr_ring_schedule``)."""
    total = 2 * max(nranks - 1, 0) * nranks
    ev = (RingEvent * max(total, 1))()
    got = ctypes.c_size_t(0)
    check(lib().rr_ring_schedule(nranks, count, _dtype_code(dtype), ev, total, ctypes.byref(got)),
          "ring_schedule")
    return [{k: int(getattr(ev[i], k)) for k, _ in RingEvent._fields_} for i in range(got.value)]


def reduce_scatter(send: Sequence, recv: Sequence, op="sum", algo="auto", stream=None) -> None:
    """``recv[r]`` = part r of the reduction of all ``send`` (``rr_reduce_scatter``)."""
    count, d, dev = _ranks(send, "reduce_scatter")
    rcount, rd, rdev = _ranks(recv, "reduce_scatter")
    if len(recv) != len(send) or rd != d or rdev != dev or rcount * len(send) != count:
        raise ValueError("reduce_scatter: recv must be N tensors of count/N elements of the same dtype and device")
    check(lib().rr_reduce_scatter(_ptr_array(send), _ptr_array(recv), len(send), rcount, d, _op(op),
                                  _algo(algo), _stream(stream, dev)), "reduce_scatter")


def all_gather(send: Sequence, recv: Sequence, algo="auto", stream=None) -> None:
    """``recv[r]`` = concatenation of all ``send`` parts (``rr_all_gather``)."""
    scount, d, dev = _ranks(send, "all_gather")
    rcount, rd, rdev = _ranks(recv, "all_gather")
    if len(recv) != len(send) or rd != d or rdev != dev or rcount != scount * len(send):
        raise ValueError("all_gather: recv must be N tensors of N*count elements of the same dtype and device")
    check(lib().rr_all_gather(_ptr_array(send), _ptr_array(recv), len(send), scount, d, _algo(algo),
                              _stream(stream, dev)), "all_gather")


def all_to_all(send: Sequence, recv: Sequence, stream=None) -> None:
    """Block transpose across ranks (``rr_all_to_all``)."""
    count, d, dev = _ranks(send, "all_to_all")
    rcount, rd, rdev = _ranks(recv, "all_to_all")
    n = len(send)
    if len(recv) != n or rd != d or rdev != dev or rcount != count or count % n:
        raise ValueError("all_to_all: recv must match send (size, dtype, device), and N must divide the count")
    check(lib().rr_all_to_all(_ptr_array(send), _ptr_array(recv), n, count // n, d, _stream(stream, dev)),
          "all_to_all")


class GradSet:
    """The gradient tensors of all ranks (``grads[r][t]``), checked and with
    their device pointers marshalled once.  Bucket calls accept either this or
    the nested lists; a DDP step reuses the same gradient buffers every step,
    so building the pointer array once keeps the per-bucket host cost to a
    few microseconds.  Every rank must hold the same tensor sizes, all
    contiguous CUDA tensors of one dtype on one device."""

    def __init__(self, grads: Sequence[Sequence]):
        import weakref

        if not grads or not grads[0]:
            raise ValueError("GradSet: no gradients")
        first = grads[0][0]
        numels = [int(g.numel()) for g in grads[0]]
        for rank in grads:
            if len(rank) != len(numels):
                raise ValueError("GradSet: every rank needs the same number of tensors")
            for t, g in enumerate(rank):
                if not g.is_cuda or not g.is_contiguous() or g.device != first.device or g.dtype != first.dtype:
                    raise ValueError("GradSet: gradients must be contiguous CUDA tensors of one dtype and device")
                if g.numel() != numels[t]:
                    raise ValueError(f"GradSet: tensor {t} has different sizes on different ranks")
        self.nranks = len(grads)
        self.numels = numels
        self.dtype = _dtype_code(first.dtype)
        self.device = first.device
        self.ptrs = _ptr_array([g for rank in grads for g in rank])
        self._keep = [list(rank) for rank in grads]  # the tensors must outlive the pointers
        self._plans = weakref.WeakSet()  # plans this set was checked against


class BucketPlan:
    """DDP-style bucket plan over a list of gradient sizes (``rr_bucket_plan``)."""

    def __init__(self, numels: Sequence[int], grad_dtype="bf16", cap_bytes: int = 25 * (1 << 20)):
        arr = (ctypes.c_size_t * max(len(numels), 1))(*[int(m) for m in numels])
        handle = ctypes.c_void_p()
        check(lib().rr_bucket_plan(arr, len(numels), _dtype_code(grad_dtype), int(cap_bytes),
                                   ctypes.byref(handle)), "bucket_plan")
        self._h = handle
        self._free = lib().rr_bucket_plan_free  # held: module globals may be gone when __del__ runs at exit
        self.numels = [int(m) for m in numels]
        self.grad_dtype = _dtype_code(grad_dtype)

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            self._free(h)
            self._h = None

    @property
    def num_buckets(self) -> int:
        return int(lib().rr_bucket_count(self._h))

    def info(self, bucket: int) -> tuple[int, int, int]:
        """(first tensor, number of tensors, fp32 elements) of a bucket."""
        f, c, m = ctypes.c_int(), ctypes.c_int(), ctypes.c_size_t()
        check(lib().rr_bucket_info(self._h, bucket, ctypes.byref(f), ctypes.byref(c), ctypes.byref(m)),
              "bucket_info")
        return f.value, c.value, m.value

    def tensor(self, t: int) -> tuple[int, int]:
        """(bucket, element offset in it) of a tensor."""
        b, o = ctypes.c_int(), ctypes.c_size_t()
        check(lib().rr_bucket_tensor(self._h, t, ctypes.byref(b), ctypes.byref(o)), "bucket_tensor")
        return b.value, o.value

    def _grads(self, grads):
        """(pointers, nranks, device) of gradients that match this plan's
        tensor sizes and dtype (checked once per GradSet and plan)."""
        gs = grads if isinstance(grads, GradSet) else GradSet(grads)
        if self not in gs._plans:
            if gs.numels != self.numels or gs.dtype != self.grad_dtype:
                raise ValueError("gradients do not match the bucket plan (tensor count, sizes or dtype)")
            gs._plans.add(self)
        return gs.ptrs, gs.nranks, gs.device

    def _buckets(self, bucket: int, buckets: Sequence, n: int, device):
        """Pointer array of the fp32 bucket buffers, checked against the bucket's size."""
        numel = self.info(bucket)[2]
        if len(buckets) != n:
            raise ValueError("one fp32 bucket buffer per rank")
        for t in buckets:
            if (not t.is_cuda or not t.is_contiguous() or t.device != device or _dtype_code(t.dtype) != 0
                    or t.numel() < numel):
                raise ValueError(f"bucket buffers must be contiguous fp32 CUDA tensors of at least {numel} elements")
        return _ptr_array(buckets)

    def flat_buffers(self, nranks: int, device=None, dtype=None):
        """Gradients laid out as views into one flat buffer per bucket and
        rank (DDP's ``gradient_as_bucket_view``): returns ``(flats, grads)``
        with ``flats[b][r]`` the bucket's buffer on rank r and ``grads[r][t]``
        a view of tensor t inside it.  A bucket sync on this layout is
        ``all_reduce(flats[b], op, "oneshot")``, with the same bits as
        ``all_reduce(b, grads, op)`` and no gather or scatter at all.  (The
        buffers are allocated by PyTorch here, not by the library.)"""
        import torch

        dtype = dtype or torch.bfloat16
        flats, grads = [], [[None] * len(self.numels) for _ in range(nranks)]
        for b in range(self.num_buckets):
            first, cnt, numel = self.info(b)
            row = [torch.zeros(numel, dtype=dtype, device=device) for _ in range(nranks)]
            flats.append(row)
            for t in range(first, first + cnt):
                off = self.tensor(t)[1]
                for r in range(nranks):
                    grads[r][t] = row[r][off:off + self.numels[t]]
        return flats, grads

    def pack(self, bucket: int, grads: Sequence[Sequence], buckets: Sequence, stream=None) -> None:
        """``grads[r][t]`` -> fp32 ``buckets[r]`` for the bucket's tensors."""
        g, n, dev = self._grads(grads)
        check(lib().rr_bucket_pack(self._h, bucket, g, self._buckets(bucket, buckets, n, dev), n,
                                   _stream(stream, dev)), "bucket_pack")

    def unpack(self, bucket: int, buckets: Sequence, grads: Sequence[Sequence], op="avg", stream=None) -> None:
        """fp32 ``buckets[r]`` -> ``grads[r][t]`` (AVG divides by N)."""
        g, n, dev = self._grads(grads)
        check(lib().rr_bucket_unpack(self._h, bucket, self._buckets(bucket, buckets, n, dev), g, n, _op(op),
                                     _stream(stream, dev)), "bucket_unpack")

    def all_reduce(self, bucket: int, grads: Sequence[Sequence], op="avg", stream=None) -> None:
        """Fused pack + ring-order all-reduce + unpack, in place on ``grads``."""
        g, n, dev = self._grads(grads)
        check(lib().rr_bucket_allreduce(self._h, bucket, g, n, _op(op), _stream(stream, dev)),
              "bucket_allreduce")

    def all_reduce_range(self, first: int, count: int, grads: Sequence[Sequence], op="avg", stream=None) -> None:
        """Fused sync of buckets ``first .. first + count - 1`` in a few shared
        launches, with the bits of ``all_reduce`` on each of them
        (``rr_bucket_allreduce_range``)."""
        g, n, dev = self._grads(grads)
        check(lib().rr_bucket_allreduce_range(self._h, first, count, g, n, _op(op), _stream(stream, dev)),
              "bucket_allreduce_range")


class Reducer:
    """DDP-style overlapped bucket sync (``rr_reducer_*``): mark each
    gradient ready on the stream that produced it; every bucket's fused sync
    starts on ``comm`` as soon as its last gradient is ready; ``finish``
    joins the step.  Keep ``plan`` and the gradients alive while in use."""

    def __init__(self, plan: BucketPlan, grads, op="avg", comm=None, max_ctas: int = 0):
        import torch

        g = grads if isinstance(grads, GradSet) else GradSet(grads)
        plan._grads(g)  # the gradients must match the plan
        # a high-priority stream lets bucket syncs start as soon as SMs free up
        self.comm = comm if comm is not None else torch.cuda.Stream(g.device, priority=-1)
        self._plan, self._grads = plan, g
        handle = ctypes.c_void_p()
        check(lib().rr_reducer_create(plan._h, g.ptrs, g.nranks, _op(op), _stream(self.comm, g.device),
                                      int(max_ctas), ctypes.byref(handle)), "reducer_create")
        self._h = handle
        self._free = lib().rr_reducer_free  # held: module globals may be gone when __del__ runs at exit
        self._device = g.device

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            self._free(h)
            self._h = None

    def ready(self, tensor: int, stream=None) -> None:
        check(lib().rr_reducer_ready(self._h, tensor, _stream(stream, self._device)), "reducer_ready")

    def finish(self, stream=None) -> None:
        check(lib().rr_reducer_finish(self._h, _stream(stream, self._device)), "reducer_finish")


def cost_model(algo, nranks: int, bytes_per_rank: float, alpha_s: float, beta_bytes_per_s: float) -> dict:
    """The alpha-beta model terms (``rr_cost_model``)."""
    c = Cost()
    check(lib().rr_cost_model(_algo(algo), nranks, float(bytes_per_rank), float(alpha_s),
                              float(beta_bytes_per_s), ctypes.byref(c)), "cost_model")
    return {k: float(getattr(c, k)) for k, _ in Cost._fields_}


def pick_algo(nranks: int, count: int, dtype="f32") -> str:
    """The algorithm AUTO runs for this shape (``rr_pick_algo``)."""
    return ALGO_NAMES[int(lib().rr_pick_algo(nranks, count, _dtype_code(dtype)))]


def set_picker_params(launch_s: float, hbm_bytes_per_s: float) -> None:
    check(lib().rr_set_picker_params(float(launch_s), float(hbm_bytes_per_s)), "set_picker_params")


def last_stats() -> dict:
    """What the last call on this thread did (``rr_get_stats``)."""
    s = Stats()
    check(lib().rr_get_stats(ctypes.byref(s)), "get_stats")
    out = {k: int(getattr(s, k)) for k, _ in Stats._fields_}
    out["algo"] = ALGO_NAMES.get(out["algo"], out["algo"])
    return out


def check_timeouts() -> None:
    """Synchronise the device and raise ``RRError`` (status RR_ERR_TIMEOUT)
    if any bounded device wait ran out since the last check
    (``rr_check_timeouts``)."""
    check(lib().rr_check_timeouts(), "check_timeouts")
