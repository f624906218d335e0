"""ctypes loader for ``librr_virtual.so`` (the C ABI in ``include/rr.h``).

Loading fails loudly when the library has not been built: there is no
fallback path of any kind.
"""
from __future__ import annotations

import ctypes
import os
import threading

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librr_virtual.so")

RR_OK, RR_ERR_INVALID_ARG, RR_ERR_UNSUPPORTED, RR_ERR_CUDA, RR_ERR_TIMEOUT = 0, 1, 2, 3, 4
MAX_RANKS = 64


class RRError(RuntimeError):
    """A call returned a status other than RR_OK."""

    def __init__(self, status: int, what: str, detail: str):
        self.status = status
        super().__init__(f"{what}: {detail or 'status ' + str(status)} (status {status})")


class Stats(ctypes.Structure):
    _fields_ = [
        ("algo", ctypes.c_int32), ("steps", ctypes.c_int32), ("launches", ctypes.c_int32),
        ("nranks", ctypes.c_int32), ("bytes_per_rank", ctypes.c_uint64), ("bytes_sent_max", ctypes.c_uint64),
        ("bytes_sent_total", ctypes.c_uint64), ("hbm_bytes", ctypes.c_uint64), ("host_ns", ctypes.c_uint64),
        ("launch_ns", ctypes.c_uint64),
    ]


class RingEvent(ctypes.Structure):
    _fields_ = [
        ("phase", ctypes.c_int32), ("step", ctypes.c_int32), ("rank", ctypes.c_int32), ("dst", ctypes.c_int32),
        ("send_idx", ctypes.c_int32), ("recv_idx", ctypes.c_int32), ("bytes", ctypes.c_uint64),
    ]


class Cost(ctypes.Structure):
    _fields_ = [
        ("steps", ctypes.c_double), ("bytes_sent", ctypes.c_double), ("latency_s", ctypes.c_double),
        ("bandwidth_s", ctypes.c_double), ("total_s", ctypes.c_double),
    ]


_lock = threading.Lock()
_lib: ctypes.CDLL | None = None


def _declare(lib: ctypes.CDLL) -> None:
    P, PP = ctypes.c_void_p, ctypes.POINTER(ctypes.c_void_p)
    i, sz, d = ctypes.c_int, ctypes.c_size_t, ctypes.c_double
    st = ctypes.c_int
    sig = {
        "rr_allreduce": (st, [PP, i, sz, i, i, i, P]),
        "rr_allreduce_host": (st, [PP, PP, i, sz, i, i, i, P]),
        "rr_allreduce_host_noalloc": (st, [PP, i, sz, i, i, i, P]),
        "rr_allreduce_wire": (st, [PP, i, sz, i, i, i, P]),
        "rr_ring_step": (st, [PP, i, sz, i, i, i, i, P]),
        "rr_ring_schedule": (st, [i, sz, i, ctypes.POINTER(RingEvent), sz, ctypes.POINTER(sz)]),
        "rr_reduce_scatter": (st, [PP, PP, i, sz, i, i, i, P]),
        "rr_all_gather": (st, [PP, PP, i, sz, i, i, P]),
        "rr_all_to_all": (st, [PP, PP, i, sz, i, P]),
        "rr_bucket_plan": (st, [ctypes.POINTER(sz), i, i, sz, ctypes.POINTER(P)]),
        "rr_bucket_plan_free": (None, [P]),
        "rr_bucket_count": (i, [P]),
        "rr_bucket_info": (st, [P, i, ctypes.POINTER(i), ctypes.POINTER(i), ctypes.POINTER(sz)]),
        "rr_bucket_tensor": (st, [P, i, ctypes.POINTER(i), ctypes.POINTER(sz)]),
        "rr_bucket_pack": (st, [P, i, PP, PP, i, P]),
        "rr_bucket_unpack": (st, [P, i, PP, PP, i, i, P]),
        "rr_bucket_allreduce": (st, [P, i, PP, i, i, P]),
        "rr_bucket_allreduce_range": (st, [P, i, i, PP, i, i, P]),
        "rr_reducer_create": (st, [P, PP, i, i, P, i, ctypes.POINTER(P)]),
        "rr_reducer_ready": (st, [P, i, P]),
        "rr_reducer_finish": (st, [P, P]),
        "rr_reducer_free": (None, [P]),
        "rr_cost_model": (st, [i, i, d, d, d, ctypes.POINTER(Cost)]),
        "rr_pick_algo": (i, [i, sz, i]),
        "rr_set_picker_params": (st, [d, d]),
        "rr_get_stats": (st, [ctypes.POINTER(Stats)]),
        "rr_check_timeouts": (st, []),
        "rr_status_string": (ctypes.c_char_p, [i]),
        "rr_last_error": (ctypes.c_char_p, []),
        "rr_version": (i, []),
        "rr_binary_version": (st, [ctypes.POINTER(i)]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args


def lib() -> ctypes.CDLL:
    """The loaded library (loaded on first use)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"the CUDA library {LIB_PATH} is not built; run "
                    "`python -m ring_all_reduce_virtual_b200.build` (this package has no other path)")
            handle = ctypes.CDLL(LIB_PATH)
            _declare(handle)
            _lib = handle
        return _lib


def check(status: int, what: str) -> None:
    if status != RR_OK:
        detail = lib().rr_last_error().decode(errors="replace")
        raise RRError(status, what, detail)
