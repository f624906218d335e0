"""The host all-reduce for callers that cannot allocate device memory.

``rr_allreduce_host_noalloc`` serves callers that hold only host arrays and
a stream and may not call cudaMalloc -- a framework's caching allocator holds
all of the device's memory, a plug-in is handed no device buffers, or a
latency-critical path must not call cudaMalloc / cudaFree, which can
synchronise the device.  It stages the values in the library's static device
region instead of the caller's device buffers.  Here it is called through
the C ABI (ctypes) and must give the bits of ``rr_allreduce_host``, which
stages through device buffers the test allocates, on two calls in a row
whose ranks, sizes, dtypes and ops differ (so the second call cannot lean on
values the first left in the shared region); a call beyond the region's
size is refused before anything is enqueued.

This file is collected last, so a run that stops at the first failure has
run every other test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

from ring_all_reduce_virtual_b200 import _lib, synth

pytestmark = pytest.mark.gpu

F32, BF16 = 0, 1
OPS = {"sum": 0, "avg": 1, "max": 2}
ONESHOT = 2
MAX_BYTES = 16 << 20  # RR_NOALLOC_MAX_BYTES


def _ptrs(tensors):
    return (ctypes.c_void_p * len(tensors))(*[t.data_ptr() for t in tensors])


def _pinned(arrays):
    out = []
    for a in arrays:
        t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).clone().pin_memory()
        out.append(t)
    return out


def _bits(t):
    a = t.numpy()
    return a.view(np.uint16) if a.itemsize == 2 else a.view(np.uint32)


def _both(n, count, dtype, op, seed):
    lib = _lib.lib()
    stream = torch.cuda.current_stream()
    code = F32 if dtype == "f32" else BF16
    x = synth.ranks(seed, n, count, "uniform", dtype)
    # the existing entry point, through device buffers allocated here
    ref = _pinned(x)
    dev = [torch.empty(count, dtype=torch.float32 if dtype == "f32" else torch.int16, device="cuda")
           for _ in range(n)]
    _lib.check(lib.rr_allreduce_host(_ptrs(ref), _ptrs(dev), n, count, code, OPS[op], ONESHOT,
                                     ctypes.c_void_p(stream.cuda_stream)), "rr_allreduce_host")
    # the no-allocation entry point
    got = _pinned(x)
    _lib.check(lib.rr_allreduce_host_noalloc(_ptrs(got), n, count, code, OPS[op], ONESHOT,
                                             ctypes.c_void_p(stream.cuda_stream)), "rr_allreduce_host_noalloc")
    torch.cuda.synchronize()
    for r in range(n):
        assert np.array_equal(_bits(got[r]), _bits(ref[r])), f"rank {r} differs from rr_allreduce_host"
        assert np.array_equal(_bits(got[r]), _bits(got[0])), f"rank {r} differs from rank 0"
    # the call did reduce (the inputs were not all equal)
    assert not np.array_equal(_bits(got[0]), _bits(_pinned([x[0]])[0]))


def test_no_alloc_host_allreduce_matches_the_device_buffer_entry_point():
    # call 1: 8 ranks, ragged chunks, fp32 AVG; call 2: fewer ranks and
    # elements, bf16 SUM, over the region the first call left behind
    _both(8, 8 * 4096 + 5, "f32", "avg", seed=90)
    _both(3, 3 * 1000 + 1, "bf16", "sum", seed=91)
    # the region's full size: 4 ranks x 4 MiB fp32
    _both(4, MAX_BYTES // 16, "f32", "max", seed=92)


def test_no_alloc_host_allreduce_refuses_more_than_the_region():
    lib = _lib.lib()
    n = 8
    count = MAX_BYTES // 4 // n + 1  # one element too many
    host = [torch.zeros(count, dtype=torch.float32) for _ in range(n)]
    st = lib.rr_allreduce_host_noalloc(_ptrs(host), n, count, F32, OPS["sum"], ONESHOT,
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == _lib.RR_ERR_INVALID_ARG
    assert b"RR_NOALLOC_MAX_BYTES" in lib.rr_last_error()
