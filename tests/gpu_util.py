"""Helpers for the GPU tests: move synthetic host arrays to and from CUDA
tensors (bf16 travels as its 16-bit patterns, fp16 as numpy float16) and
compare bit patterns."""
import weakref

import numpy as np
import torch

TORCH = {np.dtype(np.float32): torch.float32, np.dtype(np.int32): torch.int32}


GUARD = 64  # canary elements before and after every buffer to_dev makes
CANARY = 0xA5  # every canary byte
_guarded = weakref.WeakValueDictionary()  # data_ptr -> the rank tensor (a view into its guarded allocation)


def to_dev(arrays, offsets=None, pad=0):
    """Upload host arrays as rank tensors.  With ``offsets``, rank r's tensor
    starts ``offsets[r]`` elements past a 16-byte boundary, which gives
    control over each pointer's alignment.  Every tensor sits inside its own
    allocation between canary regions (GUARD elements of CANARY bytes before
    it, and after it plus ``pad``), which ``to_host`` checks: a kernel that
    writes outside the buffers it was given fails the test that read back."""
    out = []
    for r, a in enumerate(arrays):
        if a.dtype == np.uint16:
            t = torch.from_numpy(a.view(np.int16))
            dt = torch.bfloat16
        else:
            t = torch.from_numpy(a)
            dt = None
        off = GUARD + (int(offsets[r]) if offsets is not None else 0)
        big = torch.empty(off + a.size + pad + GUARD, dtype=t.dtype, device="cuda")
        big.view(torch.uint8).fill_(CANARY)
        d = big[off:off + a.size]
        d.copy_(t.cuda())
        d = d.view(dt) if dt is not None else d
        _guarded[d.data_ptr()] = d
        out.append(d)
    return out


def check_guards(tensors):
    """Every canary byte around the given to_dev tensors is intact."""
    for t in tensors:
        d = _guarded.get(t.data_ptr())
        if d is None or d is not t and d.numel() != t.numel():
            continue
        base = d._base if d._base is not None else d
        raw = base.view(torch.uint8)
        es = d.element_size()
        lo = (d.data_ptr() - base.data_ptr())
        hi = lo + d.numel() * es
        before, after = raw[:lo], raw[hi:]
        if not (bool(torch.all(before == CANARY)) and bool(torch.all(after == CANARY))):
            raise AssertionError("a kernel wrote outside its buffer: the guard canaries around it changed")


def to_host(tensors):
    check_guards(tensors)
    res = []
    for t in tensors:
        if t.dtype == torch.bfloat16:
            res.append(t.view(torch.int16).cpu().numpy().view(np.uint16))
        else:
            res.append(t.cpu().numpy())
    return res


def bits(a):
    a = np.ascontiguousarray(a)
    return a.view(np.uint16) if a.dtype in (np.uint16, np.float16) else a.view(np.uint32)


def assert_bits_equal(got, want, what=""):
    for r, (g, w) in enumerate(zip(got, want)):
        gb, wb = bits(g), bits(w)
        if not np.array_equal(gb, wb):
            bad = np.nonzero(gb != wb)[0]
            raise AssertionError(f"{what} rank {r}: {bad.size} elements differ, first at {bad[:5]}: "
                                 f"got {g[bad[:5]]} want {w[bad[:5]]}")


def empty_like_ranks(n, count, dtype):
    if dtype == "bf16":
        return [torch.empty(count, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    td = {"f32": torch.float32, "f16": torch.float16, "i32": torch.int32}[dtype]
    return [torch.empty(count, dtype=td, device="cuda") for _ in range(n)]
