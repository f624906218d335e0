"""Helpers for the GPU tests: move synthetic host arrays to and from CUDA
tensors (bf16 travels as its 16-bit patterns, fp16 as numpy float16) and
compare bit patterns."""
import numpy as np
import torch

TORCH = {np.dtype(np.float32): torch.float32, np.dtype(np.int32): torch.int32}


def to_dev(arrays, offsets=None, pad=0):
    """Upload host arrays as rank tensors.  With ``offsets``, rank r's tensor
    starts ``offsets[r]`` elements into its own padded allocation, which
    gives control over each pointer's alignment."""
    out = []
    for r, a in enumerate(arrays):
        if a.dtype == np.uint16:
            t = torch.from_numpy(a.view(np.int16))
            dt = torch.bfloat16
        else:
            t = torch.from_numpy(a)
            dt = None
        if offsets is not None:
            off = int(offsets[r])
            big = torch.zeros(a.size + off + pad, dtype=t.dtype, device="cuda")
            big[off:off + a.size].copy_(t.cuda())
            d = big[off:off + a.size]
        else:
            d = t.cuda()
        out.append(d.view(dt) if dt is not None else d)
    return out


def to_host(tensors):
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
