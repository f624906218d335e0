"""Seeded synthetic inputs for the virtual ranks.

This module only draws numbers and describes workloads; it holds none of the
collectives' arithmetic.  The test suite, the benchmark and the smoke check
use it to feed the same host arrays to the CUDA library and to the CPU
oracle.

Every rank's values come from ``numpy.random.default_rng([seed, rank])`` (or
``[seed, rank, tensor]`` for gradient sets), so any rank can be regenerated on
its own.  Arrays are host ``numpy`` arrays: ``float32``, ``int32``, or
``uint16`` holding bf16 bit patterns (numpy has no bf16 type; the rounding of
drawn fp32 values to bf16 is done by PyTorch's CPU conversion).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

#: value distributions of the workloads
DISTS = ("uniform", "full", "normal", "prod", "int", "arange", "pow2")


def rank_values(seed: int, rank: int, count: int, dist: str = "uniform", dtype: str = "f32",
                stream: int | None = None) -> np.ndarray:
    """Draw ``count`` values for one rank.

    dist:
      - ``uniform``: uniform on [-1, 1) (numpy's float32 draws: multiples of
        2^-23, so a sum of two is always exact)
      - ``full``: uniform on [-1, 1) drawn in float64 and rounded to float32,
        so every value has a full 24-bit mantissa and short sums round: each
        fold order gives its own bits
      - ``normal``: normal(0, 1e-3)
      - ``prod``: uniform on [0.99, 1.01) (keeps long products finite)
      - ``int``: integers in [-1024, 1024), exact in fp32 and bf16 sums of a
        few ranks
      - ``arange``: ``arange(count) + 10 * rank`` (the 4-rank worked example)
      - ``pow2``: ``2 ** rank`` everywhere (shows which ranks were summed)
    dtype: ``f32``, ``bf16`` (returned as uint16 bits), ``f16`` (float16) or
      ``i32``.
    """
    key = [seed, rank] if stream is None else [seed, rank, stream]
    rng = np.random.default_rng(key)
    if dist == "uniform":
        v = rng.random(count, dtype=np.float32) * np.float32(2.0) - np.float32(1.0)
    elif dist == "full":
        v = (rng.random(count) * 2.0 - 1.0).astype(np.float32)
    elif dist == "normal":
        v = rng.standard_normal(count, dtype=np.float32) * np.float32(1e-3)
    elif dist == "prod":
        v = np.float32(0.99) + rng.random(count, dtype=np.float32) * np.float32(0.02)
    elif dist == "int":
        v = rng.integers(-1024, 1024, size=count, dtype=np.int32)
    elif dist == "arange":
        v = np.arange(count, dtype=np.int64) + 10 * rank
    elif dist == "pow2":
        v = np.full(count, 2 ** rank, dtype=np.int64)
    else:
        raise ValueError(f"unknown distribution {dist!r}")
    return cast(v, dtype)


def cast(v: np.ndarray, dtype: str) -> np.ndarray:
    """Cast drawn values to the buffer dtype (bf16 as uint16 bit patterns,
    fp16 as float16), rounding with PyTorch's CPU conversion."""
    if dtype == "f32":
        return np.ascontiguousarray(v, dtype=np.float32)
    if dtype == "i32":
        return np.ascontiguousarray(v, dtype=np.int32)
    if dtype == "bf16":
        import torch

        t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).to(torch.bfloat16)
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    if dtype == "f16":
        import torch

        return torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).to(torch.float16).numpy().copy()
    raise ValueError(f"unknown dtype {dtype!r}")


def ranks(seed: int, n: int, count: int, dist: str = "uniform", dtype: str = "f32") -> list[np.ndarray]:
    """One array per rank, ``n`` ranks."""
    return [rank_values(seed, r, count, dist, dtype) for r in range(n)]


# ------------------------------------------------------------ workloads --

@dataclass(frozen=True)
class Workload:
    name: str
    nranks: int
    count: int
    dtype: str
    dist: str
    ops: tuple[str, ...]
    algos: tuple[str, ...]


#: 4 ranks x 4096 fp32, uniform[-1, 1), SUM, ring (plus the 4-element case)
SMALL_RING = Workload("ring-4x4096-f32", 4, 4096, "f32", "uniform", ("sum",), ("ring",))
#: 8 ranks x 64 Mi fp32 (256 MiB per rank), normal(0, 1e-3), SUM and AVG, in place
AR_8x256M = Workload("allreduce-8x256MiB-f32", 8, 1 << 26, "f32", "normal", ("sum", "avg"),
                     ("ring", "oneshot"))
#: 64 ranks x 64 Mi fp32 (16 GiB in all), SUM/MAX/MIN/PROD plus RS, AG, A2A
AR_64x256M = Workload("allreduce-64x256MiB-f32", 64, 1 << 26, "f32", "uniform",
                      ("sum", "max", "min", "prod"), ("oneshot",))


def gpt_grad_tensors(layers: int = 24, d_model: int = 2048, vocab: int = 32000, n_pos: int = 2048,
                     mlp: int = 4) -> list[tuple[str, int]]:
    """The gradient set of a GPT-like model in registration order.

    Learned position embedding, untied LM head; per layer two LayerNorms,
    fused QKV, output projection and a ``mlp``-times-wide MLP, all with bias.
    The default shape (24 layers, d_model 2048, 32k vocab) has 293 tensors
    and 1,343,868,928 parameters.
    """
    d, f = d_model, mlp * d_model
    out = [("wte", vocab * d), ("wpe", n_pos * d)]
    for i in range(layers):
        p = f"h{i}."
        out += [
            (p + "ln1.w", d), (p + "ln1.b", d),
            (p + "qkv.w", d * 3 * d), (p + "qkv.b", 3 * d),
            (p + "proj.w", d * d), (p + "proj.b", d),
            (p + "ln2.w", d), (p + "ln2.b", d),
            (p + "fc1.w", d * f), (p + "fc1.b", f),
            (p + "fc2.w", f * d), (p + "fc2.b", d),
        ]
    out += [("lnf.w", d), ("lnf.b", d), ("lm_head", vocab * d)]
    return out


def grad_ready_order(tensors: list[tuple[str, int]]) -> list[tuple[str, int]]:
    """Backward produces gradients from the last layer to the first, so DDP
    sees them in reverse registration order."""
    return list(reversed(tensors))


def rank_grads(seed: int, rank: int, numels: list[int], dist: str = "normal",
               dtype: str = "bf16") -> list[np.ndarray]:
    """One rank's gradient tensors (flat), each from its own stream."""
    return [rank_values(seed, rank, int(m), dist, dtype, stream=t) for t, m in enumerate(numels)]


#: bucket cap: DDP's default bucket_cap_mb = 25, in binary megabytes
BUCKET_CAP_BYTES = 25 * (1 << 20)
