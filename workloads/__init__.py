"""Seeded synthetic inputs for the YOCO / YOCO++ attention core.

This module is the only code that both the CUDA-side tests / benchmark and
the CPU oracle use.  It draws random numbers and names workload shapes; it
holds none of the method's arithmetic (no normalisation, projection, blend,
masking or softmax).

Distributions follow the method's workloads: activations and Q/K/V ~ N(0, 1),
projection weights ~ N(0, 1/d), YOCO++ residual weights ~ U(0, 1), ragged
decode lengths integer-uniform with both ends inclusive.  Seeds are
``config_index * 1000 + layer`` unless a test states otherwise.
"""
from dataclasses import dataclass, field
from typing import List

import torch

DTYPES = {"bf16": torch.bfloat16, "fp32": torch.float32}


def gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, seed, dtype=torch.bfloat16, device="cpu", std=1.0):
    """N(0, std^2) drawn in fp32 from a seeded generator, then rounded to dtype."""
    g = gen(seed, device)
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def uniform(shape, seed, lo=0.0, hi=1.0, device="cpu"):
    g = gen(seed, device)
    return torch.rand(*shape, generator=g, device=device, dtype=torch.float64) * (hi - lo) + lo


def randint_inclusive(shape, seed, lo, hi, device="cpu"):
    g = gen(seed, device)
    return torch.randint(lo, hi + 1, shape, generator=g, device=device, dtype=torch.int64)


def sample_rows(T, n_random, seed, extra=()):
    """Row indices for sampled parity at scale: 0, 1, the given extra rows
    (window / chunk boundaries +-1), the last row, plus n_random seeded
    random rows; deduplicated, sorted, clipped to [0, T)."""
    rows = {0, 1, T - 1}
    for e in extra:
        for d in (-1, 0, 1):
            rows.add(e + d)
    if n_random > 0:
        r = torch.randint(0, T, (n_random,), generator=gen(seed))
        rows.update(int(x) for x in r)
    return sorted(x for x in rows if 0 <= x < T)


@dataclass
class TinyStack:
    """Tiny YOCO++ attention stack: fp32, B=1, T=256 (+16 decode), d=256,
    4 query / 2 KV heads, head_dim 64, 2 SWA self layers (window 32, YOCO++
    blend w=0.5 on layer 2 to layer-1 KV), 2 cross layers over one global KV."""
    T: int = 256
    n_decode: int = 16
    d: int = 256
    Hq: int = 4
    Hkv: int = 2
    D: int = 64
    window: int = 32
    n_self: int = 2
    n_cross: int = 2
    w_blend: List[float] = field(default_factory=lambda: [0.0, 0.5])
    seed: int = 0


def tiny_stack_inputs(cfg: TinyStack, dtype=torch.float32):
    """x [T + n_decode, d] ~ N(0,1) and all weights ~ N(0, 1/d), seeded from
    cfg.seed; weights are [out_features, in_features]."""
    s = cfg.seed
    d, Hq, Hkv, D = cfg.d, cfg.Hq, cfg.Hkv, cfg.D
    std = 1.0 / (d ** 0.5)
    x = normal((cfg.T + cfg.n_decode, d), s * 1000 + 0, dtype)
    w = {"self_q": [], "self_kv": [], "self_o": [], "cross_q": [], "cross_o": []}
    k = 1
    for _ in range(cfg.n_self):
        w["self_q"].append(normal((Hq * D, d), s * 1000 + k, dtype, std=std)); k += 1
        w["self_kv"].append(normal((2 * Hkv * D, d), s * 1000 + k, dtype, std=std)); k += 1
        w["self_o"].append(normal((d, Hq * D), s * 1000 + k, dtype,
                                  std=1.0 / ((Hq * D) ** 0.5))); k += 1
    w["g_kv"] = normal((2 * Hkv * D, d), s * 1000 + k, dtype, std=std); k += 1
    for _ in range(cfg.n_cross):
        w["cross_q"].append(normal((Hq * D, d), s * 1000 + k, dtype, std=std)); k += 1
        w["cross_o"].append(normal((d, Hq * D), s * 1000 + k, dtype,
                                   std=1.0 / ((Hq * D) ** 0.5))); k += 1
    return x, w


# Workload shapes of the benchmark / parity configurations (bf16 unless noted).
CROSS_PREFILL_32K = dict(B=1, T=32768, Hq=32, Hkv=8, D=128, layers=14)
CROSS_DECODE_128K = dict(B=16, len_lo=65536, len_hi=131072, Hq=32, Hkv=8, D=128, layers=16)
SWA_64K = dict(B=4, T=65536, window=1024, Hq=32, Hkv=8, D=128, d=4096, layers=16,
               decode_steps=256)
LONG_1M = dict(B=1, T=1048576, chunk=32768, Hq=32, Hkv=8, D=128, layers=16, decode_steps=64)


def ragged_lengths(B, lo, hi, seed):
    return randint_inclusive((B,), seed, lo, hi)
