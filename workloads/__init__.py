"""Seeded synthetic inputs for the quantized-GEMM hot path.

Shared by the tests, the smoke check and the benchmark, on both sides of every
parity comparison.  This module draws random numbers and casts them to fp16
(numpy's round-to-nearest-even cast); it holds none of the method's arithmetic
(no quantization, no packing, no products).

Distributions follow the LLM-linear workloads on the pages:
  * activations X ~ N(0,1) fp16, optionally with 1 % of the K channels scaled by
    20 (outlier channels, "量化与多精度算子" §六 on per-tensor outliers);
  * weights W [N,K] (the storage of a column-major [K,N]) ~ N(0, 0.02) times a
    per-output-column factor log-uniform in [0.1, 2.5] ("Ascend C per-channel
    INT8 GEMM" §4.2: some channels max|w| = 0.1, others 2.5);
  * bias ~ N(0, 0.1) fp32.
No public dataset or trained weight is used; these draws stand in for them.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

# Tags that give every tensor of a configuration its own random stream.
_TAG_X, _TAG_W, _TAG_BIAS, _TAG_OUTLIER, _TAG_COLFACTOR = 1, 2, 3, 4, 5


def _rng(seed: int, tag: int, extra: int = 0) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(tag), int(extra)])


def activations(M: int, K: int, seed: int, outliers: bool = False, ld: int | None = None) -> np.ndarray:
    """X fp16 [M, ld] (ld >= K; columns K..ld-1 are padding filled with 0)."""
    x = _rng(seed, _TAG_X).standard_normal((M, K), dtype=np.float64)
    if outliers and K > 0:
        n_out = max(1, int(round(0.01 * K)))
        cols = _rng(seed, _TAG_OUTLIER).choice(K, size=n_out, replace=False)
        x[:, cols] *= 20.0
    x16 = x.astype(np.float16)
    if ld is not None and ld != K:
        out = np.zeros((M, ld), dtype=np.float16)
        out[:, :K] = x16
        return out
    return x16


def weights(N: int, K: int, seed: int, per_column_factor: bool = True, std: float = 0.02) -> np.ndarray:
    """W fp16 stored [N, K]: row n is output column n of the column-major [K, N]."""
    w = _rng(seed, _TAG_W).standard_normal((N, K), dtype=np.float64) * std
    if per_column_factor:
        u = _rng(seed, _TAG_COLFACTOR).uniform(math.log(0.1), math.log(2.5), size=(N, 1))
        w = w * np.exp(u)
    return w.astype(np.float16)


def edge_weights(N: int, K: int, seed: int) -> np.ndarray:
    """W fp16 [N, K] built from 64-element blocks (along K) of structured patterns,
    the cases where the weight quantizers' floors and clamps act, mixed with
    ordinary N(0, 0.02) blocks.  Block b of row n takes pattern (7 n + b) % 24:
      0..15  ramp 0.125 * ((k % 16) - j) with j = the pattern: min -0.125 j, max
             0.125 (15 - j), so the block-64 asymmetric 4-bit zero point is j;
      16     all zero (flat: the scale floors);
      17     constant 0.75 (flat, nonzero);
      18     0.5 + 0.0625 (k % 16): all positive (zero point clamps to 0, codes to 15);
      19     -0.5 - 0.0625 (k % 16): all negative (zero point clamps to 15);
      20     +-5e-5 at the block's first two elements, zero elsewhere (tiny scale);
      21..23 N(0, 0.02) draws.
    Rows n % 11 == 0 are all zero and rows n % 11 == 1 all -0.75 (whole-row
    floors and constants for per-row / per-column quantizers).  K % 64 == 0."""
    assert K % 64 == 0
    k = np.arange(64, dtype=np.float64)
    pats = [0.125 * ((k % 16) - j) for j in range(16)]
    pats += [0.0 * k, 0.75 + 0.0 * k, 0.5 + 0.0625 * (k % 16), -0.5 - 0.0625 * (k % 16),
             5e-5 * (k == 0) - 5e-5 * (k == 1)]
    table = np.stack(pats)                                       # [21, 64]
    rnd = _rng(seed, _TAG_W, 77).standard_normal((N, K)) * 0.02
    nb = K // 64
    sel = (7 * np.arange(N)[:, None] + np.arange(nb)[None, :]) % 24  # [N, nb]
    w = rnd.reshape(N, nb, 64).copy()
    structured = sel < len(pats)
    w[structured] = table[sel[structured]]
    w = w.reshape(N, K)
    w[np.arange(N) % 11 == 0] = 0.0
    w[np.arange(N) % 11 == 1] = -0.75
    return w.astype(np.float16)


def bias(N: int, seed: int, std: float = 0.1) -> np.ndarray:
    return (_rng(seed, _TAG_BIAS).standard_normal(N) * std).astype(np.float32)


def sample_rows(M: int, count: int, seed: int) -> np.ndarray:
    """A seeded sorted sample of row indices (used to check full-size outputs)."""
    count = min(count, M)
    return np.sort(_rng(seed, 99).choice(M, size=count, replace=False))


@dataclass(frozen=True)
class Workload:
    """One LLM-linear shape: Y[M,N] = X[M,K] @ W[K,N]."""
    name: str
    kind: str          # "w8a8" | "w8a16" | "w4a16"
    M: int
    N: int
    K: int
    out: str           # "f32" | "f16" | "bf16"
    seed: int
    outliers: bool
    bias: bool
    per_column_factor: bool = True
    group: int = 64


# The five workload families (LLaMA-7B q_proj 4096x4096 and FFN width 11008).
W8A8_SMALL = [Workload("w8a8_m16_k256_n256", "w8a8", 16, 256, 256, "f32", 0, False, True)]
W8A8_DECODE = [Workload(f"w8a8_decode_m{m}_k4096_n4096", "w8a8", m, 4096, 4096, "f16", 1, True, True)
               for m in (1, 8, 16)]
W8A8_PREFILL = [Workload(f"w8a8_prefill_m{m}_k4096_n{n}", "w8a8", m, n, 4096, "bf16", 2, True, True)
                for m in (2048, 8192) for n in (4096, 11008)]
W8A16 = [Workload(f"w8a16_m{m}_k4096_n{n}", "w8a16", m, n, 4096, "f16", 3, False, False)
         for m in (1, 16, 256) for n in (4096, 11008)]
W4A16 = [Workload(f"w4a16_m{m}_k4096_n11008", "w4a16", m, 11008, 4096, "f16", 4, False, False,
                  per_column_factor=False) for m in (1, 16)]
ALL = W8A8_SMALL + W8A8_DECODE + W8A8_PREFILL + W8A16 + W4A16
BY_NAME = {w.name: w for w in ALL}


# --- on-device generators for the benchmark (same distributions, torch RNG) ---
# The benchmark needs several hundred MB of weights; drawing them on the GPU is
# fast.  Values differ from the numpy draws above (different generator); the
# parity tests use the numpy draws, the benchmark these.

def torch_activations(M: int, K: int, seed: int, device, outliers: bool = False):
    import torch
    g = torch.Generator(device=device).manual_seed(int(seed) * 1000003 + _TAG_X)
    x = torch.randn((M, K), generator=g, device=device, dtype=torch.float32)
    if outliers and K > 0:
        n_out = max(1, int(round(0.01 * K)))
        cols = torch.randperm(K, generator=g, device=device)[:n_out]
        x[:, cols] *= 20.0
    return x.to(torch.float16)


def torch_weights(N: int, K: int, seed: int, device, per_column_factor: bool = True, std: float = 0.02):
    import torch
    g = torch.Generator(device=device).manual_seed(int(seed) * 1000003 + _TAG_W)
    w = torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * std
    if per_column_factor:
        u = torch.empty((N, 1), device=device).uniform_(math.log(0.1), math.log(2.5), generator=g)
        w = w * torch.exp(u)
    return w.to(torch.float16)


def torch_bias(N: int, seed: int, device, std: float = 0.1):
    import torch
    g = torch.Generator(device=device).manual_seed(int(seed) * 1000003 + _TAG_BIAS)
    return torch.randn(N, generator=g, device=device) * std
