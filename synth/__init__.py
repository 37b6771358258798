"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module draws random numbers and nothing else: it holds none of the
attention arithmetic.  Both sides (the fp64 oracle and the GPU library) read
the exact same rounded bf16/fp16 values produced here.

Generator (counter based, so any element can be recomputed on its own):

* ``splitmix64(x)``: the published SplitMix64 finaliser (Steele, Lea, Flood,
  "Fast splittable pseudorandom number generators", OOPSLA 2014).
* element ``n`` of a stream with key ``seed`` uses counters
  ``2*(n//2)`` and ``2*(n//2)+1`` -> two uniforms in (0, 1] ->
  Box-Muller pair (cos for even n, sin for odd n).
* the fp64 sample is multiplied by ``sigma`` and rounded to the target dtype
  by torch's round-to-nearest-even conversion.

Workload recipes (shapes, value distributions, length mixes) follow the
flex-attention benchmark configurations: iid N(0, sigma^2) Q/K/V, per-sequence
KV lengths uniform in [1, cap], and a Bernoulli(0.1) -inf additive mask.
"""
from __future__ import annotations

import numpy as np
import torch

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def splitmix64(x: np.ndarray) -> np.ndarray:
    """SplitMix64 output function applied elementwise to uint64 counters."""
    with np.errstate(over="ignore"):
        z = x + _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def _stream_key(seed: int) -> np.uint64:
    return splitmix64(np.array([seed & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64))[0]


def uniform01(seed: int, start: int, count: int) -> np.ndarray:
    """Uniforms in (0, 1] for counters [start, start+count) of stream ``seed``."""
    key = _stream_key(seed)
    ctr = np.arange(start, start + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        bits = splitmix64(ctr * _GOLDEN + key)
    return ((bits >> np.uint64(11)).astype(np.float64) + 1.0) * (1.0 / 9007199254740992.0)


def normal_fp64(seed: int, n: int) -> np.ndarray:
    """n iid N(0,1) fp64 samples (Box-Muller over the counter stream)."""
    out = np.empty(n, dtype=np.float64)
    npairs = (n + 1) // 2
    for p0 in range(0, npairs, _CHUNK):
        p1 = min(npairs, p0 + _CHUNK)
        u = uniform01(seed, 2 * p0, 2 * (p1 - p0))
        u1, u2 = u[0::2], u[1::2]
        r = np.sqrt(-2.0 * np.log(u1))
        t = 2.0 * np.pi * u2
        pair = np.empty(2 * (p1 - p0), dtype=np.float64)
        pair[0::2] = r * np.cos(t)
        pair[1::2] = r * np.sin(t)
        lo = 2 * p0
        hi = min(n, 2 * p1)
        out[lo:hi] = pair[: hi - lo]
    return out


_DTYPES = {"bf16": torch.bfloat16, "f16": torch.float16, "fp16": torch.float16,
           "bfloat16": torch.bfloat16, "float16": torch.float16}


def torch_dtype(name) -> torch.dtype:
    if isinstance(name, torch.dtype):
        return name
    return _DTYPES[name]


def _as_i64(c: int) -> int:
    c &= 0xFFFFFFFFFFFFFFFF
    return c - (1 << 64) if c >= (1 << 63) else c


_T_GOLDEN, _T_M1, _T_M2 = _as_i64(0x9E3779B97F4A7C15), _as_i64(0xBF58476D1CE4E5B9), _as_i64(0x94D049BB133111EB)


def _shr(x: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return (x >> s) & ((1 << (64 - s)) - 1)


def _splitmix64_t(x: torch.Tensor) -> torch.Tensor:
    z = x + _T_GOLDEN
    z = (z ^ _shr(z, 30)) * _T_M1
    z = (z ^ _shr(z, 27)) * _T_M2
    return z ^ _shr(z, 31)


def normal_fp64_torch(seed: int, n: int, device) -> torch.Tensor:
    """Same stream as normal_fp64 (identical uniforms), computed with torch on ``device``."""
    key = _as_i64(int(_stream_key(seed)))
    out = torch.empty(n, dtype=torch.float64, device=device)
    npairs = (n + 1) // 2
    step = 1 << 24
    for p0 in range(0, npairs, step):
        p1 = min(npairs, p0 + step)
        ctr = torch.arange(2 * p0, 2 * p1, dtype=torch.int64, device=device)
        bits = _splitmix64_t(ctr * _T_GOLDEN + key)
        u = (_shr(bits, 11).to(torch.float64) + 1.0) * (1.0 / 9007199254740992.0)
        u1, u2 = u[0::2], u[1::2]
        r = torch.sqrt(-2.0 * torch.log(u1))
        t = (2.0 * np.pi) * u2
        pair = torch.stack((r * torch.cos(t), r * torch.sin(t)), dim=1).reshape(-1)
        lo, hi = 2 * p0, min(n, 2 * p1)
        out[lo:hi] = pair[: hi - lo]
    return out


def normal_tensor(shape, seed: int, sigma: float = 1.0, dtype="bf16", device=None) -> torch.Tensor:
    """Tensor of iid N(0, sigma^2) values rounded (RN-even) to ``dtype``.

    device None: computed with numpy on the CPU.  Otherwise the torch implementation of
    the same counter stream runs on ``device`` (used for large inputs); uniforms are
    bit-identical, the fp64 Box-Muller may differ in the last ulp.
    """
    n = int(np.prod(shape)) if len(shape) else 1
    if device is None:
        z = normal_fp64(seed, n) * sigma
        return torch.from_numpy(z).reshape(tuple(shape)).to(torch_dtype(dtype))
    z = normal_fp64_torch(seed, n, device)
    z.mul_(sigma)
    return z.to(torch_dtype(dtype)).reshape(tuple(shape))


def kv_lengths(batch: int, cap: int, seed: int, lo: int = 1) -> torch.Tensor:
    """Per-sequence KV lengths, uniform integers in [lo, cap] (int32, CPU)."""
    u = uniform01(seed, 0, batch)
    span = cap - lo + 1
    v = lo + np.minimum((u * span).astype(np.int64), span - 1)
    # u is in (0, 1]; u == 1 maps to the top bin through the clamp above
    return torch.from_numpy(v.astype(np.int32))


def bernoulli_neg_inf_mask(shape, p: float, seed: int, dtype="f16") -> torch.Tensor:
    """Additive mask: -inf with probability p, else 0 (CPU, ``dtype``)."""
    n = int(np.prod(shape))
    u = uniform01(seed, 0, n)
    m = np.where(u <= p, -np.inf, 0.0)
    return torch.from_numpy(m).reshape(tuple(shape)).to(torch_dtype(dtype))


def case_seed(config: int, case: int, rep: int = 0) -> int:
    """Seed convention: 1000*config + 10*case + rep (tensors offset it further)."""
    return 1000 * config + 10 * case + rep


def qkv(B, H, Hkv, Sq, Skv, D, seed, sigma=1.0, dtype="bf16", device=None):
    """Q [B,H,Sq,D], K/V [B,Hkv,Skv,D] with independent streams seed*8+{1,2,3}."""
    q = normal_tensor((B, H, Sq, D), seed * 8 + 1, sigma, dtype, device)
    k = normal_tensor((B, Hkv, Skv, D), seed * 8 + 2, sigma, dtype, device)
    v = normal_tensor((B, Hkv, Skv, D), seed * 8 + 3, sigma, dtype, device)
    return q, k, v
