"""Seeded synthetic inputs (shared by the tests, the oracle runs and the bench).

This module holds none of the layer's arithmetic: it only draws numbers.

Generator: a counter-based SplitMix64 stream (Steele, Lea and Flood, "Fast
splittable pseudorandom number generators", OOPSLA 2014; the finaliser
constants are the published ones).  Draw i of stream (seed, stream_id) is
``mix(key + (i + 1) * GOLDEN)`` with ``key = mix(seed * 2**32 + stream_id)``,
so any slice of a stream can be produced independently and on any device.
Uniforms take the top 53 bits; normals use the Box-Muller transform on pairs
of consecutive uniforms.  Everything is written with torch int64 / float64
tensor ops, so the same code runs on the CPU and on a GPU; integer steps are
exact on both, and float64 log/cos/sin may differ in the last ulp, which does
not survive the rounding to fp32 / bf16 except in vanishingly rare cases.  The
parity tests therefore draw on the CPU and copy the bytes to the device.
"""
from __future__ import annotations

import math

import torch

_GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK64 = (1 << 64) - 1


def _s64(v: int) -> int:
    """Python int in [0, 2^64) -> the int64 with the same bits."""
    v &= _MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _srl(z, 30)) * _s64(_M1)
    z = (z ^ _srl(z, 27)) * _s64(_M2)
    return z ^ _srl(z, 31)


def mix_int(v: int) -> int:
    """Pure-Python SplitMix64 finaliser (used for keys and in tests)."""
    z = v & _MASK64
    z = ((z ^ (z >> 30)) * _M1) & _MASK64
    z = ((z ^ (z >> 27)) * _M2) & _MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, stream: int) -> int:
    return mix_int((seed << 32) + stream)


def raw_u64(seed: int, stream: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """Draws start .. start+count-1 of a stream as int64 bit patterns."""
    key = stream_key(seed, stream)
    i = torch.arange(start + 1, start + count + 1, dtype=torch.int64, device=device)
    z = i * _s64(_GOLDEN) + _s64(key)
    return _mix(z)


def uniform(seed: int, stream: int, count: int, start: int = 0, device="cpu") -> torch.Tensor:
    """float64 uniforms in [0, 1) from the top 53 bits of each draw."""
    z = raw_u64(seed, stream, start, count, device)
    return _srl(z, 11).to(torch.float64) * (1.0 / (1 << 53))


def normal(seed: int, stream: int, count: int, device="cpu", chunk: int = 1 << 26) -> torch.Tensor:
    """float64 standard normals by Box-Muller: uniforms 2p and 2p+1 give normal
    2p (the cosine branch) and normal 2p+1 (the sine branch)."""
    out = torch.empty(count, dtype=torch.float64, device=device)
    pairs = (count + 1) // 2
    for p0 in range(0, pairs, chunk):
        p1 = min(pairs, p0 + chunk)
        u = uniform(seed, stream, 2 * (p1 - p0), start=2 * p0, device=device).view(-1, 2)
        r = torch.sqrt(-2.0 * torch.log1p(-u[:, 0]))     # 1 - u1 in (0, 1]
        th = (2.0 * math.pi) * u[:, 1]
        z = torch.stack((r * torch.cos(th), r * torch.sin(th)), dim=1).view(-1)
        n0, n1 = 2 * p0, min(count, 2 * p1)
        out[n0:n1] = z[: n1 - n0]
    return out


# -- tensors of the workloads ---------------------------------------------------

# stream id = kind << 24 | index: disjoint for every index below 2^24
STREAM_X = 1 << 24
STREAM_GAMMA = 2 << 24
STREAM_OUTLIER = 3 << 24
STREAM_W = 4 << 24


def activations(seed: int, M: int, K: int, index: int = 0, outlier_frac: float = 0.0,
                outlier_scale: float = 20.0, device="cpu") -> torch.Tensor:
    """bf16 x[M, K] ~ N(0, 1); optionally a seeded 1% (rounded) of the channels
    scaled by ``outlier_scale`` on every token."""
    z = normal(seed, STREAM_X + index, M * K, device=device).view(M, K)
    if outlier_frac > 0.0:
        n_out = max(1, int(round(outlier_frac * K)))
        keys = uniform(seed, STREAM_OUTLIER + index, K, device=device)
        ch = torch.argsort(keys)[:n_out]
        z[:, ch] *= outlier_scale
    return z.to(torch.float32).to(torch.bfloat16)


def outlier_channels(seed: int, K: int, index: int = 0, outlier_frac: float = 0.01) -> torch.Tensor:
    n_out = max(1, int(round(outlier_frac * K)))
    keys = uniform(seed, STREAM_OUTLIER + index, K)
    return torch.sort(torch.argsort(keys)[:n_out]).values


def gamma(seed: int, K: int, index: int = 0, device="cpu") -> torch.Tensor:
    """fp32 RMSNorm gain 1 + N(0, 0.1)."""
    return (1.0 + 0.1 * normal(seed, STREAM_GAMMA + index, K, device=device)).to(torch.float32)


def latent_weights(seed: int, N: int, K: int, index: int = 0, std: float = 0.02,
                   device="cpu") -> torch.Tensor:
    """fp32 latent W[N, K] ~ N(0, std^2)."""
    return (std * normal(seed, STREAM_W + index, N * K, device=device)).to(torch.float32).view(N, K)


def bf16_bits(t: torch.Tensor) -> torch.Tensor:
    """bf16 tensor -> its uint16 bit patterns as an int16 view."""
    assert t.dtype == torch.bfloat16
    return t.view(torch.int16)
