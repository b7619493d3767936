"""Seeded, counter-based synthetic inputs for the BitLinear forward.

This module holds no part of the BitLinear arithmetic.  It only draws the
numbers that stand in for activations, weights and biases: both the CPU oracle
(tests, cpu baseline) and the CUDA path (tests, bench) take their inputs from
here, so that the two sides see the same bits.

Generator (written from the published definitions):

* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): ``mix(z)`` is the 64-bit finaliser with the
  multipliers 0xBF58476D1CE4E5B9 and 0x94D049BB133111EB and shifts 30/27/31;
  draw ``c`` of stream ``(seed, stream)`` is ``mix(base + (c + 1) * GAMMA)``
  with ``GAMMA = 0x9E3779B97F4A7C15`` and ``base = mix(seed * GAMMA ^
  mix(stream + GAMMA))``.  Every value depends only on (seed, stream, index),
  never on chunking or thread count.
* Uniform on (0, 1]: ``((z >> 11) + 1) * 2**-53``.
* Normal: Box-Muller (Box and Muller 1958), cosine branch, in float64, from
  draws ``2i`` and ``2i + 1``; then scaled by sigma and rounded to the target
  dtype (float32 round-to-nearest; bfloat16 by torch's round-to-nearest-even
  from the float32 value).
* Student-t with nu = 4: ``Z / sqrt((E1 + E2) / 2)`` where Z is normal and
  E = -ln(U) are unit exponentials (chi-square with 4 degrees of freedom is
  2 (E1 + E2)).

Values made on the host use the host's libm; ``device="cuda"`` runs the same
formula with torch on the GPU, whose log/cos may differ in the last ulp, so
parity tests always generate on the host.
"""

from __future__ import annotations

import concurrent.futures as _fut
import os

import numpy as np
import torch

GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK64 = (1 << 64) - 1
_CHUNK = 1 << 22


def _mix_int(z: int) -> int:
    z &= _MASK64
    z = ((z ^ (z >> 30)) * _M1) & _MASK64
    z = ((z ^ (z >> 27)) * _M2) & _MASK64
    return z ^ (z >> 31)


def stream_base(seed: int, stream: int) -> int:
    """64-bit starting point of stream ``stream`` under ``seed``."""
    return _mix_int(((seed * GAMMA) & _MASK64) ^ _mix_int(stream + GAMMA))


def _mix_np(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(_M1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(_M2)
    return z ^ (z >> np.uint64(31))


def _draws_np(base: int, start: int, count: int) -> np.ndarray:
    """Raw 64-bit draws ``start .. start+count-1`` of a stream (numpy, host)."""
    c = np.arange(start + 1, start + 1 + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(base) + c * np.uint64(GAMMA)
        return _mix_np(z)


def _unit_np(z: np.ndarray) -> np.ndarray:
    return ((z >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)


def _normal_chunk(base: int, i0: int, n: int) -> np.ndarray:
    z = _draws_np(base, 2 * i0, 2 * n)
    u1 = _unit_np(z[0::2])
    u2 = _unit_np(z[1::2])
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def _student4_chunk(base: int, i0: int, n: int) -> np.ndarray:
    z = _draws_np(base, 4 * i0, 4 * n)
    u1 = _unit_np(z[0::4])
    u2 = _unit_np(z[1::4])
    e1 = -np.log(_unit_np(z[2::4]))
    e2 = -np.log(_unit_np(z[3::4]))
    g = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
    return g / np.sqrt(0.5 * (e1 + e2))


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _fill_f32(kind, base: int, n: int, scale: float) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)

    def job(i0):
        m = min(_CHUNK, n - i0)
        out[i0:i0 + m] = (kind(base, i0, m) * scale).astype(np.float32)

    starts = range(0, n, _CHUNK)
    if n <= _CHUNK:
        for s in starts:
            job(s)
    else:
        with _fut.ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(job, starts))
    return out


# ---- device variant (torch), same formula -----------------------------------

def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    return (z >> s) & ((1 << (64 - s)) - 1)


def _s64(v: int) -> int:
    v &= _MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def _mix_t(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _srl(z, 30)) * _s64(_M1)
    z = (z ^ _srl(z, 27)) * _s64(_M2)
    return z ^ _srl(z, 31)


def _unit_t(z: torch.Tensor) -> torch.Tensor:
    return (_srl(z, 11).to(torch.float64) + 1.0) * (2.0 ** -53)


def _normal_t(base: int, n: int, device) -> torch.Tensor:
    out = torch.empty(n, dtype=torch.float64, device=device)
    step = 1 << 24
    for i0 in range(0, n, step):
        m = min(step, n - i0)
        c = torch.arange(2 * i0 + 1, 2 * (i0 + m) + 1, dtype=torch.int64, device=device)
        z = _mix_t(c * _s64(GAMMA) + _s64(base))
        u1 = _unit_t(z[0::2])
        u2 = _unit_t(z[1::2])
        out[i0:i0 + m] = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(2.0 * torch.pi * u2)
    return out


# ---- public generators -------------------------------------------------------

def normal_f32(seed: int, stream: int, shape, sigma: float = 1.0, device: str = "cpu") -> torch.Tensor:
    """float32 tensor of N(0, sigma^2) draws, row-major ``shape``."""
    n = int(np.prod(shape))
    base = stream_base(seed, stream)
    if str(device).startswith("cuda"):
        return (_normal_t(base, n, device) * sigma).to(torch.float32).reshape(shape)
    return torch.from_numpy(_fill_f32(_normal_chunk, base, n, sigma)).reshape(shape)


def normal_bf16(seed: int, stream: int, shape, sigma: float = 1.0, device: str = "cpu") -> torch.Tensor:
    return normal_f32(seed, stream, shape, sigma, device).to(torch.bfloat16)


def student_t4_bf16(seed: int, stream: int, shape) -> torch.Tensor:
    """bfloat16 tensor of Student-t (nu = 4) draws (heavy-tailed activations)."""
    n = int(np.prod(shape))
    base = stream_base(seed, stream)
    return torch.from_numpy(_fill_f32(_student4_chunk, base, n, 1.0)).reshape(shape).to(torch.bfloat16)


def outlier_channels(seed: int, stream: int, K: int, frac: float = 0.01) -> np.ndarray:
    """Sorted indices of round(frac*K) distinct channels, chosen by a seeded
    partial Fisher-Yates shuffle driven by the same counter stream."""
    count = int(round(frac * K))
    perm = np.arange(K, dtype=np.int64)
    z = _draws_np(stream_base(seed, stream), 0, max(count, 1))
    for i in range(count):
        j = i + int(z[i] % np.uint64(K - i))
        perm[i], perm[j] = perm[j], perm[i]
    return np.sort(perm[:count])


def normal_with_outliers_bf16(seed: int, stream: int, shape, factor: float = 20.0,
                              frac: float = 0.01) -> torch.Tensor:
    """N(0,1) activations with ``frac`` of the channels (last dim) scaled by
    ``factor`` before the bfloat16 rounding (outlier columns)."""
    M, K = shape
    x = normal_f32(seed, stream, shape, 1.0)
    cols = torch.from_numpy(outlier_channels(seed, stream + 1_000_003, K, frac))
    x[:, cols] *= factor
    return x.to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 bit patterns of a bfloat16 tensor (host copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
