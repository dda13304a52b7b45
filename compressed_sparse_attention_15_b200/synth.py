"""Seeded, counter-based synthetic inputs.

This module only draws numbers. It holds none of the attention method's
arithmetic, and both the CUDA path's tests/bench and the fp64 oracle take
their inputs from it, so the two sides see bit-identical values.

Every value is a pure function of (seed, tensor id, flat element index):

* A 64-bit counter stream: state_c = key + (c + 1) * GAMMA (mod 2**64), hashed
  with the SplitMix64 finaliser (Steele, Lea & Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014). key = mix(seed << 32 | tid).
* U(0,1): the top 24 bits of hash c = i, times 2**-24.
* N(0,1): Irwin-Hall sum of 12 such 24-bit uniforms minus 6. The 12 uniforms
  come from hashes c = 6 i .. 6 i + 5 (bits 40..63 and bits 8..31 of each).
  The sum is an exact integer, converted exactly to fp64, then rounded once to
  fp32 (round-to-nearest-even) and, for bf16 tensors, once more to bf16 (RNE).
  Tails are bounded at +-6, a stated departure from the exact normal.
* A standard deviation sigma != 1 multiplies the fp32 value by fp32(sigma).

Because the stream is indexed by element, any slice (a row range, a gathered
set of rows) can be regenerated on the host without materialising the whole
tensor. The same torch integer ops run on CPU and CUDA, so host and device
produce the same bytes.
"""
from __future__ import annotations

import torch

_M64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
_C1 = 0xBF58476D1CE4E5B9
_C2 = 0x94D049BB133111EB


def _s64(u: int) -> int:
    """Unsigned 64-bit constant -> the signed int64 with the same bits."""
    u &= _M64
    return u - (1 << 64) if u >= (1 << 63) else u


def _lsr(x: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 bits (torch's >> is arithmetic)."""
    return (x >> s) & ((1 << (64 - s)) - 1)


def _mix(x: torch.Tensor) -> torch.Tensor:
    x = (x ^ _lsr(x, 30)) * _s64(_C1)
    x = (x ^ _lsr(x, 27)) * _s64(_C2)
    return x ^ _lsr(x, 31)


def mix_int(x: int) -> int:
    """Pure-Python SplitMix64 finaliser (used for the key and for checks)."""
    x &= _M64
    x = ((x ^ (x >> 30)) * _C1) & _M64
    x = ((x ^ (x >> 27)) * _C2) & _M64
    return x ^ (x >> 31)


def stream_key(seed: int, tid: int) -> int:
    return mix_int(((seed & 0xFFFFFFFF) << 32) | (tid & 0xFFFFFFFF))


def _hash(seed: int, tid: int, c: torch.Tensor) -> torch.Tensor:
    key = _s64(stream_key(seed, tid))
    return _mix((c + 1) * _s64(GAMMA) + key)


def _u24_pair(h: torch.Tensor):
    return _lsr(h, 40), _lsr(h, 8) & 0xFFFFFF


CHUNK = 1 << 24


def uniform_at(seed: int, tid: int, flat: torch.Tensor) -> torch.Tensor:
    """U(0,1) (fp32, exact multiples of 2**-24) at the given flat indices."""
    out = torch.empty(flat.shape, dtype=torch.float32, device=flat.device)
    f = flat.reshape(-1)
    o = out.view(-1)
    for s in range(0, f.numel(), CHUNK):
        c = f[s:s + CHUNK].to(torch.int64)
        hi, _ = _u24_pair(_hash(seed, tid, c))
        o[s:s + CHUNK] = hi.to(torch.float64).mul_(2.0 ** -24).to(torch.float32)
    return out


def normal_at(seed: int, tid: int, flat: torch.Tensor, std: float = 1.0) -> torch.Tensor:
    """Irwin-Hall N(0, std) (fp32) at the given flat indices."""
    out = torch.empty(flat.shape, dtype=torch.float32, device=flat.device)
    f = flat.reshape(-1)
    o = out.view(-1)
    for s in range(0, f.numel(), CHUNK // 4):
        base = f[s:s + CHUNK // 4].to(torch.int64) * 6
        acc = torch.zeros_like(base)
        for m in range(6):
            hi, lo = _u24_pair(_hash(seed, tid, base + m))
            acc += hi
            acc += lo
        v = acc.to(torch.float64).mul_(2.0 ** -24).sub_(6.0).to(torch.float32)
        if std != 1.0:
            v = v * torch.tensor(std, dtype=torch.float32, device=v.device)
        o[s:s + CHUNK // 4] = v
    return out


def _flat(shape, device) -> torch.Tensor:
    n = 1
    for d in shape:
        n *= int(d)
    return torch.arange(n, dtype=torch.int64, device=device).reshape(tuple(shape))


def normal(seed, tid, shape, *, std=1.0, dtype=torch.float32, device="cpu") -> torch.Tensor:
    """A whole tensor of N(0, std) values, rounded once to ``dtype``."""
    n = 1
    for d in shape:
        n *= int(d)
    out = torch.empty(n, dtype=dtype, device=device)
    step = 1 << 26
    for s in range(0, n, step):
        e = min(n, s + step)
        idx = torch.arange(s, e, dtype=torch.int64, device=device)
        out[s:e] = normal_at(seed, tid, idx, std).to(dtype)
    return out.reshape(tuple(shape))


def uniform(seed, tid, shape, *, dtype=torch.float32, device="cpu") -> torch.Tensor:
    return uniform_at(seed, tid, _flat(shape, device)).to(dtype)


def normal_rows(seed, tid, shape, rows, *, std=1.0, dtype=torch.float32) -> torch.Tensor:
    """Rows ``rows`` (indices into the flattened leading dims) of a tensor of
    shape ``shape`` whose last dim is the row width, regenerated on the host."""
    width = int(shape[-1])
    rows = torch.as_tensor(rows, dtype=torch.int64).reshape(-1, 1)
    flat = rows * width + torch.arange(width, dtype=torch.int64).reshape(1, -1)
    return normal_at(seed, tid, flat, std).to(dtype)
