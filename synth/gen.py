"""Counter-based seeded generator for synthetic layer inputs.

Every value is a pure function of (seed, stream name, element index), built
from 32-bit integer hashing only, so the same call gives bit-identical values
on the CPU and on a CUDA device and any slice of a tensor can be generated on
its own (the oracle asks for single batch rows of tensors that only the GPU
holds in full).

Integer hash: the 32-bit finaliser of MurmurHash3 (fmix32, Austin Appleby,
public domain), applied twice to mix the two 32-bit halves of a 64-bit counter
with a per-stream key.

Approximately normal values: each value sums twelve independent 16-bit uniform
integers (Irwin-Hall with n = 12); the sum minus its mean, divided by 2^16, has
mean 0 and variance (2^32 - 1)/2^32 and lies in [-6, 6].  Every step of that is
exact integer arithmetic followed by one exact conversion, so no libm call is
involved and CPU and GPU agree bit for bit.  Uniform values take the top 24 bits
of one hash word, also exact in fp32.

This module holds no arithmetic of the layer itself.
"""
from __future__ import annotations

import torch

_M32 = 0xFFFFFFFF
_GOLDEN = 0x9E3779B9


def _fmix32(x: torch.Tensor) -> torch.Tensor:
    # x: int64 tensor holding values in [0, 2^32).  Products are reduced mod 2^32.
    x = x ^ (x >> 16)
    x = (x * 0x85EBCA6B) & _M32
    x = x ^ (x >> 13)
    x = (x * 0xC2B2AE35) & _M32
    x = x ^ (x >> 16)
    return x


def _fmix32_int(x: int) -> int:
    x &= _M32
    x ^= x >> 16
    x = (x * 0x85EBCA6B) & _M32
    x ^= x >> 13
    x = (x * 0xC2B2AE35) & _M32
    x ^= x >> 16
    return x


def stream_key(seed: int, name: str) -> tuple[int, int]:
    """Two 32-bit keys for a named stream: FNV-1a of the name mixed with the seed."""
    h = 0x811C9DC5
    for b in name.encode("utf-8"):
        h ^= b
        h = (h * 0x01000193) & _M32
    k0 = _fmix32_int(h ^ _fmix32_int(seed & _M32) ^ _fmix32_int((seed >> 32) + _GOLDEN))
    k1 = _fmix32_int(k0 + _GOLDEN)
    return k0, k1


def _words(counter: torch.Tensor, k0: int, k1: int) -> torch.Tensor:
    lo = counter & _M32
    hi = counter >> 32
    h = _fmix32(lo ^ k0)
    return _fmix32(h ^ hi ^ k1)


def normal(n: int, seed: int, name: str, offset: int = 0, device="cpu",
           chunk: int = 1 << 24) -> torch.Tensor:
    """n approximately N(0,1) fp32 values: elements offset .. offset+n-1 of the stream."""
    k0, k1 = stream_key(seed, name)
    out = torch.empty(n, dtype=torch.float32, device=device)
    six = torch.arange(6, dtype=torch.int64, device=device)
    for s in range(0, n, chunk):
        m = min(chunk, n - s)
        idx = torch.arange(offset + s, offset + s + m, dtype=torch.int64, device=device)
        ctr = (idx * 6).unsqueeze(1) + six  # [m, 6]
        w = _words(ctr, k0, k1)
        tot = ((w & 0xFFFF) + (w >> 16)).sum(dim=1)  # twelve 16-bit uniforms
        out[s:s + m] = (tot - 393210).to(torch.float32) * (1.0 / 65536.0)
    return out


def uniform(n: int, seed: int, name: str, offset: int = 0, device="cpu",
            chunk: int = 1 << 24) -> torch.Tensor:
    """n fp32 values uniform on [0, 1), multiples of 2^-24."""
    k0, k1 = stream_key(seed, name)
    out = torch.empty(n, dtype=torch.float32, device=device)
    for s in range(0, n, chunk):
        m = min(chunk, n - s)
        idx = torch.arange(offset + s, offset + s + m, dtype=torch.int64, device=device)
        w = _words(idx, k0, k1)
        out[s:s + m] = (w >> 8).to(torch.float32) * (1.0 / 16777216.0)
    return out


def normal_tensor(shape, seed: int, name: str, std: float = 1.0, mean: float = 0.0,
                  device="cpu", dtype=torch.float32, offset: int = 0) -> torch.Tensor:
    n = 1
    for s in shape:
        n *= int(s)
    v = normal(n, seed, name, offset=offset, device=device)
    if std != 1.0:
        v = v * torch.tensor(std, dtype=torch.float32, device=device)
    if mean != 0.0:
        v = v + torch.tensor(mean, dtype=torch.float32, device=device)
    return v.reshape(tuple(shape)).to(dtype)


def uniform_tensor(shape, seed: int, name: str, low: float, high: float,
                   device="cpu", dtype=torch.float32, offset: int = 0) -> torch.Tensor:
    n = 1
    for s in shape:
        n *= int(s)
    u = uniform(n, seed, name, offset=offset, device=device)
    v = u * torch.tensor(high - low, dtype=torch.float32, device=device) + \
        torch.tensor(low, dtype=torch.float32, device=device)
    return v.reshape(tuple(shape)).to(dtype)
