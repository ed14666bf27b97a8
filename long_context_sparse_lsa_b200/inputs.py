"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module holds no arithmetic of the method: it only draws numbers. Every
value comes from a counter-based generator, SplitMix64 (Steele, Lea & Flood,
"Fast splittable pseudorandom number generators", OOPSLA 2014), evaluated
elementwise with torch int64 ops, so the same (seed, stream, index) gives the
same integers on any device and any slice can be drawn on its own:

    h(seed, stream, i) = mix(base(seed, stream) + i),  base = mix(seed * 2^20 + stream)

  * int8 uniform in [lo, hi]:   lo + (h >> 32) mod (hi - lo + 1)
  * integer weights in [1, hi]: 1 + (h >> 32) mod hi
  * N(0, 1):                    Box-Muller on two streams, u1 = ((h1 >> 11) + 1) 2^-53,
                                u2 = (h2 >> 11) 2^-53, z = sqrt(-2 ln u1) cos(2 pi u2),
                                computed in float64 and rounded to bf16 once.

The integers are bit-identical on CPU and GPU. The bf16 normals are drawn on
the device that consumes them; the oracle always reads a host copy of those
exact bits, never a second draw.
"""
from __future__ import annotations

import math

import torch

_M64 = (1 << 64) - 1


def _s64(c: int) -> int:
    c &= _M64
    return c - (1 << 64) if c >= (1 << 63) else c


_GOLDEN = _s64(0x9E3779B97F4A7C15)
_MUL1 = _s64(0xBF58476D1CE4E5B9)
_MUL2 = _s64(0x94D049BB133111EB)

CHUNK = 1 << 24  # elements drawn per batch of torch ops


def mix64_int(x: int) -> int:
    """SplitMix64 finaliser on a Python int (mod 2^64)."""
    z = (x + 0x9E3779B97F4A7C15) & _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def _srl(x: torch.Tensor, n: int) -> torch.Tensor:
    """Logical right shift of an int64 tensor."""
    return (x >> n) & ((1 << (64 - n)) - 1)


def mix64(x: torch.Tensor) -> torch.Tensor:
    """SplitMix64 finaliser on an int64 tensor (two's-complement wraparound)."""
    z = x + _GOLDEN
    z = (z ^ _srl(z, 30)) * _MUL1
    z = (z ^ _srl(z, 27)) * _MUL2
    return z ^ _srl(z, 31)


def stream_base(seed: int, stream: int) -> int:
    return mix64_int((seed << 20) + stream)


def hashes(seed: int, stream: int, start: int, count: int, device) -> torch.Tensor:
    """h(seed, stream, i) for i in [start, start + count) as int64."""
    base = _s64(stream_base(seed, stream) + start)
    idx = torch.arange(count, dtype=torch.int64, device=device)
    return mix64(idx + base)


def _fill(out: torch.Tensor, seed: int, stream: int, draw) -> torch.Tensor:
    flat = out.view(-1)
    n = flat.numel()
    for start in range(0, n, CHUNK):
        cnt = min(CHUNK, n - start)
        flat[start:start + cnt] = draw(start, cnt)
    return out


def uniform_int8(shape, lo: int, hi: int, seed: int, stream: int, device) -> torch.Tensor:
    span = hi - lo + 1
    out = torch.empty(shape, dtype=torch.int8, device=device)

    def draw(start, cnt):
        h = hashes(seed, stream, start, cnt, device)
        return (_srl(h, 32) % span + lo).to(torch.int8)

    return _fill(out, seed, stream, draw)


def uniform_weights(shape, hi: int, seed: int, stream: int, device) -> torch.Tensor:
    out = torch.empty(shape, dtype=torch.int32, device=device)

    def draw(start, cnt):
        h = hashes(seed, stream, start, cnt, device)
        return (_srl(h, 32) % hi + 1).to(torch.int32)

    return _fill(out, seed, stream, draw)


def normal_bf16(shape, seed: int, stream: int, device) -> torch.Tensor:
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    two_pi = 2.0 * math.pi

    def draw(start, cnt):
        h1 = hashes(seed, stream, start, cnt, device)
        h2 = hashes(seed, stream + (1 << 16), start, cnt, device)
        u1 = (_srl(h1, 11) + 1).to(torch.float64) * (2.0 ** -53)
        u2 = _srl(h2, 11).to(torch.float64) * (2.0 ** -53)
        z = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(two_pi * u2)
        return z.to(torch.bfloat16)

    return _fill(out, seed, stream, draw)


def normal_e4m3(shape, seed: int, stream: int, device) -> torch.Tensor:
    """FP8 E4M3 codes (uint8) of standard normal draws: the same Box-Muller
    draws, rounded to E4M3 once by torch's float8_e4m3fn conversion."""
    out = torch.empty(shape, dtype=torch.uint8, device=device)
    two_pi = 2.0 * math.pi

    def draw(start, cnt):
        h1 = hashes(seed, stream, start, cnt, device)
        h2 = hashes(seed, stream + (1 << 16), start, cnt, device)
        u1 = (_srl(h1, 11) + 1).to(torch.float64) * (2.0 ** -53)
        u2 = _srl(h2, 11).to(torch.float64) * (2.0 ** -53)
        z = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(two_pi * u2)
        return z.to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)

    return _fill(out, seed, stream, draw)


def lognormal_lengths(n: int, median: float, sigma: float, lo: int, hi: int, cap: int,
                      seed: int, stream: int) -> list[int]:
    """Ragged sequence lengths: lognormal(ln median, sigma) drawn with the same
    hash (Box-Muller in Python floats), clipped to [lo, hi]; if the total
    exceeds cap, every length is scaled by cap/total, floored and clipped at lo
    again."""
    b1 = stream_base(seed, stream)
    b2 = stream_base(seed, stream + (1 << 16))
    lens = []
    for i in range(n):
        h1 = mix64_int((b1 + i) & _M64)
        h2 = mix64_int((b2 + i) & _M64)
        u1 = ((h1 >> 11) + 1) * 2.0 ** -53
        u2 = (h2 >> 11) * 2.0 ** -53
        z = math.sqrt(-2.0 * math.log(u1)) * math.cos(2.0 * math.pi * u2)
        L = int(math.floor(math.exp(math.log(median) + sigma * z)))
        lens.append(min(max(L, lo), hi))
    total = sum(lens)
    if total > cap:
        scale = cap / total
        lens = [max(lo, int(math.floor(L * scale))) for L in lens]
    return lens


# Stream ids of the tensors of one workload.
STREAM_Q_IDX = 1
STREAM_K_IDX = 2
STREAM_W = 3
STREAM_LENS = 4
STREAM_DRAFT = 5  # which indexer-query elements a later draft row copies from the first
STREAM_Q = 16   # + layer
STREAM_K = 32   # + layer
STREAM_V = 48   # + layer
STREAM_K8 = 64  # + layer: FP8 E4M3 K cache
STREAM_V8 = 80  # + layer: FP8 E4M3 V cache
