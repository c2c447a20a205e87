"""Counter-based random numbers for the synthetic workloads.

Every value is a pure function of (seed, stream name, element index), so any
slice of any tensor can be regenerated on its own and the result does not
depend on the device, the chunking or the order of generation of the integer
part.  The generator is SplitMix64 (Steele, Lea and Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014): state_i = key + i * gamma,
output_i = mix64(state_i), with gamma = 0x9E3779B97F4A7C15 and the mix64
finaliser constants of that paper.  Normal deviates come from the Box-Muller
transform (Box and Muller, 1958) of two 53-bit uniforms.

This module holds none of the attention method's arithmetic; it only makes
numbers.  It is shared by the oracle side and the CUDA side of every test.
"""
from __future__ import annotations

import torch

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB


def _as_i64(c: int) -> int:
    """Two's-complement view of an unsigned 64-bit constant."""
    c &= MASK64
    return c - (1 << 64) if c >= (1 << 63) else c


_GAMMA_I = _as_i64(GAMMA)
_MIX1_I = _as_i64(MIX1)
_MIX2_I = _as_i64(MIX2)


def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 lanes holding uint64 bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def mix64(z: torch.Tensor) -> torch.Tensor:
    """SplitMix64 output function on int64 tensors (wrapping arithmetic)."""
    z = (z ^ _lsr(z, 30)) * _MIX1_I
    z = (z ^ _lsr(z, 27)) * _MIX2_I
    return z ^ _lsr(z, 31)


def mix64_int(z: int) -> int:
    """The same function on Python integers (used for stream keys and tests)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * MIX1) & MASK64
    z = ((z ^ (z >> 27)) * MIX2) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, name: str) -> int:
    """64-bit key of a named stream: mixes the seed with an FNV-1a hash of the name."""
    h = 0xCBF29CE484222325
    for ch in name.encode():
        h = ((h ^ ch) * 0x100000001B3) & MASK64
    return mix64_int(mix64_int(seed * GAMMA + 1) ^ h)


def raw_u64(seed: int, name: str, start: int, count: int, device="cpu") -> torch.Tensor:
    """Outputs start..start+count-1 of a stream, as int64 bit patterns."""
    key = _as_i64(stream_key(seed, name))
    i = torch.arange(start, start + count, dtype=torch.int64, device=device)
    return mix64(i * _GAMMA_I + key)


def uniform(seed: int, name: str, start: int, count: int, device="cpu") -> torch.Tensor:
    """Uniform deviates in the open interval (0, 1), fp64, from the top 53 bits."""
    u = raw_u64(seed, name, start, count, device)
    return (_lsr(u, 11).to(torch.float64) + 0.5) * (2.0 ** -53)


def normal(seed: int, name: str, start: int, count: int, device="cpu",
           chunk: int = 1 << 24) -> torch.Tensor:
    """Standard normal deviates (fp64); element i uses uniforms 2i and 2i+1."""
    out = torch.empty(count, dtype=torch.float64, device=device)
    for c0 in range(0, count, chunk):
        n = min(chunk, count - c0)
        u = uniform(seed, name, 2 * (start + c0), 2 * n, device).view(n, 2)
        out[c0:c0 + n] = torch.sqrt(-2.0 * torch.log(u[:, 0])) * torch.cos(2.0 * torch.pi * u[:, 1])
    return out


def randint_below(seed: int, name: str, start: int, count: int, bound: int,
                  device="cpu") -> torch.Tensor:
    """Integers in [0, bound) (floor of a uniform times bound), int64."""
    return torch.clamp((uniform(seed, name, start, count, device) * bound).to(torch.int64), 0, bound - 1)
