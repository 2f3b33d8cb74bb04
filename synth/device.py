"""The seeded input recipe of ``synth.inputs``, evaluated with torch on a device.

Same definition, word for word: SplitMix64 word ``i`` of stream ``seed``,
uniform ``((word >> 11) + 1) * 2**-53``, Box-Muller pairs in fp64, fp64 ->
fp32 -> bf16 with round-to-nearest-even. Only the fp64 ``log``/``cos``/``sin``
come from the device's math library instead of the host's, so a value can
differ from the host generator's in its last fp64 bits; after rounding to
fp32 and bf16 that changes a stored value with a probability of the order of
2**-28 per element. It exists so that multi-gigabyte workloads (a 131072-token
prefill holds 67 million query values) are drawn in milliseconds instead of
minutes; the host generator stays the definition.

Integer work is done in int64 with two's-complement wrap-around; logical
right shifts are arithmetic shifts masked to the remaining bits. No attention
arithmetic lives here.
"""
from __future__ import annotations

import math

import torch


def _s64(u: int) -> int:
    """An unsigned 64-bit constant as the signed int64 with the same bits."""
    return u - (1 << 64) if u >= (1 << 63) else u


_GAMMA = _s64(0x9E3779B97F4A7C15)
_MIX1 = _s64(0xBF58476D1CE4E5B9)
_MIX2 = _s64(0x94D049BB133111EB)
_CHUNK = 1 << 24


def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    return (z >> s) & ((1 << (64 - s)) - 1)


def splitmix64(seed: int, start: int, count: int, device) -> torch.Tensor:
    """Words ``start .. start+count-1`` of stream ``seed`` as int64 bit patterns."""
    idx = torch.arange(start + 1, start + count + 1, dtype=torch.int64, device=device)
    z = idx * _GAMMA + _s64(seed & 0xFFFFFFFFFFFFFFFF)
    z = (z ^ _lsr(z, 30)) * _MIX1
    z = (z ^ _lsr(z, 27)) * _MIX2
    return z ^ _lsr(z, 31)


def _normal_chunk(seed: int, first: int, count: int, device) -> torch.Tensor:
    # elements first .. first+count-1 (first even), fp64
    npairs = (count + 1) // 2
    w = splitmix64(seed, first, 2 * npairs, device).view(npairs, 2)
    u = (_lsr(w, 11) + 1).to(torch.float64) * (2.0 ** -53)
    r = torch.sqrt(-2.0 * torch.log(u[:, 0]))
    a = (2.0 * math.pi) * u[:, 1]
    return torch.stack((r * torch.cos(a), r * torch.sin(a)), dim=1).view(-1)[:count]


def bf16_normal(seed: int, shape, device) -> torch.Tensor:
    """N(0,1) values rounded fp64 -> fp32 -> bf16, as a bf16 tensor on ``device``."""
    n = math.prod(shape)
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    for s in range(0, n, _CHUNK):
        c = min(_CHUNK, n - s)
        out[s:s + c] = _normal_chunk(seed, s, c, device).to(torch.float32).to(torch.bfloat16)
    return out.view(*shape)


def bf16_normal_range(seed: int, start: int, count: int, device) -> torch.Tensor:
    """Elements ``start .. start+count-1`` (``start`` even) of the flattened stream."""
    assert start % 2 == 0
    out = torch.empty(count, dtype=torch.bfloat16, device=device)
    for s in range(0, count, _CHUNK):
        c = min(_CHUNK, count - s)
        out[s:s + c] = _normal_chunk(seed, start + s, c, device).to(torch.float32).to(
            torch.bfloat16)
    return out


def f32_normal(seed: int, shape, device) -> torch.Tensor:
    """N(0,1) values rounded fp64 -> fp32, on ``device``."""
    n = math.prod(shape)
    return _normal_chunk(seed, 0, n, device).to(torch.float32).view(*shape)
