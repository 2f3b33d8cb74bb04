"""Counter-based seeded generator for the attention inputs.

Recipe (the same for every consumer):

* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): word ``i`` of stream ``seed`` is the SplitMix64
  output mix of ``seed + (i + 1) * 0x9E3779B97F4A7C15`` (mod 2**64).
* Uniform in (0, 1]: ``((word >> 11) + 1) * 2**-53``.
* Standard normal by Box-Muller in fp64: element ``2p`` is ``r cos(2 pi u2)``
  and element ``2p + 1`` is ``r sin(2 pi u2)`` with ``r = sqrt(-2 ln u1)``,
  ``u1 = U(2p)`` and ``u2 = U(2p + 1)``.
* Storage: fp64 -> fp32 (numpy rounding, to nearest) -> bf16 by
  round-to-nearest-even on the fp32 bit pattern.

Seeds follow ``0x6A77 ^ (config << 24) ^ (layer << 12) ^ tensor_id`` with
tensor ids q=1, k=2, v=3, sinks=4, so every layer of every workload has
independent tensors.

Everything here is numpy integer and elementwise float work; no attention
arithmetic lives in this module.
"""
from __future__ import annotations

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_MIX1 = np.uint64(0xBF58476D1CE4E5B9)
_MIX2 = np.uint64(0x94D049BB133111EB)

TENSOR_Q = 1
TENSOR_K = 2
TENSOR_V = 3
TENSOR_SINKS = 4

_CHUNK = 1 << 22


def seed_for(config: int, layer: int, tensor_id: int) -> int:
    """Seed of one tensor of one layer of one workload."""
    return (0x6A77 ^ (config << 24) ^ (layer << 12) ^ tensor_id) & 0xFFFFFFFFFFFFFFFF


def splitmix64(seed: int, start: int, count: int) -> np.ndarray:
    """Words ``start .. start+count-1`` of the SplitMix64 stream ``seed`` (uint64)."""
    with np.errstate(over="ignore"):
        idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        z = np.uint64(seed) + idx * _GAMMA
        z = (z ^ (z >> np.uint64(30))) * _MIX1
        z = (z ^ (z >> np.uint64(27))) * _MIX2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform01(seed: int, start: int, count: int) -> np.ndarray:
    """Uniform fp64 samples in (0, 1] from words ``start ..`` of stream ``seed``."""
    w = splitmix64(seed, start, count)
    return ((w >> np.uint64(11)) + np.uint64(1)).astype(np.float64) * (2.0 ** -53)


def _normal_chunk(seed: int, first: int, count: int) -> np.ndarray:
    # elements first .. first+count-1; first is even
    npairs = (count + 1) // 2
    u = uniform01(seed, first, 2 * npairs).reshape(npairs, 2)
    r = np.sqrt(-2.0 * np.log(u[:, 0]))
    a = (2.0 * np.pi) * u[:, 1]
    out = np.empty((npairs, 2), dtype=np.float64)
    out[:, 0] = r * np.cos(a)
    out[:, 1] = r * np.sin(a)
    return out.reshape(-1)[:count]


def normal(seed: int, n: int) -> np.ndarray:
    """``n`` standard-normal fp64 samples of stream ``seed``."""
    out = np.empty(n, dtype=np.float64)
    for s in range(0, n, _CHUNK):
        c = min(_CHUNK, n - s)
        out[s:s + c] = _normal_chunk(seed, s, c)
    return out


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    with np.errstate(over="ignore"):
        r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact fp64 values of bf16 bit patterns."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def bf16_normal(seed: int, shape) -> np.ndarray:
    """N(0,1) samples rounded to bf16, as uint16 bit patterns of the given shape."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for s in range(0, n, _CHUNK):
        c = min(_CHUNK, n - s)
        out[s:s + c] = f32_to_bf16_bits(_normal_chunk(seed, s, c).astype(np.float32))
    return out.reshape(shape)


def bf16_normal_range(seed: int, start: int, count: int) -> np.ndarray:
    """Elements ``start .. start+count-1`` (``start`` even) of ``bf16_normal(seed, ...)``
    flattened: the generator is counter-based, so any slice is drawn on its own."""
    assert start % 2 == 0
    out = np.empty(count, dtype=np.uint16)
    for s in range(0, count, _CHUNK):
        c = min(_CHUNK, count - s)
        out[s:s + c] = f32_to_bf16_bits(_normal_chunk(seed, start + s, c).astype(np.float32))
    return out


def f32_normal(seed: int, shape) -> np.ndarray:
    """N(0,1) samples rounded to fp32."""
    return normal(seed, int(np.prod(shape))).astype(np.float32).reshape(shape)


N_Q_HEADS = 64
N_KV_HEADS = 8
HEAD_DIM = 64


def make_prefill_inputs(config: int, layer: int, batch: int, seqlen: int) -> dict:
    """Q, K, V (bf16 bits), sinks (fp32) and positions 0..S-1 of one prefill layer."""
    q = bf16_normal(seed_for(config, layer, TENSOR_Q), (batch, seqlen, N_Q_HEADS, HEAD_DIM))
    k = bf16_normal(seed_for(config, layer, TENSOR_K), (batch, seqlen, N_KV_HEADS, HEAD_DIM))
    v = bf16_normal(seed_for(config, layer, TENSOR_V), (batch, seqlen, N_KV_HEADS, HEAD_DIM))
    sinks = f32_normal(seed_for(config, layer, TENSOR_SINKS), (N_Q_HEADS,))
    pos = np.broadcast_to(np.arange(seqlen, dtype=np.int32), (batch, seqlen)).copy()
    return {"q": q, "k": k, "v": v, "sinks": sinks, "pos": pos}


def make_decode_inputs(config: int, layer: int, batch: int, max_len: int, lengths=None) -> dict:
    """One decode step: q (bf16 bits), K/V caches (bf16 bits), sinks (fp32), lengths (int32).

    The cache contents stand for keys that were rotated when they were written.
    ``lengths`` defaults to a full cache for every sequence.
    """
    q = bf16_normal(seed_for(config, layer, TENSOR_Q), (batch, N_Q_HEADS, HEAD_DIM))
    kc = bf16_normal(seed_for(config, layer, TENSOR_K), (batch, max_len, N_KV_HEADS, HEAD_DIM))
    vc = bf16_normal(seed_for(config, layer, TENSOR_V), (batch, max_len, N_KV_HEADS, HEAD_DIM))
    sinks = f32_normal(seed_for(config, layer, TENSOR_SINKS), (N_Q_HEADS,))
    if lengths is None:
        lengths = np.full(batch, max_len, dtype=np.int32)
    lengths = np.asarray(lengths, dtype=np.int32).reshape(batch)
    return {"q": q, "kcache": kc, "vcache": vc, "sinks": sinks, "len": lengths}
