"""fp64 CPU oracle for gpt-oss-style grouped-query attention with sinks.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg may import this package. It shares no code with the
CUDA library: the arithmetic lives in ``gptoss_attn_oracle.c`` (plain loops,
fp64), wrapped here with ctypes, and ``brute.py`` holds a second, literal
pure-Python transcription used to pin it on tiny inputs.

Functions take numpy arrays of exact input values (bf16 inputs converted to
fp64 without rounding) and return fp64 results.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

NQ, NKV, D = 64, 8, 64
ROPE_THETA = 150000.0
SCALE = 0.125

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int64)
        i32, f64 = ctypes.c_int, ctypes.c_double
        lib.oracle_rope_rows.argtypes = [dp, dp, ctypes.c_int64, i32, dp]
        lib.oracle_rope_yarn.argtypes = [dp, f64, f64, f64, f64, f64, dp]
        lib.oracle_prefill.argtypes = [dp, dp, dp, dp, dp, i32, i32, i32, i32, dp]
        lib.oracle_prefill_rows.argtypes = [dp, dp, dp, dp, dp, i32, i32, i32, i32, ip,
                                            ctypes.c_int64, dp]
        lib.oracle_decode.argtypes = [dp, dp, dp, dp, ip, i32, i32, i32, i32, dp]
        _lib = lib
    return _lib


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a, t=ctypes.c_double):
    return a.ctypes.data_as(ctypes.POINTER(t))


ROPE_MODES = {"plain": 0, "yarn": 1}


def _mode(rope):
    if rope not in ROPE_MODES:
        raise ValueError("rope must be one of %s" % sorted(ROPE_MODES))
    return ROPE_MODES[rope]


def rope(x, pos, rope="plain"):
    """Rotate head vectors ``x[..., 64]`` by positions ``pos`` (shape ``x.shape[:-1]``).
    ``rope="yarn"`` uses the YaRN frequencies and attention factor of the model."""
    x = _f64(x)
    p = _f64(np.broadcast_to(pos, x.shape[:-1]))
    y = np.empty_like(x)
    _load().oracle_rope_rows(_ptr(x), _ptr(p), x.size // D, _mode(rope), _ptr(y))
    return y


def rope_yarn(x, p, factor=32.0, original=4096.0, beta_fast=32.0, beta_slow=1.0):
    """One head vector ``x[64]`` rotated at position ``p`` by YaRN with the given
    scaling factor, original context length and betas."""
    x = _f64(x).reshape(D)
    y = np.empty_like(x)
    _load().oracle_rope_yarn(_ptr(x), float(p), float(factor), float(original), float(beta_fast),
                             float(beta_slow), _ptr(y))
    return y


def _norm_window(window, seqlen):
    return int(window) if window is not None else 0


def prefill(q, k, v, sinks, pos, window, rope="plain"):
    """Attention output ``[B, S, 64, 64]`` (fp64) for every query row.

    q: [B, S, 64, 64]; k, v: [B, S, 8, 64]; sinks: [64]; pos: [B, S];
    window <= 0 means full causal, W > 0 the W-key sliding window;
    rope "plain" or "yarn".
    """
    q, k, v, sinks, pos = _f64(q), _f64(k), _f64(v), _f64(sinks), _f64(pos)
    B, S = q.shape[0], q.shape[1]
    out = np.empty((B, S, NQ, D), dtype=np.float64)
    _load().oracle_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(sinks), _ptr(pos), B, S,
                           _norm_window(window, S), _mode(rope), _ptr(out))
    return out


def prefill_rows(q_rows, k, v, sinks, pos, window, rows, rope="plain"):
    """Attention output ``[n, 64, 64]`` for the query rows ``rows`` = [(b, i), ...].

    ``q_rows[n]`` is the query vector block ``[64, 64]`` of row ``rows[n]``;
    k, v: [B, S, 8, 64]; pos: [B, S].
    """
    q, k, v, sinks, pos = _f64(q_rows), _f64(k), _f64(v), _f64(sinks), _f64(pos)
    B, S = k.shape[0], k.shape[1]
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2))
    assert q.shape == (r.shape[0], NQ, D)
    out = np.empty((r.shape[0], NQ, D), dtype=np.float64)
    _load().oracle_prefill_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(sinks), _ptr(pos), B, S,
                                _norm_window(window, S), _mode(rope), _ptr(r, ctypes.c_int64),
                                r.shape[0], _ptr(out))
    return out


def decode(q, kcache, vcache, sinks, lengths, window, rope="plain"):
    """One decode step, ``[B, 64, 64]`` fp64.

    q: [B, 64, 64] un-rotated (rotated here at position len-1);
    kcache, vcache: [B, max_len, 8, 64], kcache already rotated; lengths: [B].
    """
    q, kc, vc, sinks = _f64(q), _f64(kcache), _f64(vcache), _f64(sinks)
    L = np.ascontiguousarray(np.asarray(lengths, dtype=np.int64))
    B, max_len = kc.shape[0], kc.shape[1]
    out = np.empty((B, NQ, D), dtype=np.float64)
    _load().oracle_decode(_ptr(q), _ptr(kc), _ptr(vc), _ptr(sinks), _ptr(L, ctypes.c_int64), B,
                          max_len, int(window), _mode(rope), _ptr(out))
    return out
