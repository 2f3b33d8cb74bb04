"""Pins of the fp64 backward oracle (oracle/backward.py), CPU only.

The backward pass is the next workload after prefill and decode; these pins
fix its gradients before any kernel computes them:
  * central finite differences of L = sum(dO * out) through the C forward
    oracle (a different implementation of the forward), at random positions,
    full-causal and windowed;
  * the sink gradient against its closed form when V is constant
    (out = c (1 - p_sink), so dL/dsigma = -sum_i (dO_i . c) p_sink,i (1 - p_sink,i));
  * with sigma = -inf and positions 0, the gradients of plain softmax
    attention from torch autograd (fp64) on keys and values repeated per group.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward

NQ, NKV, D = 64, 8, 64


def _inputs(rng, S, scale=0.6):
    q = rng.normal(size=(1, S, NQ, D)) * scale
    k = rng.normal(size=(1, S, NKV, D)) * scale
    v = rng.normal(size=(1, S, NKV, D))
    sinks = rng.normal(size=NQ)
    return q, k, v, sinks


@pytest.mark.parametrize("window", [0, 3])
def test_gradients_match_finite_differences(window):
    rng = np.random.default_rng(11 + window)
    S = 6
    q, k, v, sinks = _inputs(rng, S)
    pos = np.array([[5, 17, 100, 1000, 60000, 7]], dtype=np.float64)
    dout = rng.normal(size=(1, S, NQ, D))
    dq, dk, dv, dsinks = backward.prefill_backward(q, k, v, sinks, pos, window, dout)

    def loss(q_, k_, v_, s_):
        return float(np.sum(dout * oracle.prefill(q_, k_, v_, s_, pos, window)))

    h = 1e-5
    checks = [("q", q, dq), ("k", k, dk), ("v", v, dv)]
    for name, x, g in checks:
        for _ in range(12):
            idx = tuple(int(rng.integers(0, n)) for n in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd = (loss(*args_p, sinks) - loss(*args_m, sinks)) / (2 * h)
            assert abs(fd - g[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, g[idx])
    for hh in range(0, NQ, 7):
        sp, sm = sinks.copy(), sinks.copy()
        sp[hh] += h
        sm[hh] -= h
        fd = (loss(q, k, v, sp) - loss(q, k, v, sm)) / (2 * h)
        assert abs(fd - dsinks[hh]) <= 1e-6 * max(1.0, abs(fd)), (hh, fd, dsinks[hh])


def test_sink_gradient_closed_form_with_constant_values():
    rng = np.random.default_rng(5)
    S = 9
    q, k, _, sinks = _inputs(rng, S)
    cval = rng.normal(size=D)
    v = np.broadcast_to(cval, (1, S, NKV, D)).copy()
    pos = np.arange(S, dtype=np.float64)[None, :]
    dout = rng.normal(size=(1, S, NQ, D))
    window = 4
    _, _, _, dsinks = backward.prefill_backward(q, k, v, sinks, pos, window, dout)
    out = oracle.prefill(q, k, v, sinks, pos, window)
    # out_i = c (1 - p_sink,i): recover p_sink from the forward oracle's output
    p_sink = 1.0 - out[0] @ cval / (cval @ cval)            # [S, 64]
    want = -np.sum((dout[0] @ cval) * p_sink * (1.0 - p_sink), axis=0)
    assert np.allclose(dsinks, want, rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("window", [0, 2])
def test_no_sink_matches_autograd_attention(window):
    rng = np.random.default_rng(21)
    S = 7
    q, k, v, _ = _inputs(rng, S)
    sinks = np.full(NQ, -np.inf)
    pos = np.zeros((1, S))
    dout = rng.normal(size=(1, S, NQ, D))
    dq, dk, dv, dsinks = backward.prefill_backward(q, k, v, sinks, pos, window, dout)
    assert np.all(dsinks == 0.0)

    tq = torch.tensor(q, requires_grad=True)
    tk = torch.tensor(k, requires_grad=True)
    tv = torch.tensor(v, requires_grad=True)
    qh = tq[0].transpose(0, 1)                                   # [64, S, 64]
    kh = tk[0].transpose(0, 1).repeat_interleave(NQ // NKV, 0)   # head h reads kv head h // 8
    vh = tv[0].transpose(0, 1).repeat_interleave(NQ // NKV, 0)
    i = torch.arange(S)[:, None]
    j = torch.arange(S)[None, :]
    mask = (j <= i) & ((j > i - window) if window > 0 else torch.ones_like(j <= i))
    o = torch.nn.functional.scaled_dot_product_attention(qh, kh, vh, attn_mask=mask, scale=0.125)
    (o * torch.tensor(dout[0]).transpose(0, 1)).sum().backward()
    assert np.allclose(dq, tq.grad.numpy(), rtol=1e-10, atol=1e-12)
    assert np.allclose(dk, tk.grad.numpy(), rtol=1e-10, atol=1e-12)
    assert np.allclose(dv, tv.grad.numpy(), rtol=1e-10, atol=1e-12)


MUTANTS = [
    ("dqr[:, h] = ds @ kr[:, g] / 8.0", "dqr[:, h] = ds @ kr[:, g] / 4.0"),        # scale dropped
    ("return np.concatenate([y1 * c + y2 * s, y2 * c - y1 * s], axis=-1)",
     "return np.concatenate([y1 * c - y2 * s, y2 * c + y1 * s], axis=-1)"),     # R instead of R^T
    ("dsinks[h] -= np.sum(ps * dd)", "dsinks[h] += np.sum(ps * dd)"),            # sink sign
    ("ds = np.where(vis, p * (dp - dd[:, None]), 0.0)",
     "ds = np.where(vis, p * dp, 0.0)"),                                         # softmax Jacobian
    ("g = h // GROUP", "g = h % NKV"),                                           # GQA mapping
    ("dkr[:, g] += ds.T @ qr[:, h] / 8.0", "dkr[:, g] = ds.T @ qr[:, h] / 8.0"),  # no group sum
]


@pytest.mark.parametrize("old,new", MUTANTS)
def test_planted_mistakes_are_caught(old, new):
    """Each plausible slip in the backward oracle moves its gradients by far more
    than the finite-difference pin above allows (the unmutated oracle meets it)."""
    import inspect
    import types
    src = inspect.getsource(backward)
    assert src.count(old) == 1, old
    mod = types.ModuleType("backward_mutant")
    exec(compile(src.replace(old, new), "backward_mutant", "exec"), mod.__dict__)
    rng = np.random.default_rng(3)
    S, window = 5, 0
    q, k, v, sinks = _inputs(rng, S)
    pos = np.array([[3, 40, 900, 20000, 1]], dtype=np.float64)
    dout = rng.normal(size=(1, S, NQ, D))
    good = backward.prefill_backward(q, k, v, sinks, pos, window, dout)
    bad = mod.prefill_backward(q, k, v, sinks, pos, window, dout)
    assert any(not np.allclose(a, b, rtol=1e-6, atol=1e-9) for a, b in zip(good, bad))
