"""fp64 gradients of gpt-oss-style attention with sinks (TEST INFRASTRUCTURE).

The backward pass of the prefill operation, for a future backward kernel to be
checked against: given the upstream gradient dO of out[b, i, h, :], return
dL/dq, dL/dk, dL/dv (with respect to the un-rotated inputs) and dL/dsinks.

The forward it differentiates is the one the gpt-oss pages define (inteligile
"gpt-oss-120b" techniques map, rows "Grouped-query attention", "Partial RoPE",
"Learnable attention sink", "Sliding-window attention"): half-split rotation
of q and k by their positions, scores q'.k'/8 over the visible keys, the
per-head sink logit sigma_h appended to the row before the softmax and its
probability dropped, out = sum_j p_j v_j. With the softmax over the row
[s_1 .. s_n, sigma] and the sink column carrying a zero value:

    dP_ij   = dO_i . v_j                    (visible j)
    D_i     = sum_j p_ij dP_ij = dO_i . O_i (the sink adds nothing: its value is 0)
    dS_ij   = p_ij (dP_ij - D_i)
    dsigma  = sum_i p_sink,i (0 - D_i)
    dv_j    = sum_i p_ij dO_i               (summed over the 8 heads of a group)
    dq'_i   = sum_j dS_ij k'_j / 8,   dk'_j = sum_i dS_ij q'_i / 8
    dq = R(pos)^T dq',  dk = R(pos)^T dk'   (R^T rotates by the opposite angle)

Plain numpy, fp64, loops over (batch, head) with whole-row matrix products; no
blocking or online rescaling. Only the tests import this module. The pages
print no backward pass: these are the textbook derivatives of the forward
above, and the tests pin them to the forward oracle by finite differences.
"""
from __future__ import annotations

import numpy as np

NQ, NKV, D = 64, 8, 64
GROUP = NQ // NKV
ROPE_THETA = 150000.0


def _angles(pos):
    k = np.arange(D // 2, dtype=np.float64)
    inv = ROPE_THETA ** (-2.0 * k / D)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv
    return np.cos(ang), np.sin(ang)


def _rotate(x, c, s):
    x1, x2 = x[..., : D // 2], x[..., D // 2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def _rotate_back(y, c, s):
    y1, y2 = y[..., : D // 2], y[..., D // 2:]
    return np.concatenate([y1 * c + y2 * s, y2 * c - y1 * s], axis=-1)


def _visible(S, window):
    i = np.arange(S)[:, None]
    j = np.arange(S)[None, :]
    vis = j <= i
    if 0 < window < S:
        vis &= j > i - window
    return vis


def prefill_backward(q, k, v, sinks, pos, window, dout):
    """Gradients (dq [B,S,64,64], dk [B,S,8,64], dv [B,S,8,64], dsinks [64]) of
    L = sum(dout * out) for the prefill operation, all fp64."""
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    sinks = np.asarray(sinks, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    B, S = q.shape[0], q.shape[1]
    vis = _visible(S, window)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dsinks = np.zeros(NQ)
    for b in range(B):
        c, s = _angles(pos[b])                      # [S, 32]
        kr = _rotate(k[b], c[:, None, :], s[:, None, :])   # [S, 8, 64]
        qr = _rotate(q[b], c[:, None, :], s[:, None, :])   # [S, 64, 64]
        dkr = np.zeros((S, NKV, D))
        dqr = np.zeros((S, NQ, D))
        for h in range(NQ):
            g = h // GROUP
            sc = qr[:, h] @ kr[:, g].T / 8.0                # [S, S]
            sc = np.where(vis, sc, -np.inf)
            m = np.maximum(sc.max(axis=1), sinks[h])       # row max, the sink included
            e = np.where(vis, np.exp(sc - m[:, None]), 0.0)
            es = np.exp(sinks[h] - m)
            z = es + e.sum(axis=1)
            p = e / z[:, None]
            ps = es / z
            o = p @ v[b, :, g]                              # [S, 64]
            do = dout[b, :, h]
            dp = do @ v[b, :, g].T                          # [S, S]
            dd = np.sum(do * o, axis=1)                     # D_i
            ds = np.where(vis, p * (dp - dd[:, None]), 0.0)
            dsinks[h] -= np.sum(ps * dd)
            dv[b, :, g] += p.T @ do
            dqr[:, h] = ds @ kr[:, g] / 8.0
            dkr[:, g] += ds.T @ qr[:, h] / 8.0
        dq[b] = _rotate_back(dqr, c[:, None, :], s[:, None, :])
        dk[b] = _rotate_back(dkr, c[:, None, :], s[:, None, :])
    return dq, dk, dv, dsinks
