"""Literal pure-Python fp64 transcription of the attention-with-sinks forward.

TEST INFRASTRUCTURE, for tiny inputs (S <= 16) only. It is written
independently of ``gptoss_attn_oracle.c`` and follows the order in which the
gpt-oss modeling code is quoted on the inteligile "gpt-oss-120b" techniques
map: rotate q and k with the half-split rotary embedding (row "Partial
RoPE"), form the full score matrix per query head with the key/value head
chosen by grouping (row "Grouped-query attention"), mask it causally or with
the sliding window (rows "Sliding-window attention", "Interleaved ..."),
append the sink logit as one more column (row "Learnable attention sink"),
take a softmax over that extended row, drop the sink column and multiply by
V. Sums use ``math.fsum``; nothing is rescaled online.
"""
from __future__ import annotations

import math

NQ, NKV, D = 64, 8, 64
THETA = 150000.0


def _rotate(x, p):
    half = D // 2
    first, second = x[:half], x[half:]
    out_first, out_second = [], []
    for k in range(half):
        ang = p * THETA ** (-(2.0 * k) / D)
        c, s = math.cos(ang), math.sin(ang)
        out_first.append(first[k] * c - second[k] * s)
        out_second.append(second[k] * c + first[k] * s)
    return out_first + out_second


def attention(q, k, v, sinks, pos, window):
    """q: [B][S][64][64], k/v: [B][S][8][64] nested lists (or arrays); returns nested lists."""
    B, S = len(q), len(q[0])
    groups = NQ // NKV
    out = []
    for b in range(B):
        kr = [[_rotate(list(k[b][j][g]), float(pos[b][j])) for g in range(NKV)] for j in range(S)]
        ob = []
        for i in range(S):
            oi = []
            for h in range(NQ):
                g = h // groups
                qr = _rotate(list(q[b][i][h]), float(pos[b][i]))
                row = []
                for j in range(S):
                    visible = j <= i and (window <= 0 or j > i - window)
                    if visible:
                        row.append(math.fsum(qr[e] * kr[j][g][e] for e in range(D)) / math.sqrt(D))
                    else:
                        row.append(-math.inf)
                row.append(float(sinks[h]))          # the sink column
                mx = max(row)
                if mx == -math.inf:
                    oi.append([0.0] * D)
                    continue
                ex = [math.exp(x - mx) if x != -math.inf else 0.0 for x in row]
                den = math.fsum(ex)
                probs = [e / den for e in ex][:-1]   # drop the sink column
                oi.append([math.fsum(probs[j] * float(v[b][j][g][e]) for j in range(S))
                           for e in range(D)])
            ob.append(oi)
        out.append(ob)
    return out
