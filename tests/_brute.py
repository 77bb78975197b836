"""Brute-force restatement of the expert-choice MoE layer with Python scalars.

Used only to pin the oracle on tiny inputs. It shares nothing with the oracle: no
numpy matmul, no sort. Selection is decided by counting, for each (token, expert),
how many tokens of the same group beat it under (fp32 score descending, token index
ascending); the token is chosen iff fewer than C do.
"""

import math
import struct


def _f32(v):
    return struct.unpack("f", struct.pack("f", v))[0]


def _dot(a, b):
    s = 0.0
    for u, v in zip(a, b):
        s += u * v
    return s


def brute_layer(x, W_r, W1, W3, W2, C, score_fn="softmax", combine="raw",
                route_scale=1.0, n_segments=1, router_bias=None):
    """All arguments are nested Python lists of floats (or numpy arrays indexable the
    same way). Returns (out [T][d], scores32 [T][E], chosen[e] = set of tokens)."""
    T = len(x)
    d = len(x[0])
    E = len(W_r[0])
    F = len(W1[0][0])
    S = T // n_segments
    cols = [[W_r[k][e] for k in range(d)] for e in range(E)]
    logits = [[_dot(x[t], cols[e]) for e in range(E)] for t in range(T)]
    if router_bias is not None:
        for t in range(T):
            for e in range(E):
                logits[t][e] += router_bias[t // S][e]
    p = []
    for t in range(T):
        if score_fn == "softmax":
            m = max(logits[t])
            ex = [math.exp(v - m) for v in logits[t]]
            z = sum(ex)
            p.append([v / z for v in ex])
        else:
            p.append([1.0 / (1.0 + math.exp(-v)) for v in logits[t]])
    s32 = [[_f32(v) for v in row] for row in p]
    chosen = []
    for e in range(E):
        sel = set()
        for t in range(T):
            g0 = (t // S) * S
            beat = 0
            for u in range(g0, g0 + S):
                if s32[u][e] > s32[t][e] or (s32[u][e] == s32[t][e] and u < t):
                    beat += 1
            if beat < C:
                sel.add(t)
        chosen.append(sel)
    out = [[0.0] * d for _ in range(T)]
    for t in range(T):
        mine = [e for e in range(E) if t in chosen[e]]
        tot = sum(p[t][e] for e in mine)
        for e in mine:  # ascending expert order
            w = p[t][e] if combine == "raw" else route_scale * p[t][e] / tot
            h = []
            for j in range(F):
                g = sum(x[t][k] * W1[e][k][j] for k in range(d))
                u = sum(x[t][k] * W3[e][k][j] for k in range(d))
                h.append(g / (1.0 + math.exp(-g)) * u)
            for i in range(d):
                out[t][i] += w * sum(h[j] * W2[e][j][i] for j in range(F))
    return out, s32, chosen
