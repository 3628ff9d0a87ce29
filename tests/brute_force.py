"""Pure-Python brute force of bifocal attention, for pinning the fp64 oracle.

Written independently of the oracle: positions rotate complex numbers
z_k = x_k + i x_{k+D/2} by e^{i p omega_k} (cmath), the factor G is found by
counting up rather than by a ceiling formula, and the softmax is a loop with
math.exp. Every score is formed one (i, j) pair at a time. Small inputs only.
"""
from __future__ import annotations

import cmath
import math


def factor_by_search(L: int, w_pretrained: int) -> int:
    """Smallest integer G >= 1 with G * w_pretrained >= L."""
    g = 1
    while g * w_pretrained < L:
        g += 1
    return g


def _rot(x, pos, theta, freq_scale):
    D = len(x)
    P = D // 2
    y = [0.0] * D
    for kk in range(P):
        w = theta ** (-(2.0 * kk) / D) * freq_scale
        z = complex(x[kk], x[kk + P]) * cmath.exp(1j * pos * w)
        y[kk] = z.real
        y[kk + P] = z.imag
    return y


def _dot(a, b):
    return math.fsum(x * y for x, y in zip(a, b))


def brute_bifocal(q, k, v, w0, w_pretrained, theta, mode, scale=None, pos_offset=0):
    """q: [L][Hq][D], k, v: [L][Hkv][D] nested lists (batch 1).

    Returns out [L][Hq][D] and lse [Hq][L].
    """
    L = len(q)
    hq, D = len(q[0]), len(q[0][0])
    hkv = len(k[0])
    grp = hq // hkv
    G = factor_by_search(L, w_pretrained)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    out = [[None] * hq for _ in range(L)]
    lse = [[None] * L for _ in range(hq)]
    for h in range(hq):
        kvh = h // grp
        for i in range(L):
            pi = i + pos_offset
            scores = []
            for j in range(i + 1):
                pj = j + pos_offset
                if i - j < w0:
                    a = _rot(q[i][h], pi, theta, 1.0)
                    b = _rot(k[j][kvh], pj, theta, 1.0)
                elif mode == "freq_interp":
                    a = _rot(q[i][h], pi, theta, 1.0 / G)
                    b = _rot(k[j][kvh], pj, theta, 1.0 / G)
                elif mode == "pos_alias":
                    a = _rot(q[i][h], pi // G, theta, 1.0)
                    b = _rot(k[j][kvh], pj // G, theta, 1.0)
                else:
                    raise ValueError(mode)
                scores.append(scale * _dot(a, b))
            m = max(scores)
            ex = [math.exp(s - m) for s in scores]
            tot = math.fsum(ex)
            out[i][h] = [math.fsum(ex[j] * v[j][kvh][d] for j in range(i + 1)) / tot for d in range(D)]
            lse[h][i] = m + math.log(tot)
    return out, lse
