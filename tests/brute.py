"""Pure-Python brute force of every step of the CSA / HCA layer.

Written independently of the oracle (lists, `math`, explicit loops, the RoPE
rotation done as complex multiplication) so that the oracle can be checked
against it on tiny inputs.  Same definitions: "DeepSeek-V4-Pro vs Inkling",
component table, rows "Compressed Sparse Attention", "Heavily Compressed
Attention", "Partial RoPE" and "Output gate + sink".
"""
from __future__ import annotations

import cmath
import math


def _freq(i, rope_dim, theta):
    """Frequency of rotary pair i.  `theta` is a base, or a tuple
    (base, s, L, beta, alpha) for YaRN (Peng et al. 2023, section 3): the
    pair turns L * w / (2 pi) times over L tokens; below alpha turns it runs
    s times slower, above beta it is unchanged, linear blend in between."""
    if not isinstance(theta, tuple):
        return theta ** (-(2.0 * i) / rope_dim)
    base, s, L, beta, alpha = theta
    w = base ** (-(2.0 * i) / rope_dim)
    if s <= 1.0:
        return w
    turns = L / (2.0 * math.pi / w)
    if turns < alpha:
        return w / s
    if turns > beta:
        return w
    blend = (turns - alpha) / (beta - alpha)
    return w / s * (1.0 - blend) + w * blend


def temperature(theta):
    """YaRN's factor on the logits, sqrt(1/t) = 0.1 ln s + 1; 1 otherwise."""
    if isinstance(theta, tuple) and theta[1] > 1.0:
        return (1.0 + 0.1 * math.log(theta[1])) ** 2
    return 1.0


def _rot(vec, pos, rope_dim, theta):
    d = len(vec)
    out = list(vec)
    base = d - rope_dim
    for i in range(rope_dim // 2):
        w = _freq(i, rope_dim, theta)
        z = complex(vec[base + 2 * i], vec[base + 2 * i + 1]) * cmath.exp(1j * pos * w)
        out[base + 2 * i] = z.real
        out[base + 2 * i + 1] = z.imag
    return out


def compress(x, g, width, stride, rope_dim, theta, pos_offset=0):
    T = len(x)
    d = len(x[0])
    out = []
    j = 0
    while stride * j + width <= T:
        e = [0.0] * d
        for c in range(d):
            logits = [g[stride * j + u][c] for u in range(width)]
            mx = max(logits)
            ws = [math.exp(v - mx) for v in logits]
            tot = sum(ws)
            e[c] = sum(ws[u] / tot * x[stride * j + u][c] for u in range(width))
        out.append(_rot(e, stride * j + pos_offset, rope_dim, theta))
        j += 1
    return out


def scores(q_idx_t, w_t, k_idx):
    """One query token: q_idx_t [H_I][d_I], w_t [H_I], k_idx [N][d_I]."""
    res = []
    for key in k_idx:
        s = 0.0
        for h, qh in enumerate(q_idx_t):
            dot = sum(a * b for a, b in zip(qh, key))
            s += w_t[h] * (dot if dot > 0 else 0.0)
        res.append(s)
    return res


def topk(sc, n_vis, k):
    order = sorted(range(n_vis), key=lambda j: (-sc[j], j))[:k]
    order.sort()
    return order + [-1] * (k - len(order))


def attend(q, t, rows, sink, scale, rope_dim, theta):
    """q [H][d] unrotated, rows [R][d] rotated; returns [H][d]."""
    out = []
    for h, qv in enumerate(q):
        qr = _rot(qv, t, rope_dim, theta)
        tau = temperature(theta)
        z = [tau * scale * sum(a * b for a, b in zip(qr, r)) for r in rows]
        mx = max(z + [sink[h]])
        ex = [math.exp(v - mx) for v in z]
        den = math.exp(sink[h] - mx) + sum(ex)
        o = [sum(ex[i] * rows[i][c] for i in range(len(rows))) / den for c in range(len(qv))]
        out.append(_rot(o, -t, rope_dim, theta))
    return out


def window(t, W, raw_pos0, n_raw):
    return [u for u in range(max(0, t - W + 1), t + 1) if raw_pos0 <= u < raw_pos0 + n_raw]


def visible(t, n_cmp, width, stride):
    return [j for j in range(n_cmp) if stride * j + width - 1 <= t]
