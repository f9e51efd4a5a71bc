"""Scalar pure-Python restatements for tiny inputs (a few hundred elements).

TEST INFRASTRUCTURE.  These loops take the index formulas and the textbook
softmax one element at a time, so that the NumPy reshapes and broadcasts of
``reference`` can be cross-checked by something structurally different.
Sources are the same as in ``reference``.
"""
from __future__ import annotations

import math


def patchify(latent, pt, ph, pw):
    """out[n][(t'*H' + h')*W' + w'][((c*pt + dt)*ph + dh)*pw + dw]
    = latent[n][c][t'*pt + dt][h'*ph + dh][w'*pw + dw], as nested lists."""
    N = len(latent)
    C = len(latent[0])
    T = len(latent[0][0])
    H = len(latent[0][0][0])
    W = len(latent[0][0][0][0])
    Tg, Hg, Wg = T // pt, H // ph, W // pw
    F = C * pt * ph * pw
    out = [[[0.0] * F for _ in range(Tg * Hg * Wg)] for _ in range(N)]
    for n in range(N):
        for tq in range(Tg):
            for hq in range(Hg):
                for wq in range(Wg):
                    row = (tq * Hg + hq) * Wg + wq
                    for c in range(C):
                        for dt in range(pt):
                            for dh in range(ph):
                                for dw in range(pw):
                                    col = ((c * pt + dt) * ph + dh) * pw + dw
                                    out[n][row][col] = latent[n][c][tq * pt + dt][hq * ph + dh][wq * pw + dw]
    return out


def rope_vector(x, pos, split, theta=10000.0):
    """Rotate one head vector (a list of D floats) at grid position pos = (t', h, w)."""
    out = list(x)
    off = 0
    for p, d in zip(pos, split):
        for i in range(d // 2):
            f = 1.0 / (theta ** ((2 * i) / d))
            a = p * f
            x0, x1 = x[off + 2 * i], x[off + 2 * i + 1]
            out[off + 2 * i] = x0 * math.cos(a) - x1 * math.sin(a)
            out[off + 2 * i + 1] = x0 * math.sin(a) + x1 * math.cos(a)
        off += d
    return out


def attention(q, k, v, scale):
    """One head: q [Lq][D], k and v [Lk][D] lists; returns [Lq][Dv] and lse [Lq]."""
    out, lse = [], []
    for qi in q:
        s = [scale * sum(a * b for a, b in zip(qi, kj)) for kj in k]
        m = max(s)
        p = [math.exp(x - m) for x in s]
        z = sum(p)
        out.append([sum(p[j] * v[j][d] for j in range(len(k))) / z for d in range(len(v[0]))])
        lse.append(m + math.log(z))
    return out, lse


def rms_norm(x, weight, eps):
    """One group: list of floats -> x / sqrt(mean of squares + eps) * weight."""
    ms = sum(a * a for a in x) / len(x)
    r = math.sqrt(ms + eps)
    return [a / r * w for a, w in zip(x, weight)]


def unpatchify(tokens, C, grid, pt, ph, pw):
    """latent[n][c][t'*pt + dt][h'*ph + dh][w'*pw + dw]
    = tokens[n][(t'*H' + h')*W' + w'][((c*pt + dt)*ph + dh)*pw + dw], as nested lists."""
    Tg, Hg, Wg = grid
    N = len(tokens)
    out = [[[[[0.0] * (Wg * pw) for _ in range(Hg * ph)] for _ in range(Tg * pt)] for _ in range(C)]
           for _ in range(N)]
    for n in range(N):
        for tq in range(Tg):
            for hq in range(Hg):
                for wq in range(Wg):
                    row = (tq * Hg + hq) * Wg + wq
                    for c in range(C):
                        for dt in range(pt):
                            for dh in range(ph):
                                for dw in range(pw):
                                    col = ((c * pt + dt) * ph + dh) * pw + dw
                                    out[n][c][tq * pt + dt][hq * ph + dh][wq * pw + dw] = tokens[n][row][col]
    return out
