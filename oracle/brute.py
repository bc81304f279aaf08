"""Pure-Python (``math`` only) restatement of one decoder block, for tiny shapes.

TEST INFRASTRUCTURE ONLY.  It is an independent second writing of the same
definition as ``oracle.block`` -- lists of floats and explicit loops, no
NumPy -- so that a transposed operand, a wrong index or a dropped term in
either one shows up as a disagreement.  Pages are cited as in
``oracle.block``.
"""

from __future__ import annotations

import math


def _matvec(Wrows, x):
    """``W x`` with ``W`` given as a list of output rows ([out][in])."""
    return [sum(w * xi for w, xi in zip(row, x)) for row in Wrows]


def _rmsnorm(x, g, eps):
    ms = sum(v * v for v in x) / len(x)
    r = 1.0 / math.sqrt(ms + eps)
    return [gi * (v * r) for gi, v in zip(g, x)]


def _rope(vec, p, theta, style):
    hd = len(vec)
    half = hd // 2
    out = [0.0] * hd
    for i in range(half):
        ang = p * theta ** (-(2.0 * i) / hd)
        c, s = math.cos(ang), math.sin(ang)
        if style == "half":
            a, b = vec[i], vec[i + half]
            out[i] = a * c - b * s
            out[i + half] = b * c + a * s
        else:
            a, b = vec[2 * i], vec[2 * i + 1]
            out[2 * i] = a * c - b * s
            out[2 * i + 1] = a * s + b * c
    return out


def block_forward(d, W, x, k_cache, v_cache):
    """One sequence.  ``x``: list of L rows (positions len(k_cache) ..).

    ``k_cache[j][g]`` / ``v_cache[j][g]``: cached (rotated) key / value of
    position ``j`` and KV head ``g``; both lists are extended in place.
    Returns the list of output rows.
    """
    nh, nkv, hd = d.n_heads, d.n_kv_heads, d.head_dim
    n_rep = nh // nkv
    p0 = len(k_cache)
    qs = []
    for i, row in enumerate(x):
        p = p0 + i
        h = _rmsnorm(row, W["attn_norm"], d.eps)
        q = _matvec(W["wq"], h)
        k = _matvec(W["wk"], h)
        v = _matvec(W["wv"], h)
        qh = [_rope(q[a * hd:(a + 1) * hd], p, d.rope_theta, d.rope_style) for a in range(nh)]
        kh = [_rope(k[g * hd:(g + 1) * hd], p, d.rope_theta, d.rope_style) for g in range(nkv)]
        vh = [v[g * hd:(g + 1) * hd] for g in range(nkv)]
        k_cache.append(kh)
        v_cache.append(vh)
        qs.append(qh)
    outs = []
    for i, row in enumerate(x):
        p = p0 + i
        o = []
        for a in range(nh):
            g = a // n_rep
            scores = []
            for j in range(p + 1):
                dot = sum(qq * kk for qq, kk in zip(qs[i][a], k_cache[j][g]))
                scores.append(dot / math.sqrt(hd))
            mx = max(scores)
            w = [math.exp(s - mx) for s in scores]
            tot = sum(w)
            for t in range(hd):
                o.append(sum(w[j] / tot * v_cache[j][g][t] for j in range(p + 1)))
        attn = _matvec(W["wo"], o)
        xm = [a + b for a, b in zip(row, attn)]
        h2 = _rmsnorm(xm, W["ffn_norm"], d.eps)
        gate = _matvec(W["w1"], h2)
        up = _matvec(W["w3"], h2)
        m = [gv / (1.0 + math.exp(-gv)) * uv for gv, uv in zip(gate, up)]
        down = _matvec(W["w2"], m)
        outs.append([a + b for a, b in zip(xm, down)])
    return outs
