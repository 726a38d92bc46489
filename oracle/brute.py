"""Pure-Python loop versions of the layer for tiny inputs (test infrastructure only).

Written independently of ``moe_lora_ref``: its own stored-precision decoding (via
``struct`` for bf16 and ``math.ldexp`` for e4m3), its own selection (a full sort of
each logit row), its own counting sort and scalar loops for every product.  Used to
pin the vectorised oracle; meant for M, E, H, I, r of a few units to a few tens.
"""
from __future__ import annotations

import math
import struct


def bf16(u: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (int(u) & 0xFFFF) << 16))[0]


def e4m3(c: int) -> float:
    c = int(c) & 0xFF
    s = -1.0 if c & 0x80 else 1.0
    e, m = (c >> 3) & 0xF, c & 7
    if e == 15 and m == 7:
        return math.nan
    if e == 0:
        return s * math.ldexp(m, -9)
    return s * math.ldexp(8 + m, e - 10)


def decode(raw, dtype: str):
    """Nested lists of Python floats from a numpy array of raw storage."""
    f = {"bf16": bf16, "e4m3": e4m3, "f32": float}[dtype]
    if hasattr(raw, "ndim") and raw.ndim > 1:
        return [decode(r, dtype) for r in raw]
    return [f(v) for v in raw]


def dot(a, b) -> float:
    s = 0.0
    for u, v in zip(a, b):
        s += u * v
    return s


def matvec(w_rows, v):
    """w_rows [n_out][n_in] (each row one output feature) times v [n_in]."""
    return [dot(row, v) for row in w_rows]


def vecmat_t(v, rows):
    """sum_i v[i] * rows[i] for rows [len(v)][n]."""
    out = [0.0] * len(rows[0]) if rows else []
    for i, coef in enumerate(v):
        for n, val in enumerate(rows[i]):
            out[n] += coef * val
    return out


def route(x, w_router, bias, k):
    """logits, top-k ids (descending, ties to lower index), renormalised weights."""
    logits, ids, ws = [], [], []
    for xt in x:
        lt = [dot(xt, we) + (bias[e] if bias is not None else 0.0) for e, we in enumerate(w_router)]
        ranked = sorted(range(len(lt)), key=lambda e: (-lt[e], e))
        top = ranked[:k]
        mx = max(lt)
        ex_all = [math.exp(v - mx) for v in lt]
        tot_all = sum(ex_all)
        p = [v / tot_all for v in ex_all]
        sel = [p[e] for e in top]
        z = sum(sel)
        logits.append(lt)
        ids.append(top)
        ws.append([v / z for v in sel])
    return logits, ids, ws


def sort_pairs(ids, adapters, E, L):
    k = len(ids[0]) if ids else 0
    buckets = [[] for _ in range(E * (L + 1))]
    for t, row in enumerate(ids):
        ap = adapters[t] if adapters[t] >= 0 else L
        for j, e in enumerate(row):
            buckets[e * (L + 1) + ap].append(t * k + j)
    pairs, offs = [], [0]
    for b in buckets:
        pairs.extend(b)
        offs.append(len(pairs))
    return pairs, offs


def silu(g: float) -> float:
    return g / (1.0 + math.exp(-g))


def moe_layer(x, ids, ws, adapters, I, experts, lora, split=False, scale_gu=1.0, scale_d=1.0):
    """experts[e] = (w_gu rows [2I][H], w_d rows [H][I], s_gu, s_d);
    lora[(a, e)] = (A_gu [r][H], B_gu [r][2I], A_d [r][I], B_d [r][H]); all floats.
    split: A_gu = (A_gate [r][H], A_up [r][H]) and B_gu = (B_gate [r][I], B_up [r][I]),
    each feature of the gate half taking its delta from the gate adapter, the up half
    from the up adapter.  scale_gu / scale_d multiply each projection's delta."""
    H = len(x[0])
    y = []
    for t, xt in enumerate(x):
        acc = [0.0] * H
        a = adapters[t]
        for j, e in enumerate(ids[t]):
            w_gu, w_d, s_gu, s_d = experts[e]
            h = [s_gu * v for v in matvec(w_gu, xt)]
            if a >= 0:
                ag, bg, _, _ = lora[(a, e)]
                if split:
                    d = vecmat_t(matvec(ag[0], xt), bg[0]) + vecmat_t(matvec(ag[1], xt), bg[1])
                else:
                    d = vecmat_t(matvec(ag, xt), bg)
                h = [u + scale_gu * v for u, v in zip(h, d)]
            act = [silu(h[i]) * h[I + i] for i in range(I)]
            o = [s_d * v for v in matvec(w_d, act)]
            if a >= 0:
                _, _, ad, bd = lora[(a, e)]
                d = vecmat_t(matvec(ad, act), bd)
                o = [u + scale_d * v for u, v in zip(o, d)]
            for n in range(H):
                acc[n] += ws[t][j] * o[n]
        y.append(acc)
    return y


def dense_lora(x, w, lora_a, lora_b, token_adapter):
    """y_t = W x_t + (A_a x_t) B_a per token (no segments: the per-token definition)."""
    y = []
    for t, xt in enumerate(x):
        yt = matvec(w, xt)
        a = token_adapter[t]
        if a >= 0:
            d = vecmat_t(matvec(lora_a[a], xt), lora_b[a])
            yt = [u + v for u, v in zip(yt, d)]
        y.append(yt)
    return y
