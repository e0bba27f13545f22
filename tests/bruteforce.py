"""Independent brute-force restatements used to pin the oracle (tiny inputs only).

Nothing here is imported by the oracle or by the library. Everything is plain Python over
exact rationals or Python floats, written without reference to the oracle's code: the fp32
rounding picks the nearest of the candidate fp32 neighbours by exact comparison, top-k sorts
with an explicit key, experts are evaluated with explicit loops and ``math.exp``.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np


def f32_neighbors(c: np.float32):
    return (np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf)))


def nearest_f32(v: Fraction) -> float:
    """Nearest fp32 to the exact rational v, ties to the even significand (brute force)."""
    with np.errstate(over="ignore"):
        c = np.float32(float(v))  # within one fp32 step of the answer
    cands = set()
    for a in f32_neighbors(c):
        for b in f32_neighbors(a):
            if np.isfinite(b):
                cands.add(float(b))
    best = None
    for cnd in sorted(cands):
        dist = abs(Fraction(cnd) - v)
        if best is None or dist < best[0]:
            best = (dist, cnd)
        elif dist == best[0]:
            even_new = int(np.float32(cnd).view(np.uint32)) & 1 == 0
            if even_new:
                best = (dist, cnd)
    return best[1]


def exact_logit(xrow, wrow, off=None) -> float:
    s = Fraction(0)
    for a, b in zip(xrow, wrow):
        s += Fraction(float(a)) * Fraction(float(b))
    if off is not None:
        s += Fraction(float(off))
    return nearest_f32(s)


def exp_enclosure(y: Fraction, terms: int = 60):
    """Rigorous rational enclosure [lo, hi] of e**y for |y| <= 1 by Taylor series + remainder."""
    assert abs(y) <= 1
    s = Fraction(0)
    term = Fraction(1)
    for n in range(terms):
        s += term
        term = term * y / (n + 1)
    # remainder |R| <= |y|^N / N! * e (|y| <= 1), with N = terms
    rem = abs(term) * 3
    return s - rem, s + rem


def sigmoid_key(l32: float, b32: float) -> float:
    """Nearest fp32 of sigma(l) + b via a rational enclosure of exp(-l) (|l| small or large)."""
    l = Fraction(float(l32))
    b = Fraction(float(b32))
    if l == 0:
        return nearest_f32(Fraction(1, 2) + b)
    # e^{-l} = (e^{-l/2^m})^(2^m) with |l/2^m| <= 1
    m = 0
    while abs(l) / (2 ** m) > 1:
        m += 1
    lo, hi = exp_enclosure(-l / (2 ** m))
    for _ in range(m):
        lo, hi = lo * lo, hi * hi
    # sigma decreasing in e^{-l}
    s_lo = 1 / (1 + hi) + b
    s_hi = 1 / (1 + lo) + b
    a, c = nearest_f32(s_lo), nearest_f32(s_hi)
    assert a == c, "enclosure too wide to decide the rounding"
    return a


def topk_ref(keys_row, k):
    E = len(keys_row)
    return sorted(range(E), key=lambda e: (-float(keys_row[e]), e))[:k]


def silu(z: float) -> float:
    if z < -700:
        return 0.0
    return z / (1.0 + math.exp(-z))


def swiglu_token(x, Wg, Wu, Wd):
    f, d = len(Wg), len(x)
    h = []
    for i in range(f):
        g = sum(float(Wg[i][c]) * float(x[c]) for c in range(d))
        u = sum(float(Wu[i][c]) * float(x[c]) for c in range(d))
        h.append(silu(g) * u)
    return [sum(float(Wd[o][i]) * h[i] for i in range(f)) for o in range(len(Wd))]


def lowrank_token(x, V, s, U):
    r, d = len(V), len(x)
    z = [float(s[j]) * sum(float(V[j][c]) * float(x[c]) for c in range(d)) for j in range(r)]
    return [sum(float(U[o][j]) * z[j] for j in range(r)) for o in range(len(U))]


def layer_bruteforce(cfg, inp):
    """Per-token definition of the whole layer, loops only. Returns idx, w, kept, y, aux."""
    x = inp["x"]
    T, d = x.shape
    E, k = cfg.E, cfg.top_k
    off = inp.get("logit_offset")
    bias = inp.get("select_bias")
    idx = []
    wts = []
    probs_all = []
    for t in range(T):
        l = [exact_logit(x[t], inp["w_router"][e], None if off is None else off[e])
             for e in range(E)]
        if cfg.score == "softmax":
            keys = l
            m = max(l)
            ex = [math.exp(v - m) for v in l]
            z = sum(ex)
            p = [v / z for v in ex]
            pb = p
        else:
            keys = [sigmoid_key(l[e], 0.0 if bias is None else float(bias[e])) for e in range(E)]
            p = [1.0 / (1.0 + math.exp(-v)) for v in l]
            z = sum(p)
            pb = [v / z for v in p]
        sel = topk_ref(keys, k)
        w = [p[e] for e in sel]
        if cfg.norm_topk:
            sw = sum(w)
            w = [v / sw for v in w]
        idx.append(sel)
        wts.append(w)
        probs_all.append(pb)
    # capacity in token order
    cf = float(np.float32(cfg.capacity_factor))
    C = math.ceil(Fraction(cf) * T * k / E) if cf > 0 else None
    seen = [0] * E
    kept = []
    for t in range(T):
        row = []
        for j in range(k):
            e = idx[t][j]
            row.append(C is None or seen[e] < C)
            seen[e] += 1
        kept.append(row)
    y = []
    for t in range(T):
        acc = [0.0] * d
        for s_ in range(cfg.n_shared):
            v = swiglu_token(x[t], inp["ws_gate"][s_], inp["ws_up"][s_], inp["ws_down"][s_])
            acc = [a + b for a, b in zip(acc, v)]
        for j in range(k):
            if not kept[t][j]:
                continue
            e = idx[t][j]
            if cfg.expert == "swiglu":
                v = swiglu_token(x[t], inp["w_gate"][e], inp["w_up"][e], inp["w_down"][e])
            else:
                v = lowrank_token(x[t], inp["lr_V"][e], inp["lr_s"][e], inp["lr_U"][e])
            acc = [a + wts[t][j] * b for a, b in zip(acc, v)]
        y.append(acc)
    counts = [0] * E
    for t in range(T):
        for e in idx[t]:
            counts[e] += 1
    P = [sum(probs_all[t][e] for t in range(T)) / T for e in range(E)]
    # DeepSeekMoE form: alpha * sum_i f'_i P_i, f'_i = E/(k T) * count_i
    aux = cfg.aux_alpha * sum((E / (k * T)) * counts[e] * P[e] for e in range(E))
    return dict(idx=np.array(idx), w=np.array(wts), kept=np.array(kept), y=np.array(y),
                aux=aux, counts=np.array(counts), C=C)
