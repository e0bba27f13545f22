"""Plain, slow CPU oracle of the fine-grained MoE FFN layer forward pass.

TEST INFRASTRUCTURE. This module is the correctness reference for the CUDA library; it is
imported only by the tests, by ``__graft_entry__.smoke()`` and by the benchmark's CPU-baseline
leg. It shares no code with the CUDA path, and nothing in the product calls it.

What it computes (every step evaluated in fp64 on the exact fp32 / bf16 input values):

1. Router logits (Vertex AGI research page and quartz-micro-preview-base card, architecture
   table, row "Router": 6 of 24 experts; Moonfrost, expert card: top-3 routing):
   ``l[t,e] = RN32( sum_i x[t,i] * W_r[e,i] + off[e] )``, the exact real value rounded once to
   fp32 with round-to-nearest-even. ``off`` is an optional per-expert logit offset.
2. Selection keys: softmax scoring uses ``key = l``. Sigmoid scoring with a per-expert selection
   bias (Sutra-1.3B, "48 + 1 experts": sigmoid scoring and balancing through a per-expert bias) uses
   ``key = RN32( sigma(l) + b[e] )``, again the exact real value rounded once.
3. Top-k: the k largest keys; equal keys go to the lower expert index first; slot j is the j-th
   entry of that ranking.
4. Probabilities and combine weights: softmax over all E experts of the fp32 logits, or
   ``sigma(l)`` for sigmoid scoring (the selection bias is not part of the weight). The combine
   weight of slot j is the selected expert's probability, divided by the sum over the k
   selected probabilities when ``norm_topk`` is set.
5. Capacity (Moonfrost, expert card: routing under a per-expert capacity): ``C = ceil(cf * T * k / E)`` over the T tokens
   of the call; ``cf <= 0`` is dropless (dormouse, "dropless MoE": no capacity drops). Per
   expert, routed tokens are ranked by ascending token index; rank >= C is dropped.
6. Permutation grouped by expert (the stacked-expert layout of the Moonfrost card):
   ``offsets`` = exclusive scan of kept counts; kept pair (t, j) on expert e lands in row
   ``offsets[e] + rank``.
7. Experts: SwiGLU ``W_down (silu(W_gate x) * (W_up x))`` with ``silu(z) = z / (1 + e^-z)`` and no
   biases; low-rank (dormouse, "TSCT low-rank experts") ``U (s * (V^T x))``; shared experts
   (always active) are SwiGLU experts on every token, their outputs summed.
8. Combine: ``y[t] = sum_shared + sum_j [kept] w[t,j] * E_{e_j}(x[t])``; dropped slots add 0 and
   the remaining weights are not renormalised.
9. Load-balancing loss (research page, architecture table, row "Router": load-balancing loss with weight 0.01):
   ``L = alpha * E * sum_i f_i * P_i`` with ``f_i = count_i / (T k)`` counted before capacity
   drops, and ``P_i`` the mean over tokens of the token's probability of expert i (for sigmoid
   scoring, ``sigma(l_i)`` normalised over all E experts).
10. Loss-free balancing (dormouse, "dropless MoE": a bias on the router balances the load instead
    of an auxiliary loss, after arXiv 2408.15664): ``b_i <- RN32(b_i + u * sign(mean - count_i))``
    with mean = sum(count) / E, compared exactly on integers; u is the caller's step size (the
    pages give none).

Exactness of steps 1-2: the fp64 evaluation is screened with a rigorous error bound; only the
entries whose enclosure contains an fp32 rounding boundary are recomputed exactly (integer
dyadic arithmetic for step 1, an 80-digit ``decimal`` evaluation for the sigmoid of step 2).
Steps 3-6 are integer work and are exact. Steps 7-9 are fp64 and carry no claim of exactness;
the device path is compared with them within a tolerance.

A per-expert matrix product evaluates the same expert on each of its rows independently; it is
the library primitive standing in for the per-token definition and changes no arithmetic.
"""
from __future__ import annotations

import decimal
import math
from fractions import Fraction
from typing import Dict, Optional

import numpy as np

__all__ = [
    "rn32_dyadic", "rn32_fraction", "router_logits", "selection_keys", "topk",
    "probabilities", "aux_probabilities", "combine_weights", "capacity", "route",
    "permute", "swiglu", "lowrank", "expert_forward", "combine", "aux_loss",
    "layer_forward", "token_output", "bias_update",
]

_U64 = 2.0 ** -53


# ---------------------------------------------------------------------------------------------
# Exact rounding helpers
# ---------------------------------------------------------------------------------------------
def rn32_dyadic(M: int, e: int) -> float:
    """Round the exact value ``M * 2**e`` (M an integer) to the nearest fp32, ties to even.

    Returns the fp32 value as a Python float (exact). Overflow gives +-inf.
    """
    if M == 0:
        return 0.0
    neg = M < 0
    M = -M if neg else M
    lead = M.bit_length() - 1 + e              # exponent of the leading bit
    if lead >= 128:
        return -math.inf if neg else math.inf
    q = max(lead, -126) - 23                    # quantum of fp32 at this magnitude
    sh = q - e
    if sh <= 0:
        R = M << (-sh)
    else:
        R = M >> sh
        rem = M - (R << sh)
        half = 1 << (sh - 1)
        if rem > half or (rem == half and (R & 1)):
            R += 1
    if R.bit_length() + q > 128:                # rounded up to 2**128
        return -math.inf if neg else math.inf
    v = math.ldexp(float(R), q)                 # R < 2**25: exact
    return -v if neg else v


def rn32_fraction(v: Fraction) -> float:
    """Round an exact rational to the nearest fp32, ties to even."""
    if v == 0:
        return 0.0
    neg = v < 0
    a = -v if neg else v
    n, dd = a.numerator, a.denominator
    lead = n.bit_length() - dd.bit_length()
    # adjust so that 2**lead <= a < 2**(lead+1)
    if lead >= 0:
        if n < (dd << lead):
            lead -= 1
    else:
        if (n << -lead) < dd:
            lead -= 1
    if lead >= 128:
        return -math.inf if neg else math.inf
    q = max(lead, -126) - 23
    # R = round(a / 2**q)
    if q >= 0:
        num, den = n, dd << q
    else:
        num, den = n << (-q), dd
    R, rem = divmod(num, den)
    if 2 * rem > den or (2 * rem == den and (R & 1)):
        R += 1
    if R.bit_length() + q > 128:
        return -math.inf if neg else math.inf
    val = math.ldexp(float(R), q)
    return -val if neg else val


def _dyadic(v: float):
    """Exact (M, e) with v = M * 2**e for a finite float."""
    if v == 0.0:
        return 0, 0
    m, ex = math.frexp(v)
    M = int(m * (1 << 53))
    return M, ex - 53


def _exact_dot_rn32(xrow: np.ndarray, wrow: np.ndarray, off: Optional[float]) -> float:
    """RN32 of the exact sum of products (plus offset), by integer dyadic arithmetic."""
    terms = []
    for a, b in zip(xrow.tolist(), wrow.tolist()):
        if a == 0.0 or b == 0.0:
            continue
        Ma, ea = _dyadic(a)
        Mb, eb = _dyadic(b)
        terms.append((Ma * Mb, ea + eb))
    if off is not None and off != 0.0:
        terms.append(_dyadic(off))
    if not terms:
        return 0.0
    emin = min(e for _, e in terms)
    total = 0
    for M, e in terms:
        total += M << (e - emin)
    return rn32_dyadic(total, emin)


def _rn32_certain(v: np.ndarray, bound: np.ndarray):
    """Round fp64 approximations ``v`` to fp32 and report where the result is certain.

    The exact value is known to lie in ``[v - bound, v + bound]``. Rounding is certain when that
    interval lies strictly between the two fp32 rounding boundaries around ``RN32(v)``.
    """
    with np.errstate(over="ignore", invalid="ignore"):
        r = v.astype(np.float32)
        r64 = r.astype(np.float64)
        up = np.nextafter(r, np.float32(np.inf)).astype(np.float64)
        dn = np.nextafter(r, np.float32(-np.inf)).astype(np.float64)
        mid_hi = (r64 + up) * 0.5               # exact: fp32 midpoints fit in fp64
        mid_lo = (r64 + dn) * 0.5
        ok = (v + bound < mid_hi) & (v - bound > mid_lo) & np.isfinite(v) & \
             (np.abs(r64) < 2.0 ** 126)
    return r, ok


# ---------------------------------------------------------------------------------------------
# 1-4. Routing
# ---------------------------------------------------------------------------------------------
def router_logits(x: np.ndarray, w_router: np.ndarray,
                  logit_offset: Optional[np.ndarray] = None) -> np.ndarray:
    """fp32 logits ``RN32(sum_i x[t,i] W_r[e,i] + off[e])``, exact (see module doc, step 1).

    Screen: the fp64 product ``x @ W_r^T`` (+ off) has absolute error at most
    ``gamma_{d+1} * (|x| @ |W_r|^T + |off|)`` whatever the summation order; the bound used is
    twice that, which also covers the rounding of the computed magnitude sum.
    """
    x64 = np.asarray(x, np.float64)
    w64 = np.asarray(w_router, np.float64)
    T, d = x64.shape
    s = x64 @ w64.T
    a = np.abs(x64) @ np.abs(w64).T
    off64 = None
    if logit_offset is not None:
        off64 = np.asarray(logit_offset, np.float64)
        s = s + off64[None, :]
        a = a + np.abs(off64)[None, :]
    n = d + 1
    gam = n * _U64 / (1.0 - n * _U64)
    r, ok = _rn32_certain(s, 2.0 * gam * a)
    out = r.copy()
    for t, e in zip(*np.nonzero(~ok)):
        out[t, e] = _exact_dot_rn32(x64[t], w64[e], None if off64 is None else float(off64[e]))
    return out


def _sigmoid_key_exact(l32: float, b32: float) -> float:
    """RN32(sigma(l) + b) from an 80-digit evaluation (l = 0 handled exactly)."""
    l32 = float(l32)
    b32 = float(b32)
    if l32 == 0.0:
        return rn32_fraction(Fraction(1, 2) + Fraction(b32))
    with decimal.localcontext() as ctx:
        ctx.prec = 80
        L = decimal.Decimal(l32)
        sig = decimal.Decimal(1) / (decimal.Decimal(1) + (-L).exp())
        v = sig + decimal.Decimal(b32)
    vf = Fraction(v)
    r = rn32_fraction(vf)
    # the 80-digit value is within ~1e-78 relative of the true one; refuse to guess if a
    # rounding boundary is closer than 1e-70 relative (sigma(l) is irrational for l != 0,
    # so this never triggers for representable inputs in practice)
    rr = np.float32(r)
    for nb in (np.nextafter(rr, np.float32(np.inf)), np.nextafter(rr, np.float32(-np.inf))):
        mid = (Fraction(float(rr)) + Fraction(float(nb))) / 2
        if abs(vf - mid) <= Fraction(1, 10 ** 70) * (abs(vf) + Fraction(1, 10 ** 40)):
            raise ArithmeticError("sigmoid key too close to an fp32 rounding boundary")
    return r


def selection_keys(logits: np.ndarray, score: str,
                   select_bias: Optional[np.ndarray] = None) -> np.ndarray:
    """fp32 selection keys (module doc, step 2)."""
    if score == "softmax":
        return np.asarray(logits, np.float32).copy()
    if score != "sigmoid":
        raise ValueError(score)
    l64 = np.asarray(logits, np.float64)
    b64 = np.zeros(l64.shape[1]) if select_bias is None else np.asarray(select_bias, np.float64)
    with np.errstate(over="ignore"):
        sig = 1.0 / (1.0 + np.exp(-l64))
    v = sig + b64[None, :]
    # generous enclosure: 32 ulps of sigma plus the rounding of the addition
    bound = 2.0 ** -48 * sig + 2.0 ** -52 * np.abs(v) + 2.0 ** -1000
    r, ok = _rn32_certain(v, bound)
    out = r.copy()
    for t, e in zip(*np.nonzero(~ok)):
        out[t, e] = _sigmoid_key_exact(float(np.float32(logits[t, e])), float(b64[e]))
    return out


def topk(keys: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest keys per row; equal keys -> lower index first (module doc, 3)."""
    order = np.argsort(-np.asarray(keys, np.float32), axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def probabilities(logits: np.ndarray, score: str) -> np.ndarray:
    """fp64 expert probabilities from the fp32 logits (module doc, step 4)."""
    l64 = np.asarray(logits, np.float64)
    if score == "softmax":
        m = l64.max(axis=1, keepdims=True)
        ex = np.exp(l64 - m)
        return ex / ex.sum(axis=1, keepdims=True)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-l64))


def aux_probabilities(p: np.ndarray, score: str) -> np.ndarray:
    """Per-token distribution entering P_i: softmax p, or sigmoids normalised over all E."""
    if score == "softmax":
        return p
    return p / p.sum(axis=1, keepdims=True)


def combine_weights(p: np.ndarray, idx: np.ndarray, norm_topk: bool) -> np.ndarray:
    w = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    if norm_topk:
        w = w / w.sum(axis=1, keepdims=True)
    return w


def capacity(T: int, k: int, E: int, capacity_factor: float) -> Optional[int]:
    """``ceil(cf * T * k / E)`` evaluated exactly on the fp32 value of cf; None = dropless."""
    cf = float(np.float32(capacity_factor))
    if cf <= 0.0:
        return None
    return math.ceil(Fraction(cf) * T * k / E)


def route(x, w_router, logit_offset, select_bias, score: str, top_k: int,
          norm_topk: bool) -> Dict[str, np.ndarray]:
    """Steps 1-4 plus the per-expert statistics of the load-balancing loss.

    Returns idx [T,k] int32, w [T,k] fp64, count [E] int64 (pre-capacity selections),
    prob_sum [E] fp64 (sum over tokens of the P-basis probabilities), logits, keys, p.
    """
    logits = router_logits(x, w_router, logit_offset)
    keys = selection_keys(logits, score, select_bias)
    E = logits.shape[1]
    idx = topk(keys, top_k)
    p = probabilities(logits, score)
    w = combine_weights(p, idx, norm_topk)
    count = np.bincount(idx.reshape(-1).astype(np.int64), minlength=E)
    prob_sum = aux_probabilities(p, score).sum(axis=0) if len(p) else np.zeros(E)
    return dict(idx=idx, w=w, count=count, prob_sum=prob_sum, logits=logits, keys=keys, p=p)


# ---------------------------------------------------------------------------------------------
# 5-6. Capacity and permutation
# ---------------------------------------------------------------------------------------------
def permute(idx: np.ndarray, E: int, C: Optional[int]) -> Dict[str, np.ndarray]:
    """Stable grouping of the (token, slot) pairs by expert (module doc, steps 5-6).

    Returns offsets [E+1], slot_pos [T,k] (-1 = dropped), src [N] (row -> token), count [E],
    kept [E].
    """
    T, k = idx.shape
    count = np.zeros(E, np.int64)
    for t in range(T):
        for j in range(k):
            count[idx[t, j]] += 1
    kept = count.copy() if C is None else np.minimum(count, C)
    offsets = np.zeros(E + 1, np.int64)
    offsets[1:] = np.cumsum(kept)
    rank = np.zeros(E, np.int64)
    slot_pos = np.full((T, k), -1, np.int64)
    src = np.zeros(int(offsets[E]), np.int64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            r = int(rank[e])
            rank[e] += 1
            if C is None or r < C:
                pos = int(offsets[e]) + r
                slot_pos[t, j] = pos
                src[pos] = t
    return dict(offsets=offsets, slot_pos=slot_pos, src=src, count=count, kept=kept)


# ---------------------------------------------------------------------------------------------
# 7. Experts
# ---------------------------------------------------------------------------------------------
def _silu(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu(X: np.ndarray, Wg: np.ndarray, Wu: np.ndarray, Wd: np.ndarray) -> np.ndarray:
    """Rows of X through ``W_down (silu(W_gate x) * (W_up x))``; W stored [out, in]."""
    X = np.asarray(X, np.float64)
    g = X @ np.asarray(Wg, np.float64).T
    u = X @ np.asarray(Wu, np.float64).T
    return (_silu(g) * u) @ np.asarray(Wd, np.float64).T


def lowrank(X: np.ndarray, V: np.ndarray, s: np.ndarray, U: np.ndarray) -> np.ndarray:
    """Rows of X through ``U (s * (V^T x))`` with V stored [r, d] and U stored [d, r]."""
    X = np.asarray(X, np.float64)
    z = X @ np.asarray(V, np.float64).T
    return (z * np.asarray(s, np.float64)[None, :]) @ np.asarray(U, np.float64).T


def expert_forward(x_perm: np.ndarray, offsets: np.ndarray, x: np.ndarray, W: dict,
                   expert: str) -> Dict[str, np.ndarray]:
    """Routed experts on their permuted rows, and the summed shared experts on every token."""
    N = int(offsets[-1])
    d = x.shape[1]
    E = len(offsets) - 1
    Y = np.zeros((N, d))
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if a == b:
            continue
        if expert == "swiglu":
            Y[a:b] = swiglu(x_perm[a:b], W["w_gate"][e], W["w_up"][e], W["w_down"][e])
        else:
            Y[a:b] = lowrank(x_perm[a:b], W["lr_V"][e], W["lr_s"][e], W["lr_U"][e])
    Ysh = np.zeros((x.shape[0], d))
    if W.get("ws_gate") is not None:
        for s_ in range(W["ws_gate"].shape[0]):
            Ysh += swiglu(x, W["ws_gate"][s_], W["ws_up"][s_], W["ws_down"][s_])
    return dict(y_perm=Y, y_shared=Ysh)


# ---------------------------------------------------------------------------------------------
# 8-9. Combine and load-balancing loss
# ---------------------------------------------------------------------------------------------
def combine(y_perm: np.ndarray, y_shared: Optional[np.ndarray], slot_pos: np.ndarray,
            w: np.ndarray) -> np.ndarray:
    T, k = slot_pos.shape
    d = y_perm.shape[1] if y_perm.ndim == 2 and y_perm.shape[0] else \
        (y_shared.shape[1] if y_shared is not None else 0)
    y = np.zeros((T, d)) if y_shared is None else np.array(y_shared, np.float64)
    for j in range(k):
        kept = slot_pos[:, j] >= 0
        y[kept] += w[kept, j][:, None] * y_perm[slot_pos[kept, j]]
    return y


def bias_update(count: np.ndarray, bias: np.ndarray, u: float) -> np.ndarray:
    """Loss-free balancing step on the per-expert selection bias (dormouse, "dropless MoE":
    balancing by a bias on the router instead of an auxiliary loss, after arXiv 2408.15664):
    ``b_i <- b_i + u * sign(mean_load - load_i)`` with load_i = count_i and mean_load =
    sum(count) / E. The comparison is made exactly on integers (sign(sum(count) - E count_i));
    the new fp32 bias is the exact real b_i + u*s rounded once to fp32 (nearest even).
    """
    count = np.asarray(count, np.int64)
    E = count.shape[0]
    total = int(count.sum())
    u32 = Fraction(float(np.float32(u)))
    out = np.empty(E, np.float32)
    for i in range(E):
        s = (total > E * int(count[i])) - (total < E * int(count[i]))
        out[i] = rn32_fraction(Fraction(float(np.float32(bias[i]))) + u32 * s)
    return out


def aux_loss(count: np.ndarray, prob_sum: np.ndarray, T: int, k: int, alpha: float) -> float:
    """``alpha * E * sum_i (count_i / (T k)) * (prob_sum_i / T)``; 0 for an empty call."""
    E = len(count)
    if T == 0:
        return 0.0
    f = np.asarray(count, np.float64) / (T * k)
    P = np.asarray(prob_sum, np.float64) / T
    return float(alpha * E * np.sum(f * P))


# ---------------------------------------------------------------------------------------------
# Whole layer
# ---------------------------------------------------------------------------------------------
def layer_forward(cfg, inp: Dict[str, np.ndarray], with_outputs: bool = True) -> Dict:
    """All steps on the inputs ``inp`` (arrays as drawn by the input generator).

    ``cfg`` supplies E, top_k, score, expert, norm_topk, capacity_factor, aux_alpha.
    """
    x = inp["x"]
    T = x.shape[0]
    r = route(x, inp["w_router"], inp.get("logit_offset"), inp.get("select_bias"),
              cfg.score, cfg.top_k, cfg.norm_topk)
    C = capacity(T, cfg.top_k, cfg.E, cfg.capacity_factor)
    pm = permute(r["idx"], cfg.E, C)
    out = dict(route=r, perm=pm, capacity=C,
               aux=aux_loss(r["count"], r["prob_sum"], T, cfg.top_k, cfg.aux_alpha))
    if with_outputs:
        x64 = np.asarray(x, np.float64)
        ef = expert_forward(x64[pm["src"]], pm["offsets"], x64, inp, cfg.expert)
        out["experts"] = ef
        out["y"] = combine(ef["y_perm"], ef["y_shared"] if cfg.n_shared else None,
                           pm["slot_pos"], r["w"])
    return out


def token_output(cfg, inp: Dict[str, np.ndarray], t: int, idx_t: np.ndarray,
                 w_t: np.ndarray, kept_t: np.ndarray) -> np.ndarray:
    """y[t] straight from the per-token definition (for sampled checks at full size).

    ``idx_t``/``w_t``/``kept_t`` are the token's selected experts, combine weights and kept
    flags (from :func:`route` and :func:`permute`).
    """
    xt = np.asarray(inp["x"][t:t + 1], np.float64)
    y = np.zeros(xt.shape[1])
    if cfg.n_shared:
        for s_ in range(cfg.n_shared):
            y += swiglu(xt, inp["ws_gate"][s_], inp["ws_up"][s_], inp["ws_down"][s_])[0]
    for j in range(len(idx_t)):
        if not kept_t[j]:
            continue
        e = int(idx_t[j])
        if cfg.expert == "swiglu":
            ye = swiglu(xt, inp["w_gate"][e], inp["w_up"][e], inp["w_down"][e])[0]
        else:
            ye = lowrank(xt, inp["lr_V"][e], inp["lr_s"][e], inp["lr_U"][e])[0]
        y += float(w_t[j]) * ye
    return y
