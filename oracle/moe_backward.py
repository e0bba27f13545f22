"""Plain, slow CPU oracle of the backward pass of the fine-grained MoE FFN layer.

TEST INFRASTRUCTURE, like ``moe_oracle``: imported only by the tests. It shares no code with the
CUDA path. CUDA kernels compute steps a and d-g below (the combine and the router); the expert
steps b and c have none yet.

The pages train whole models with this layer (research page, training setup: gradient
accumulation and full gradient checkpointing), but none of them writes the backward out. Read
plainly, it is the derivative of the forward that ``moe_oracle`` defines. Given an upstream
gradient ``dy`` [T, d] of the layer output y and a scalar ``dL`` for the load-balancing loss L,
this module returns the gradient of the scalar ``J = sum(dy * y) + dL * L`` with respect to every
trained input. Where the forward is not differentiable, these readings apply:

B1. The selection is piecewise constant in the inputs: the top-k indices, the capacity drops and
    the counts f_i of the loss. No gradient passes through it (the derivative almost everywhere).
B2. The selection bias is moved by the loss-free balancing step, not by a gradient, and the
    per-expert logit offsets are a fixed skew of the inputs. Neither gets a gradient.
B3. The fp32 rounding of each router logit has derivative 1 almost everywhere: the logit's
    gradient goes to ``sum_i x_i W_r[e,i]`` unchanged. Probabilities are formed from the fp32
    logits, as in the forward.
B4. A dropped (token, slot) pair adds nothing to y and gets no gradient through its expert. With
    ``norm_topk`` its probability still sits in the normalising sum of the token's k selected
    probabilities, as in the forward, so it gets that share.

Steps, the forward's in reverse (every product in fp64):

a. Combine (Moonfrost, expert card: a token passes through the shared expert and its top-k
   routed ones): ``dY_perm[pos(t,j)] = w[t,j] dy[t]``, ``dw[t,j] = <dy[t], Y_perm[pos(t,j)]>`` for
   kept pairs, and ``dY_shared = dy``.
b. Experts on their grouped rows. SwiGLU with ``g = X Wg^T``, ``u = X Wu^T``,
   ``h = silu(g) * u``, ``Y = h Wd^T``:
   ``dWd = dY^T h``, ``dh = dY Wd``, ``du = dh * silu(g)``, ``dg = dh * u * silu'(g)`` with
   ``silu'(z) = sigma(z) (1 + z (1 - sigma(z)))``, ``dWg = dg^T X``, ``dWu = du^T X``,
   ``dX = dg Wg + du Wu``.
   Low-rank (dormouse, "TSCT low-rank experts") with ``z = X V^T``, ``Y = (z * s) U^T``:
   ``dU = dY^T (z * s)``, ``dzs = dY U``, ``ds = sum over rows of dzs * z``,
   ``dV = (dzs * s)^T X``, ``dX = (dzs * s) V``.
   Shared experts: the SwiGLU step on every token, with ``dY = dy``.
c. Un-permute: ``dx[t] += dX_perm[pos(t,j)]`` over the kept pairs, plus the shared experts' dX.
d. Combine weights to probabilities: ``w_j = p_{e_j}``, or ``w_j = p_{e_j} / S`` with S the sum
   of the k selected probabilities (``norm_topk``), so
   ``dp_{e_j} = (dw_j - sum_i dw_i w_i) / S``.
e. Load-balancing loss (research page, architecture table, row "Router": weight 0.01):
   ``L = alpha E sum_i f_i P_i`` and ``P_i = (1/T) sum_t q[t,i]``, where q is the softmax
   probability, or for sigmoid scoring ``sigma(l_i)`` divided by the sum over all E experts. So
   ``dq[t,i] = dL alpha E f_i / T``. For sigmoid scoring this goes back to the sigmoids as
   ``dsigma_i = (dq_i - sum_j dq_j q_j) / sum_j sigma_j``.
f. Scores to logits: softmax ``dl = p * (dp - <dp, p>)``; sigmoid (Sutra-1.3B, "48 + 1
   experts") ``dl = dsigma * sigma * (1 - sigma)``.
g. Router: ``dW_r = dl^T x`` and ``dx += dl W_r``.
"""
from __future__ import annotations

from typing import Dict

import numpy as np

from . import moe_oracle as F

__all__ = ["swiglu_backward", "lowrank_backward", "layer_backward"]


def _sigmoid(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def swiglu_backward(X, Wg, Wu, Wd, dY) -> Dict[str, np.ndarray]:
    """Step b for one SwiGLU expert on the rows X (W stored [out, in])."""
    X = np.asarray(X, np.float64)
    Wg = np.asarray(Wg, np.float64)
    Wu = np.asarray(Wu, np.float64)
    Wd = np.asarray(Wd, np.float64)
    dY = np.asarray(dY, np.float64)
    g = X @ Wg.T
    u = X @ Wu.T
    sg = _sigmoid(g)
    silu = g * sg
    h = silu * u
    dWd = dY.T @ h
    dh = dY @ Wd
    du = dh * silu
    dg = dh * u * (sg * (1.0 + g * (1.0 - sg)))
    return dict(dX=dg @ Wg + du @ Wu, dWg=dg.T @ X, dWu=du.T @ X, dWd=dWd)


def lowrank_backward(X, V, s, U, dY) -> Dict[str, np.ndarray]:
    """Step b for one low-rank expert ``U (s * (V^T x))`` (V stored [r, d], U stored [d, r])."""
    X = np.asarray(X, np.float64)
    V = np.asarray(V, np.float64)
    s = np.asarray(s, np.float64)
    U = np.asarray(U, np.float64)
    dY = np.asarray(dY, np.float64)
    z = X @ V.T
    zs = z * s[None, :]
    dzs = dY @ U
    dz = dzs * s[None, :]
    return dict(dX=dz @ V, dV=dz.T @ X, ds=(dzs * z).sum(axis=0), dU=dY.T @ zs)


def layer_backward(cfg, inp: Dict[str, np.ndarray], dy: np.ndarray, dL: float = 1.0,
                   loss_count=None, loss_T=None) -> Dict:
    """Gradients of ``J = sum(dy * y) + dL * L`` for the layer of ``moe_oracle.layer_forward``.

    ``loss_count`` [E] and ``loss_T`` are the statistics L is formed from when they are not this
    call's own: data-parallel replicas form it from the counts summed over the ranks and the
    global token count (module doc, step e). By default they are this call's counts and T.

    Returns dx [T, d], d_w_router [E, d], the expert gradients under the weights' own names with
    a ``d_`` prefix (d_w_gate ... d_ws_down, or d_lr_V, d_lr_s, d_lr_U), and the intermediate
    gradients d_logits [T, E], d_w [T, k] (of the combine weights), d_y_perm [N, d] (of the
    grouped expert outputs) and dx_router [T, d] (the router's part of dx).
    """
    x = np.asarray(inp["x"], np.float64)
    T, d = x.shape
    E, k = cfg.E, cfg.top_k
    dy = np.asarray(dy, np.float64).reshape(T, d)
    fwd = F.layer_forward(cfg, inp, with_outputs=True)
    r, pm = fwd["route"], fwd["perm"]
    idx = r["idx"].astype(np.int64)
    w = r["w"]
    p = r["p"]
    slot_pos = pm["slot_pos"]
    offsets = pm["offsets"]
    src = pm["src"]
    Y = fwd["experts"]["y_perm"]
    out: Dict[str, np.ndarray] = {}

    # a. combine
    N = int(offsets[-1])
    dY = np.zeros((N, d))
    dw = np.zeros((T, k))
    for t in range(T):
        for j in range(k):
            pos = int(slot_pos[t, j])
            if pos >= 0:
                dY[pos] = w[t, j] * dy[t]
                dw[t, j] = float(np.dot(dy[t], Y[pos]))

    # b, c. experts and un-permute
    dx = np.zeros((T, d))
    Xp = x[src]
    if cfg.expert == "swiglu":
        names = ("w_gate", "w_up", "w_down")
        grads = {n: np.zeros_like(np.asarray(inp[n], np.float64)) for n in names}
    else:
        names = ("lr_V", "lr_s", "lr_U")
        grads = {n: np.zeros_like(np.asarray(inp[n], np.float64)) for n in names}
    dXp = np.zeros((N, d))
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if a == b:
            continue
        if cfg.expert == "swiglu":
            g = swiglu_backward(Xp[a:b], inp["w_gate"][e], inp["w_up"][e], inp["w_down"][e],
                                dY[a:b])
            grads["w_gate"][e] = g["dWg"]
            grads["w_up"][e] = g["dWu"]
            grads["w_down"][e] = g["dWd"]
        else:
            g = lowrank_backward(Xp[a:b], inp["lr_V"][e], inp["lr_s"][e], inp["lr_U"][e],
                                 dY[a:b])
            grads["lr_V"][e] = g["dV"]
            grads["lr_s"][e] = g["ds"]
            grads["lr_U"][e] = g["dU"]
        dXp[a:b] = g["dX"]
    for pos in range(N):
        dx[int(src[pos])] += dXp[pos]
    for n in names:
        out["d_" + n] = grads[n]
    if cfg.n_shared:
        for n in ("ws_gate", "ws_up", "ws_down"):
            out["d_" + n] = np.zeros_like(np.asarray(inp[n], np.float64))
        for s_ in range(cfg.n_shared):
            g = swiglu_backward(x, inp["ws_gate"][s_], inp["ws_up"][s_], inp["ws_down"][s_], dy)
            out["d_ws_gate"][s_] = g["dWg"]
            out["d_ws_up"][s_] = g["dWu"]
            out["d_ws_down"][s_] = g["dWd"]
            dx += g["dX"]

    # d. combine weights -> probabilities of the selected experts
    dp = np.zeros((T, E))
    for t in range(T):
        if cfg.norm_topk:
            S = float(sum(p[t, idx[t, j]] for j in range(k)))
            inner = float(sum(dw[t, j] * w[t, j] for j in range(k)))
            for j in range(k):
                dp[t, idx[t, j]] += (dw[t, j] - inner) / S
        else:
            for j in range(k):
                dp[t, idx[t, j]] += dw[t, j]

    # e, f. load-balancing loss and the scores -> logits
    cnt_L = np.asarray(r["count"] if loss_count is None else loss_count, np.float64)
    T_L = T if loss_T is None else int(loss_T)
    f = cnt_L / (T_L * k) if T_L else np.zeros(E)
    dq = np.broadcast_to(dL * cfg.aux_alpha * E * f / T_L, (T, E)) if T_L else np.zeros((T, E))
    if cfg.score == "softmax":
        dp_all = dp + dq
        dlog = p * (dp_all - (dp_all * p).sum(axis=1, keepdims=True))
    else:
        sig = p  # the sigmoids of the fp32 logits
        ssum = sig.sum(axis=1, keepdims=True)
        q = sig / ssum
        dsig = dp + (dq - (dq * q).sum(axis=1, keepdims=True)) / ssum
        dlog = dsig * sig * (1.0 - sig)

    # g. router
    Wr = np.asarray(inp["w_router"], np.float64)
    out["d_w_router"] = dlog.T @ x
    out["dx_router"] = dlog @ Wr
    dx += out["dx_router"]
    out["dx"] = dx
    out["d_logits"] = dlog
    out["d_w"] = dw
    out["d_y_perm"] = dY
    return out
