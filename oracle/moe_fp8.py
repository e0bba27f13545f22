"""Plain CPU oracle of the low-rank experts with fp8 (e4m3) storage.

TEST INFRASTRUCTURE. Imported only by the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg; it shares no code with the CUDA path.

The pages (dormouse, "TSCT low-rank experts") say that each expert's factorisation
``U diag(s) V^T`` of rank 64 also carries a storage ladder fp8 -> NVFP4 -> ternary, and (same
page, "QAT ladder") that training runs in bf16 while a release is one rung of that ladder. They
give no scale granularity or rounding, so this oracle takes the plainest reading of the fp8 rung
(each choice is listed with the design notes):

* Format: OCP FP8 E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; subnormals;
  largest finite 448; codes 0x7F / 0xFF are NaN; no infinities).
* Scaling: one fp32 scale per row of a matrix (per output channel of V and U, per token row of
  the activations): ``s = amax / 448`` in fp32 (1 for an all-zero row), and
  ``code = E4M3(v / s)`` with the quotient rounded once to fp32 and then to the nearest E4M3 value,
  ties to the even code, saturating at +-448.
* The step, per expert e on its grouped rows (the activations quantised per token before the
  permutation, so a token's rows share one scale):
      z = (Xq Vq_e^T) * sx[row] * sV_e[j] * s_e[j]                   (exact sum of the decoded
                                                                        products, fp64)
      zq, sz = quantised rows of RN32(z)
      y = (zq Uq_e^T) * sz[row] * sU_e[c]
  The fp8 products run on the tensor cores; the scales act on the fp32 sums, so nothing else is
  quantised.
"""
from __future__ import annotations

from typing import Dict, Tuple

import numpy as np

__all__ = ["E4M3_MAX", "e4m3_decode_table", "e4m3_encode", "e4m3_decode", "quantize_rows",
           "dequantize_rows", "lowrank_fp8", "expert_forward_fp8", "quantize_lowrank_weights",
           "layer_forward_fp8"]

E4M3_MAX = 448.0


def e4m3_decode_table() -> np.ndarray:
    """Value of every byte under E4M3 (NaN for 0x7F and 0xFF), from the format definition."""
    out = np.empty(256, np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        exp = (code >> 3) & 0xF
        man = code & 0x7
        if exp == 0xF and man == 0x7:
            out[code] = np.nan
        elif exp == 0:
            out[code] = sign * (man / 8.0) * 2.0 ** -6
        else:
            out[code] = sign * (1.0 + man / 8.0) * 2.0 ** (exp - 7)
    return out


_TABLE = e4m3_decode_table()
_MAG = _TABLE[:0x7F]                     # codes 0x00..0x7E: 0, 2^-9, ..., 448, increasing
_MID = (_MAG[:-1] + _MAG[1:]) / 2.0      # exact dyadic midpoints between neighbours


def e4m3_encode(v) -> np.ndarray:
    """Nearest E4M3 code of each finite value (compared exactly in fp64), ties to the even code,
    magnitudes above 448 saturated to 448."""
    a = np.asarray(v, np.float64)
    mag = np.abs(a)
    # index i with _MID[i-1] < mag < _MID[i] is code i; at a midpoint pick the even code
    i = np.searchsorted(_MID, mag, side="left")
    tie = (i < len(_MID)) & (mag == _MID[np.minimum(i, len(_MID) - 1)])
    i = np.where(tie & (i % 2 == 1), i + 1, i)
    i = np.minimum(i, 0x7E)
    sign = np.where(np.signbit(a), 0x80, 0)  # the sign survives rounding to zero (-0 = 0x80)
    return (i | sign).astype(np.uint8)


def e4m3_decode(codes) -> np.ndarray:
    return _TABLE[np.asarray(codes, np.uint8)]


def quantize_rows(M) -> Tuple[np.ndarray, np.ndarray]:
    """Per-row E4M3 codes and fp32 scales of a matrix of fp32-representable values."""
    M = np.asarray(M, np.float32)
    amax = np.max(np.abs(M), axis=-1) if M.shape[-1] else np.zeros(M.shape[:-1], np.float32)
    s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    q = e4m3_encode((M / s[..., None]).astype(np.float32))
    return q, s


def dequantize_rows(q, s) -> np.ndarray:
    return e4m3_decode(q) * np.asarray(s, np.float64)[..., None]


def lowrank_fp8(Xq, sx, Vq, sV, s, Uq, sU) -> np.ndarray:
    """One expert on its quantised rows (see the module header)."""
    X = e4m3_decode(Xq)
    z = (X @ e4m3_decode(Vq).T) * np.asarray(sx, np.float64)[:, None] \
        * np.asarray(sV, np.float64)[None, :] * np.asarray(s, np.float64)[None, :]
    zq, sz = quantize_rows(z.astype(np.float32))
    return (e4m3_decode(zq) @ e4m3_decode(Uq).T) * np.asarray(sz, np.float64)[:, None] \
        * np.asarray(sU, np.float64)[None, :]


def quantize_lowrank_weights(inp: Dict[str, np.ndarray]) -> Dict[str, np.ndarray]:
    """E4M3 rows of every expert's V [E, r, d] and U [E, d, r], with their scales."""
    Vq, sV = quantize_rows(inp["lr_V"])
    Uq, sU = quantize_rows(inp["lr_U"])
    return dict(V8=Vq, sV=sV, U8=Uq, sU=sU, lr_s=np.asarray(inp["lr_s"], np.float32))


def expert_forward_fp8(xq_perm, sx_perm, offsets, W8) -> np.ndarray:
    """Routed low-rank fp8 experts on their grouped rows -> y_perm [N, d] (fp64)."""
    N = int(offsets[-1])
    d = W8["U8"].shape[1]
    Y = np.zeros((N, d))
    for e in range(len(offsets) - 1):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if a < b:
            Y[a:b] = lowrank_fp8(xq_perm[a:b], sx_perm[a:b], W8["V8"][e], W8["sV"][e],
                                 W8["lr_s"][e], W8["U8"][e], W8["sU"][e])
    return Y


def layer_forward_fp8(cfg, inp: Dict[str, np.ndarray], W8=None) -> Dict:
    """The layer with fp8 low-rank experts: routing and permutation as in the bf16 layer (on
    the same x), the token rows quantised once, the experts above, the same combine."""
    from . import moe_oracle as O
    x = inp["x"]
    T = x.shape[0]
    r = O.route(x, inp["w_router"], inp.get("logit_offset"), inp.get("select_bias"),
                cfg.score, cfg.top_k, cfg.norm_topk)
    C = O.capacity(T, cfg.top_k, cfg.E, cfg.capacity_factor)
    pm = O.permute(r["idx"], cfg.E, C)
    W8 = W8 if W8 is not None else quantize_lowrank_weights(inp)
    xq, sx = quantize_rows(np.asarray(x, np.float32))
    y_perm = expert_forward_fp8(xq[pm["src"]], sx[pm["src"]], pm["offsets"], W8)
    y_shared = None
    if cfg.n_shared:  # the shared SwiGLU experts keep the layer's dtype
        x64 = np.asarray(x, np.float64)
        y_shared = np.zeros_like(x64)
        for j in range(inp["ws_gate"].shape[0]):
            y_shared += O.swiglu(x64, inp["ws_gate"][j], inp["ws_up"][j], inp["ws_down"][j])
    y = O.combine(y_perm, y_shared, pm["slot_pos"], r["w"])
    return dict(route=r, perm=pm, xq=xq, sx=sx, W8=W8, y_perm=y_perm, y_shared=y_shared, y=y,
                aux=O.aux_loss(r["count"], r["prob_sum"], T, cfg.top_k, cfg.aux_alpha))
