"""Pins of the fp8 (E4M3) low-rank oracle against things other than itself: the format's
defined code points (OCP FP8 E4M3), torch's CPU float8_e4m3fn conversion (round to nearest even,
no saturation), a brute-force nearest-value search in exact rationals, the plain low-rank
definition within a derived error bound, and a per-token restatement of the layer."""
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import moe_fp8 as F8
from oracle import moe_oracle as O


def test_e4m3_code_points():
    t = F8.e4m3_decode_table()
    known = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 / 8 * 2.0 ** -6, 0x08: 2.0 ** -6, 0x38: 1.0,
             0x39: 1.125, 0x40: 2.0, 0x7E: 448.0, 0xC0: -2.0, 0xFE: -448.0}
    for code, v in known.items():
        assert t[code] == v, hex(code)
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert np.signbit(t[0x80]) and t[0x80] == 0.0
    assert np.isfinite(t).sum() == 254
    assert np.all(np.diff(t[:0x7F]) > 0)              # codes 0..0x7E increase
    assert np.array_equal(t[0x80:0xFF], -t[0x00:0x7F])  # sign-magnitude


def _bruteforce_code(v: float) -> int:
    """Nearest finite E4M3 magnitude in exact rationals; ties to the even code; above 448
    saturates; the sign of v is kept."""
    t = F8.e4m3_decode_table()
    a = abs(Fraction(float(v)))
    best, bd = None, None
    for code in range(0x7F):
        dist = abs(a - Fraction(float(t[code])))
        if bd is None or dist < bd or (dist == bd and code % 2 == 0):
            best, bd = code, dist
    return best | (0x80 if np.signbit(v) else 0)


def _sample_values(rng, n):
    t = F8.e4m3_decode_table()[:0x7F]
    mids = (t[:-1] + t[1:]) / 2
    v = np.concatenate([
        rng.standard_normal(n) * 100, rng.standard_normal(n) * 1e-3,
        rng.uniform(-464, 464, n), mids, -mids, t, np.nextafter(mids.astype(np.float32), np.float32(0)),
        np.nextafter(mids.astype(np.float32), np.float32(1e9)), [0.0, -0.0, 2.0 ** -10, -2.0 ** -10]])
    return v.astype(np.float32)


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(0)
    v = _sample_values(rng, 4000)
    v = v[np.abs(v) <= 464]  # torch does not saturate above the last midpoint
    ours = F8.e4m3_encode(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_encode_bruteforce_with_saturation():
    rng = np.random.default_rng(1)
    v = np.concatenate([_sample_values(rng, 60)[::7], np.float32([464.0, 465.0, 1e6, -3e4])])
    ours = F8.e4m3_encode(v)
    ref = np.array([_bruteforce_code(float(x)) for x in v], np.uint8)
    assert np.array_equal(ours, ref)


def test_quantize_rows_properties():
    rng = np.random.default_rng(2)
    M = (rng.standard_normal((40, 96)) * np.exp(rng.uniform(-20, 20, (40, 1)))).astype(np.float32)
    M[3] = 0.0
    M[5, :] = 0.0
    M[5, 7] = -3.5e-30
    q, s = F8.quantize_rows(M)
    assert s.dtype == np.float32 and s[3] == 1.0 and np.all(q[3] == 0)
    dec = F8.e4m3_decode(q)
    nz = np.abs(M).max(axis=1) > 0
    # the row maximum lands on +-448 (its quotient is 448 within two fp32 roundings)
    assert np.all(np.abs(dec[nz]).max(axis=1) == 448.0)
    # reconstruction within half an E4M3 step of v / s (relative 2^-4 for normals, 2^-10 floor)
    vs = M.astype(np.float64) / s[:, None].astype(np.float64)
    step = np.where(np.abs(vs) >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(np.abs(vs), 1e-300))) - 3),
                    2.0 ** -9)
    assert np.all(np.abs(dec - vs) <= step / 2 * (1 + 1e-6) + 1e-30)


def test_lowrank_fp8_within_bound_of_plain_definition():
    """With the quantised operands decoded, the only extra error is z's own quantisation:
    |y - U (s * V^T x)| <= sum_j |U[c,j]| e_j, e_j = half an E4M3 step of z_j / sz times sz (plus
    z's fp32 rounding). A transposed operand, a misplaced scale or a dropped term breaks it."""
    rng = np.random.default_rng(3)
    n, d, r = 37, 96, 64
    x = rng.standard_normal((n, d)).astype(np.float32)
    V = (rng.standard_normal((r, d)) / np.sqrt(d)).astype(np.float32)
    U = (rng.standard_normal((d, r)) / np.sqrt(r)).astype(np.float32)
    s = rng.uniform(0.5, 1.5, r).astype(np.float32)
    xq, sx = F8.quantize_rows(x)
    Vq, sV = F8.quantize_rows(V)
    Uq, sU = F8.quantize_rows(U)
    y = F8.lowrank_fp8(xq, sx, Vq, sV, s, Uq, sU)
    Xd, Vd, Ud = (F8.dequantize_rows(a, b) for a, b in ((xq, sx), (Vq, sV), (Uq, sU)))
    y_plain = O.lowrank(Xd, Vd, s, Ud)
    z = (Xd @ Vd.T) * s[None, :].astype(np.float64)
    sz = np.abs(z.astype(np.float32)).max(axis=1).astype(np.float64) / 448.0
    zs = np.abs(z) / sz[:, None]
    half = np.where(zs >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(zs, 1e-300))) - 4), 2.0 ** -10)
    e = (half * (1 + 1e-5) + 1e-6 * zs) * sz[:, None]
    bound = e @ np.abs(Ud).T
    err = np.abs(y - y_plain)
    assert np.all(err <= bound)
    assert err.max() > 0  # the quantisation of z is really there


def test_layer_fp8_per_token():
    """y[t] = sum over kept slots of w[t,j] * expert_{e_j}(token t's quantised row)."""
    from moe_synth import get_config, make_inputs
    c = get_config("lowrank", T=96, E=16, d=128)
    inp = make_inputs(c)
    out = F8.layer_forward_fp8(c, inp)
    W8 = out["W8"]
    r, pm = out["route"], out["perm"]
    for t in range(0, c.T, 5):
        acc = np.zeros(c.d)
        for j in range(c.top_k):
            if pm["slot_pos"][t, j] < 0:
                continue
            e = int(r["idx"][t, j])
            yt = F8.lowrank_fp8(out["xq"][t:t + 1], out["sx"][t:t + 1], W8["V8"][e], W8["sV"][e],
                                W8["lr_s"][e], W8["U8"][e], W8["sU"][e])[0]
            acc += r["w"][t, j] * yt
        assert np.allclose(out["y"][t], acc, rtol=1e-12, atol=1e-12)
