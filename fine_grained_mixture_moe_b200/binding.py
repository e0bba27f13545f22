"""ctypes binding of ``libmoe.so`` (declared in ``include/moe.h``).

Argument marshalling only: every function below converts its arguments to the C types of the
header and calls the function of the same name. Buffers may be given as torch tensors (their
``data_ptr()`` is passed) or as integer addresses. A non-OK status raises :class:`MoEError`.
The library must be built (``fine_grained_mixture_moe_b200.build``); there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

from . import build as _build

c_int32, c_int64, c_float, c_size_t, c_void_p = (ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                                                 ctypes.c_size_t, ctypes.c_void_p)

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_WORKSPACE", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT",
                6: "MOE_ERR_DEVICE_CHECK"}
SCORE = {"softmax": 0, "sigmoid": 1}
EXPERT = {"swiglu": 0, "lowrank": 1}
DTYPE = {"f32": 0, "bf16": 1}
STORAGE = {"dtype": 0, "fp8": 1}
DEBUG_FORCE_EXACT, DEBUG_WAIT_LIMIT_NS, DEBUG_PROFILE, DEBUG_STAMP = 1, 2, 3, 4


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {status_str(status)}")


class MoEConfig(ctypes.Structure):
    _fields_ = [("T", c_int32), ("d", c_int32), ("E", c_int32), ("top_k", c_int32),
                ("n_shared", c_int32), ("ffn", c_int32), ("ffn_shared", c_int32),
                ("rank", c_int32), ("score", c_int32), ("expert", c_int32), ("dtype", c_int32),
                ("norm_topk", c_int32), ("capacity_factor", c_float), ("aux_alpha", c_float),
                ("expert_storage", c_int32)]


class MoEWeights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ("w_router", "logit_offset", "select_bias", "w_gate",
                                        "w_up", "w_down", "lr_V", "lr_U", "lr_s", "ws_gate",
                                        "ws_up", "ws_down", "lr_V8", "lr_V_scale", "lr_U8",
                                        "lr_U_scale")]


class MoEGrads(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ("d_w_gate", "d_w_up", "d_w_down", "d_lr_V", "d_lr_s",
                                        "d_lr_U", "d_ws_gate", "d_ws_up", "d_ws_down")]


def make_grads(tensors: Dict[str, object]) -> "MoEGrads":
    """moe_grads_t from a dict name -> tensor (names of MoEGrads' fields; missing ones NULL)."""
    g = MoEGrads()
    for name, _ in MoEGrads._fields_:
        if tensors.get(name) is not None:
            setattr(g, name, _ptr(tensors[name]))
    return g


_lib: Optional[ctypes.CDLL] = None


def lib_path() -> str:
    return _build.LIB


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load ``libmoe.so`` (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or lib_path()
    if not os.path.exists(path):
        raise RuntimeError(f"MoE CUDA library not built: {path} is missing "
                           "(run python -m fine_grained_mixture_moe_b200.build)")
    L = ctypes.CDLL(path)
    P = ctypes.POINTER
    sig = {
        "moe_workspace_size": (c_size_t, [P(MoEConfig)]),
        "moe_capacity": (c_int32, [P(MoEConfig)]),
        "moe_route": (c_int32, [P(MoEConfig), c_void_p, P(MoEWeights), c_void_p, c_void_p,
                                c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
        "moe_permute": (c_int32, [P(MoEConfig), c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                  c_void_p, c_void_p, c_size_t, c_void_p]),
        "moe_expert_forward": (c_int32, [P(MoEConfig), c_void_p, c_void_p, c_void_p,
                                         P(MoEWeights), c_void_p, c_void_p, c_void_p, c_size_t,
                                         c_void_p]),
        "moe_combine": (c_int32, [P(MoEConfig), c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                  c_void_p]),
        "moe_aux_loss": (c_int32, [P(MoEConfig), c_void_p, c_void_p, c_void_p, c_void_p]),
        "moe_combine_backward": (c_int32, [P(MoEConfig), c_void_p, c_void_p, c_void_p, c_void_p,
                                           c_void_p, c_void_p, c_void_p]),
        "moe_route_backward": (c_int32, [P(MoEConfig), c_void_p, P(MoEWeights), c_void_p,
                                         c_void_p, c_void_p, ctypes.c_float, c_void_p, c_void_p,
                                         c_void_p, c_void_p]),
        "moe_bias_update": (c_int32, [P(MoEConfig), c_void_p, c_void_p, ctypes.c_float, c_void_p]),
        "moe_layer_forward": (c_int32, [P(MoEConfig), c_void_p, P(MoEWeights), c_void_p,
                                        c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
        "moe_status_str": (ctypes.c_char_p, [c_int32]),
        "moe_get_device_error": (c_int32, [c_void_p, P(c_int64)]),
        "moe_debug_set": (c_int32, [c_int32, c_int64]),
        "moe_profile_read": (c_int32, [P(ctypes.c_char_p), P(ctypes.c_double), P(c_int64),
                                       c_int32]),
        "moe_stamp_read": (c_int32, [P(ctypes.c_char_p), P(ctypes.c_double), c_int32]),
        "moe_backward_workspace_size": (c_size_t, [P(MoEConfig)]),
        "moe_expert_backward": (c_int32, [P(MoEConfig), c_void_p, c_void_p, c_void_p, c_void_p,
                                          P(MoEWeights), c_void_p, c_void_p, c_void_p,
                                          P(MoEGrads), c_void_p, c_size_t, c_void_p]),
        "moe_debug_wait_timeout_probe": (c_int32, [c_void_p]),
        "moe_route_noalloc": (c_int32, [P(MoEConfig), c_void_p, P(MoEWeights), c_void_p,
                                        c_void_p, c_void_p, c_void_p, c_void_p]),
        "moe_quantize_fp8": (c_int32, [c_void_p, c_int32, c_int64, c_int32, c_void_p, c_void_p,
                                       c_void_p]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


EXPORTED = ("moe_workspace_size", "moe_capacity", "moe_route", "moe_permute",
            "moe_expert_forward", "moe_combine", "moe_aux_loss", "moe_bias_update",
            "moe_combine_backward", "moe_route_backward", "moe_backward_workspace_size",
            "moe_expert_backward",
            "moe_layer_forward",
            "moe_status_str", "moe_get_device_error", "moe_debug_set", "moe_profile_read",
            "moe_stamp_read", "moe_debug_wait_timeout_probe", "moe_route_noalloc",
            "moe_quantize_fp8")


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, status: int) -> None:
    if status != MOE_OK:
        raise MoEError(fn, status)


def status_str(status: int) -> str:
    try:
        return load().moe_status_str(status).decode()
    except Exception:
        return STATUS_NAMES.get(status, f"status {status}")


def make_config(T: int, d: int, E: int, top_k: int, n_shared: int = 0, ffn: int = 0,
                ffn_shared: int = 0, rank: int = 0, score: str = "softmax",
                expert: str = "swiglu", dtype: str = "bf16", norm_topk: bool = False,
                capacity_factor: float = 0.0, aux_alpha: float = 0.01,
                expert_storage: str = "dtype") -> MoEConfig:
    return MoEConfig(T, d, E, top_k, n_shared, ffn, ffn_shared, rank, SCORE[score],
                     EXPERT[expert], DTYPE[dtype], int(bool(norm_topk)), capacity_factor,
                     aux_alpha, STORAGE[expert_storage])


def make_weights(tensors: Dict[str, object]) -> MoEWeights:
    """Weights struct from a dict of device tensors (missing or None entries are NULL)."""
    w = MoEWeights()
    for name, _ in MoEWeights._fields_:
        setattr(w, name, _ptr(tensors.get(name)))
    return w


# ------------------------------------------------------------------ the C functions
def moe_workspace_size(cfg: MoEConfig) -> int:
    return int(load().moe_workspace_size(ctypes.byref(cfg)))


def moe_capacity(cfg: MoEConfig) -> int:
    return int(load().moe_capacity(ctypes.byref(cfg)))


def moe_route(cfg, x, w: MoEWeights, topk_idx, topk_w, expert_count, prob_sum, ws, ws_bytes,
              stream=None) -> None:
    _check("moe_route", load().moe_route(ctypes.byref(cfg), _ptr(x), ctypes.byref(w),
                                         _ptr(topk_idx), _ptr(topk_w), _ptr(expert_count),
                                         _ptr(prob_sum), _ptr(ws), ws_bytes, _stream(stream)))


def moe_permute(cfg, x, topk_idx, offsets, slot_pos, src_token, x_perm, ws, ws_bytes,
                stream=None) -> None:
    _check("moe_permute", load().moe_permute(ctypes.byref(cfg), _ptr(x), _ptr(topk_idx),
                                             _ptr(offsets), _ptr(slot_pos), _ptr(src_token),
                                             _ptr(x_perm), _ptr(ws), ws_bytes, _stream(stream)))


def moe_expert_forward(cfg, x_perm, offsets, x, w: MoEWeights, y_perm, y_shared, ws, ws_bytes,
                       stream=None) -> None:
    _check("moe_expert_forward",
           load().moe_expert_forward(ctypes.byref(cfg), _ptr(x_perm), _ptr(offsets), _ptr(x),
                                     ctypes.byref(w), _ptr(y_perm), _ptr(y_shared), _ptr(ws),
                                     ws_bytes, _stream(stream)))


def moe_combine(cfg, y_perm, y_shared, slot_pos, topk_w, y, stream=None) -> None:
    _check("moe_combine", load().moe_combine(ctypes.byref(cfg), _ptr(y_perm), _ptr(y_shared),
                                             _ptr(slot_pos), _ptr(topk_w), _ptr(y),
                                             _stream(stream)))


def moe_combine_backward(cfg, dy, y_perm, slot_pos, topk_w, dy_perm, d_topk_w,
                         stream=None) -> None:
    _check("moe_combine_backward",
           load().moe_combine_backward(ctypes.byref(cfg), _ptr(dy), _ptr(y_perm), _ptr(slot_pos),
                                       _ptr(topk_w), _ptr(dy_perm), _ptr(d_topk_w),
                                       _stream(stream)))


def moe_route_backward(cfg, x, w: MoEWeights, topk_idx, expert_count, d_topk_w, d_loss: float,
                       d_logits, d_w_router, dx, stream=None) -> None:
    _check("moe_route_backward",
           load().moe_route_backward(ctypes.byref(cfg), _ptr(x), ctypes.byref(w), _ptr(topk_idx),
                                     _ptr(expert_count), _ptr(d_topk_w), ctypes.c_float(d_loss),
                                     _ptr(d_logits), _ptr(d_w_router), _ptr(dx),
                                     _stream(stream)))


def moe_aux_loss(cfg, expert_count, prob_sum, loss, stream=None) -> None:
    _check("moe_aux_loss", load().moe_aux_loss(ctypes.byref(cfg), _ptr(expert_count),
                                               _ptr(prob_sum), _ptr(loss), _stream(stream)))


def moe_bias_update(cfg, expert_count, select_bias, u: float, stream=None) -> None:
    _check("moe_bias_update", load().moe_bias_update(ctypes.byref(cfg), _ptr(expert_count),
                                                     _ptr(select_bias), ctypes.c_float(u),
                                                     _stream(stream)))


def moe_layer_forward(cfg, x, w: MoEWeights, y, aux_loss, expert_count, ws, ws_bytes,
                      stream=None) -> None:
    _check("moe_layer_forward",
           load().moe_layer_forward(ctypes.byref(cfg), _ptr(x), ctypes.byref(w), _ptr(y),
                                    _ptr(aux_loss), _ptr(expert_count), _ptr(ws), ws_bytes,
                                    _stream(stream)))


def moe_get_device_error(stream=None):
    info = c_int64(0)
    st = load().moe_get_device_error(_stream(stream), ctypes.byref(info))
    return int(st), int(info.value)


def moe_debug_set(what: int, value: int) -> None:
    _check("moe_debug_set", load().moe_debug_set(what, value))


def moe_profile_read(max_kinds: int = 32):
    names = (ctypes.c_char_p * max_kinds)()
    ms = (ctypes.c_double * max_kinds)()
    n = (c_int64 * max_kinds)()
    cnt = load().moe_profile_read(names, ms, n, max_kinds)
    return {names[i].decode(): (ms[i], int(n[i])) for i in range(min(cnt, max_kinds))}


def moe_backward_workspace_size(cfg) -> int:
    return int(load().moe_backward_workspace_size(ctypes.byref(cfg)))


def moe_expert_backward(cfg, x_perm, offsets, slot_pos, x, w: MoEWeights, dy_perm, dy, dx,
                        grads: MoEGrads, ws, ws_bytes: int, stream=None) -> None:
    _check("moe_expert_backward",
           load().moe_expert_backward(ctypes.byref(cfg), _ptr(x_perm), _ptr(offsets),
                                      _ptr(slot_pos), _ptr(x), ctypes.byref(w), _ptr(dy_perm),
                                      _ptr(dy), _ptr(dx), ctypes.byref(grads), _ptr(ws),
                                      ws_bytes, _stream(stream)))


def moe_stamp_read(max_kinds: int = 32):
    """In-step kernel durations (microseconds) per kind since the last read (moe_stamp_read)."""
    names = (ctypes.c_char_p * max_kinds)()
    us = (ctypes.c_double * max_kinds)()
    cnt = load().moe_stamp_read(names, us, max_kinds)
    if cnt < 0:
        raise MoEError("moe_stamp_read", 4)
    return {names[i].decode(): us[i] for i in range(min(cnt, max_kinds))}


def moe_debug_wait_timeout_probe(stream=None) -> None:
    _check("moe_debug_wait_timeout_probe", load().moe_debug_wait_timeout_probe(_stream(stream)))


ROUTE_NOALLOC_SCRATCH_BYTES = 4 << 20


def moe_quantize_fp8(x, rows: int, cols: int, q, scale, stream=None) -> None:
    """Per-row E4M3 codes q [rows, cols] uint8 and fp32 scales [rows] of x (bf16 or fp32)."""
    import torch
    dt = DTYPE["bf16"] if x.dtype == torch.bfloat16 else DTYPE["f32"]
    _check("moe_quantize_fp8", load().moe_quantize_fp8(_ptr(x), dt, rows, cols, _ptr(q),
                                                       _ptr(scale), _stream(stream)))


def moe_route_noalloc(cfg, x, w: MoEWeights, topk_idx, topk_w, expert_count, prob_sum,
                      stream=None) -> None:
    """moe_route with its scratch in the library's fixed device array (no workspace)."""
    _check("moe_route_noalloc",
           load().moe_route_noalloc(ctypes.byref(cfg), _ptr(x), ctypes.byref(w), _ptr(topk_idx),
                                    _ptr(topk_w), _ptr(expert_count), _ptr(prob_sum),
                                    _stream(stream)))
