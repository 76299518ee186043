"""ctypes binding of libmoe_b200.so -- argument marshalling only.

Every function here has the name of the C entry point it calls (include/moe.h)
and takes torch tensors (device memory) or None for optional pointers; it
raises MoEError when the library returns a non-zero status. No step of the
layer runs in Python: there is no CPU fallback, and on a machine without the
compiled library load() raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import build as _build

_lock = threading.Lock()
_lib = None

MOE_SCORE_SOFTMAX, MOE_SCORE_SIGMOID = 0, 1
MOE_DT_BF16, MOE_DT_MXFP8, MOE_DT_NVFP4 = 0, 1, 2
_DTYPES = {"bf16": MOE_DT_BF16, "mxfp8": MOE_DT_MXFP8, "nvfp4": MOE_DT_NVFP4}
MOE_GEMM_GATEUP_SWIGLU, MOE_GEMM_DOWN = 0, 1


class MoEError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn} -> {status}: {msg}")
        self.status = status


class moe_config(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("F", ctypes.c_int32), ("n_shared", ctypes.c_int32), ("score", ctypes.c_int32),
                ("norm_topk", ctypes.c_int32), ("route_scale", ctypes.c_float), ("expert_dtype", ctypes.c_int32),
                ("compute_aux", ctypes.c_int32), ("save_for_bwd", ctypes.c_int32),
                ("capacity_factor", ctypes.c_float), ("n_group", ctypes.c_int32), ("topk_group", ctypes.c_int32)]


_VP = ctypes.c_void_p
_SZ = ctypes.c_size_t
_I = ctypes.c_int
_CFG = ctypes.POINTER(moe_config)

_SIGS = {
    "moe_status_string": (ctypes.c_char_p, [_I]),
    "moe_get_device_status": (_I, [ctypes.POINTER(ctypes.c_int32), _I]),
    "moe_selftest_wait_timeout": (_I, [_VP]),
    "moe_router_workspace_size": (_SZ, [_CFG]),
    "moe_router_topk": (_I, [_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_permute_workspace_size": (_SZ, [_CFG]),
    "moe_permute": (_I, [_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_permute_noalloc_scratch_capacity": (_SZ, []),
    "moe_permute_noalloc": (_I, [_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "moe_grouped_gemm_workspace_size": (_SZ, [_CFG, _I]),
    "moe_grouped_gemm_fwd": (_I, [_CFG, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_grouped_gemm_bwd_workspace_size": (_SZ, [_CFG, _I]),
    "moe_grouped_gemm_bwd": (_I, [_CFG, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_unpermute": (_I, [_CFG, _VP, _VP, _VP, _VP, _VP]),
    "moe_quantize_mxfp8": (_I, [_VP, ctypes.c_int64, ctypes.c_int32, _VP, _VP, _VP]),
    "moe_nvfp4_sf_bytes": (_SZ, [ctypes.c_int32, ctypes.c_int64, ctypes.c_int32]),
    "moe_quantize_nvfp4": (_I, [_VP, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, _VP, _VP, _VP]),
    "moe_quantize_nvfp4_act": (_I, [_VP, ctypes.c_int64, ctypes.c_int32, _VP, _VP, _VP]),
    "moe_layer_workspace_size": (_SZ, [_CFG]),
    "moe_layer_saved_size": (_SZ, [_CFG]),
    "moe_layer_fwd": (_I, [_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                           _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_layer_bwd_workspace_size": (_SZ, [_CFG]),
    "moe_layer_bwd": (_I, [_CFG, _VP, ctypes.c_float, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                           _VP, _SZ, _VP]),
    "moe_quantize_mxfp8_t": (_I, [_VP, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _VP, ctypes.c_int64, _VP,
                                  _VP]),
    "moe_mxfp8_t_padded_rows": (ctypes.c_int64, [_CFG]),
    "moe_quantize_mxfp8_t_grouped": (_I, [_CFG, ctypes.c_int32, _VP, _VP, _VP, _VP, _VP, ctypes.c_int32, _VP,
                                          ctypes.c_int64, _VP, _VP]),
    "moe_grouped_gemm_dgrad_mxfp8": (_I, [_CFG, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "moe_grouped_gemm_wgrad_mxfp8": (_I, [_CFG, _I, _VP, _VP, _VP, _VP, _VP, ctypes.c_int64, _VP, _VP, _VP]),
    "moe_layer_bwd_mxfp8_workspace_size": (_SZ, [_CFG]),
    "moe_layer_bwd_mxfp8": (_I, [_CFG, _VP, ctypes.c_float, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                                 _VP, _VP, _VP, _SZ, _VP]),
}


def lib_path() -> str:
    return _build.LIB


def load(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load the CUDA library (building it in-tree with nvcc if it is absent or stale)."""
    global _lib
    with _lock:
        if _lib is None:
            if build_if_missing and not _build.up_to_date():
                _build.build()
            if not os.path.exists(_build.LIB):
                raise RuntimeError(f"CUDA library not found: {_build.LIB}")
            lib = ctypes.CDLL(_build.LIB)
            for name, (res, args) in _SIGS.items():
                f = getattr(lib, name)
                f.restype = res
                f.argtypes = args
            _lib = lib
        return _lib


def exported_symbols():
    return list(_SIGS)


# ------------------------------------------------------------------ marshalling

def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    assert t.is_cuda, "device tensors only"
    assert t.is_contiguous()
    return t.data_ptr()


def _st(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check(fn, rc):
    if rc != 0:
        raise MoEError(fn, rc, load().moe_status_string(rc).decode())
    return rc


def make_config(wl=None, **kw) -> moe_config:
    """moe_config from a synthetic.Workload (or keyword fields)."""
    d = dict(T=0, H=0, E=0, k=0, F=0, n_shared=0, score=MOE_SCORE_SOFTMAX, norm_topk=1, route_scale=1.0,
             expert_dtype=MOE_DT_BF16, compute_aux=0, save_for_bwd=0, capacity_factor=0.0, n_group=0, topk_group=0)
    if wl is not None:
        d.update(T=wl.T, H=wl.H, E=wl.E, k=wl.k, F=wl.F, n_shared=wl.S,
                 score=MOE_SCORE_SOFTMAX if wl.score == "softmax" else MOE_SCORE_SIGMOID,
                 norm_topk=int(wl.norm_topk), route_scale=wl.route_scale,
                 expert_dtype=_DTYPES[wl.dtype],
                 compute_aux=int(wl.aux and wl.score == "softmax"), save_for_bwd=int(wl.bwd),
                 capacity_factor=wl.capacity_factor, n_group=wl.n_group, topk_group=wl.topk_group)
    d.update(kw)
    return moe_config(**d)


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ entry points

def moe_status_string(status: int) -> str:
    return load().moe_status_string(status).decode()


def moe_get_device_status(clear: bool = True) -> int:
    w = ctypes.c_int32(0)
    rc = load().moe_get_device_status(ctypes.byref(w), int(clear))
    if rc not in (0, 6):
        _check("moe_get_device_status", rc)
    return int(w.value)


def moe_selftest_wait_timeout(stream=None):
    return _check("moe_selftest_wait_timeout", load().moe_selftest_wait_timeout(_st(stream)))


def moe_router_workspace_size(cfg) -> int:
    return load().moe_router_workspace_size(ctypes.byref(cfg))


def moe_router_topk(cfg, x, W_r, logit_bias, logits, probs, idx, gates, counts, aux, ws, stream=None,
                    expert_bias=None):
    """expert_bias (the DeepSeek-V3 selection bias) is a keyword here; in the C ABI it follows logit_bias."""
    return _check("moe_router_topk", load().moe_router_topk(
        ctypes.byref(cfg), _p(x), _p(W_r), _p(logit_bias), _p(expert_bias), _p(logits), _p(probs), _p(idx), _p(gates), _p(counts),
        _p(aux), _p(ws), ws.numel() if ws is not None else 0, _st(stream)))


def moe_permute_workspace_size(cfg) -> int:
    return load().moe_permute_workspace_size(ctypes.byref(cfg))


def moe_permute(cfg, x, idx, gates, counts, offsets, row_of, src_of, row_gate, xp, xp_sf, ws, stream=None):
    return _check("moe_permute", load().moe_permute(
        ctypes.byref(cfg), _p(x), _p(idx), _p(gates), _p(counts), _p(offsets), _p(row_of), _p(src_of), _p(row_gate),
        _p(xp), _p(xp_sf), _p(ws), ws.numel() if ws is not None else 0, _st(stream)))


def moe_permute_noalloc_scratch_capacity() -> int:
    return load().moe_permute_noalloc_scratch_capacity()


def moe_permute_noalloc(cfg, x, idx, gates, counts, offsets, row_of, src_of, row_gate, xp, xp_sf, stream=None):
    """moe_permute with its scratch in the library's own fixed device array (no workspace argument)."""
    return _check("moe_permute_noalloc", load().moe_permute_noalloc(
        ctypes.byref(cfg), _p(x), _p(idx), _p(gates), _p(counts), _p(offsets), _p(row_of), _p(src_of),
        _p(row_gate), _p(xp), _p(xp_sf), _st(stream)))


def moe_grouped_gemm_workspace_size(cfg, which) -> int:
    return load().moe_grouped_gemm_workspace_size(ctypes.byref(cfg), which)


def moe_grouped_gemm_fwd(cfg, which, A, A_sf, B0, B0_sf, B1, B1_sf, offsets, row_gate, C, C_sf, save_gateup, ws,
                         stream=None):
    return _check("moe_grouped_gemm_fwd", load().moe_grouped_gemm_fwd(
        ctypes.byref(cfg), which, _p(A), _p(A_sf), _p(B0), _p(B0_sf), _p(B1), _p(B1_sf), _p(offsets), _p(row_gate),
        _p(C), _p(C_sf), _p(save_gateup), _p(ws), ws.numel() if ws is not None else 0, _st(stream)))


def moe_grouped_gemm_bwd_workspace_size(cfg, which) -> int:
    return load().moe_grouped_gemm_bwd_workspace_size(ctypes.byref(cfg), which)


def moe_grouped_gemm_bwd(cfg, which, dO, act, saved_gateup, row_gate, W0, W1, offsets, d_in, dg, dW0, dW1, ws,
                         stream=None):
    return _check("moe_grouped_gemm_bwd", load().moe_grouped_gemm_bwd(
        ctypes.byref(cfg), which, _p(dO), _p(act), _p(saved_gateup), _p(row_gate), _p(W0), _p(W1), _p(offsets),
        _p(d_in), _p(dg), _p(dW0), _p(dW1), _p(ws), ws.numel() if ws is not None else 0, _st(stream)))


def moe_unpermute(cfg, o, row_of, extra, y, stream=None):
    return _check("moe_unpermute", load().moe_unpermute(ctypes.byref(cfg), _p(o), _p(row_of), _p(extra), _p(y),
                                                        _st(stream)))


def moe_quantize_mxfp8(src, dst, sf, stream=None):
    K = src.shape[-1]
    rows = src.numel() // K
    return _check("moe_quantize_mxfp8", load().moe_quantize_mxfp8(_p(src), rows, K, _p(dst), _p(sf), _st(stream)))


def moe_nvfp4_sf_bytes(batch: int, R: int, C: int) -> int:
    return int(load().moe_nvfp4_sf_bytes(batch, R, C))


def moe_quantize_nvfp4(src, dst, sf, stream=None):
    """src [batch, R, C] (or [R, C]) bf16 -> dst packed uint8 [..., C/2], sf uint8 of moe_nvfp4_sf_bytes bytes."""
    C = src.shape[-1]
    R = src.shape[-2]
    batch = src.numel() // (R * C)
    return _check("moe_quantize_nvfp4", load().moe_quantize_nvfp4(_p(src), batch, R, C, _p(dst), _p(sf), _st(stream)))


def moe_quantize_nvfp4_act(src, dst, sf, stream=None):
    K = src.shape[-1]
    rows = src.numel() // K
    return _check("moe_quantize_nvfp4_act",
                  load().moe_quantize_nvfp4_act(_p(src), rows, K, _p(dst), _p(sf), _st(stream)))


def moe_layer_workspace_size(cfg) -> int:
    return load().moe_layer_workspace_size(ctypes.byref(cfg))


def moe_layer_saved_size(cfg) -> int:
    return load().moe_layer_saved_size(ctypes.byref(cfg))


def moe_layer_fwd(cfg, x, W_r, logit_bias, W_g, W_u, W_d, W_g_sf, W_u_sf, W_d_sf, Ws_g, Ws_u, Ws_d, Ws_g_sf,
                  Ws_u_sf, Ws_d_sf, y, aux, idx, gates, counts, offsets, saved, ws, stream=None, expert_bias=None):
    """expert_bias (the DeepSeek-V3 selection bias) is a keyword here; in the C ABI it follows logit_bias."""
    return _check("moe_layer_fwd", load().moe_layer_fwd(
        ctypes.byref(cfg), _p(x), _p(W_r), _p(logit_bias), _p(expert_bias), _p(W_g), _p(W_u), _p(W_d), _p(W_g_sf), _p(W_u_sf),
        _p(W_d_sf), _p(Ws_g), _p(Ws_u), _p(Ws_d), _p(Ws_g_sf), _p(Ws_u_sf), _p(Ws_d_sf), _p(y), _p(aux), _p(idx),
        _p(gates), _p(counts), _p(offsets), _p(saved), _p(ws), ws.numel() if ws is not None else 0, _st(stream)))


def moe_layer_bwd_workspace_size(cfg) -> int:
    return load().moe_layer_bwd_workspace_size(ctypes.byref(cfg))


def moe_layer_bwd(cfg, dY, d_aux, x, W_r, W_g, W_u, W_d, saved, dX, dW_r, dW_g, dW_u, dW_d, dlogits, ws,
                  stream=None):
    return _check("moe_layer_bwd", load().moe_layer_bwd(
        ctypes.byref(cfg), _p(dY), float(d_aux), _p(x), _p(W_r), _p(W_g), _p(W_u), _p(W_d), _p(saved), _p(dX),
        _p(dW_r), _p(dW_g), _p(dW_u), _p(dW_d), _p(dlogits), _p(ws), ws.numel() if ws is not None else 0,
        _st(stream)))


def moe_quantize_mxfp8_t(src, dst, sf, ldd=None, col0=0, stream=None):
    """src [B, R, C] bf16 -> dst [B, C, ldd] e4m3 (blocks along R), sf [B, C, ldd/32], written from column
    col0 of each dst row (col0 % 32 == 0; e.g. W_u^T beside W_g^T in one [E, H, 2F] buffer)."""
    B, R, C = src.shape
    assert col0 % 32 == 0
    return _check("moe_quantize_mxfp8_t", load().moe_quantize_mxfp8_t(
        _p(src), B, R, C, _p(dst) + col0, ldd if ldd is not None else R, _p(sf) + col0 // 32, _st(stream)))


def moe_mxfp8_t_padded_rows(cfg) -> int:
    return load().moe_mxfp8_t_padded_rows(ctypes.byref(cfg))


def moe_quantize_mxfp8_t_grouped(cfg, mode, src, src_of, row_gate, offsets, poff, C, dst, ldd, sf, stream=None):
    return _check("moe_quantize_mxfp8_t_grouped", load().moe_quantize_mxfp8_t_grouped(
        ctypes.byref(cfg), mode, _p(src), _p(src_of), _p(row_gate), _p(offsets), _p(poff), C, _p(dst), ldd, _p(sf),
        _st(stream)))


def moe_grouped_gemm_dgrad_mxfp8(cfg, which, A, A_sf, B, B_sf, offsets, saved_gateup, row_gate, out, dg, ws,
                                 stream=None):
    return _check("moe_grouped_gemm_dgrad_mxfp8", load().moe_grouped_gemm_dgrad_mxfp8(
        ctypes.byref(cfg), which, _p(A), _p(A_sf), _p(B), _p(B_sf), _p(offsets), _p(saved_gateup), _p(row_gate),
        _p(out), _p(dg), _p(ws), ws.numel() if ws is not None else 0, _st(stream)))


def moe_grouped_gemm_wgrad_mxfp8(cfg, which, AT, AT_sf, BT, BT_sf, poff, ldp, dW0, dW1, stream=None):
    return _check("moe_grouped_gemm_wgrad_mxfp8", load().moe_grouped_gemm_wgrad_mxfp8(
        ctypes.byref(cfg), which, _p(AT), _p(AT_sf), _p(BT), _p(BT_sf), _p(poff), ldp, _p(dW0), _p(dW1),
        _st(stream)))


def moe_layer_bwd_mxfp8_workspace_size(cfg) -> int:
    return load().moe_layer_bwd_mxfp8_workspace_size(ctypes.byref(cfg))


def moe_layer_bwd_mxfp8(cfg, dY, d_aux, x, W_r, W_dT, W_dT_sf, W_guT, W_guT_sf, saved, dX, dW_r, dW_g, dW_u, dW_d,
                        dlogits, ws, stream=None):
    return _check("moe_layer_bwd_mxfp8", load().moe_layer_bwd_mxfp8(
        ctypes.byref(cfg), _p(dY), ctypes.c_float(d_aux), _p(x), _p(W_r), _p(W_dT), _p(W_dT_sf), _p(W_guT),
        _p(W_guT_sf), _p(saved), _p(dX), _p(dW_r), _p(dW_g), _p(dW_u), _p(dW_d), _p(dlogits), _p(ws),
        ws.numel() if ws is not None else 0, _st(stream)))
