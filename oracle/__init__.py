"""fp64 CPU oracle for the LatentMoE layer forward (ctypes wrapper of ``oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg are the only callers.  The product path never imports this
package, and this package never imports the product's CUDA library.

Each function follows the layer as the pages describe it; ``oracle.c`` states
the steps and their sources.  Inputs are the bf16 tensors from
``latent_mixture_experts_gemm_b200.synth`` (widened exactly); every output is
fp64 (indices int32).
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import numpy as np
import torch

from . import build as _build

_lib = None


class _Cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "d", "latent", "m", "n_ffn", "top_k", "act", "n_zero", "n_copy", "n_const", "has_proj", "latent_router",
        "shared_m", "expert_fmt")]


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        L.oracle_forward.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int] + [P] * 17
        L.oracle_forward.restype = ctypes.c_int
        L.oracle_route.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P]
        L.oracle_route.restype = ctypes.c_int
        L.oracle_dispatch.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, P, P]
        L.oracle_dispatch.restype = ctypes.c_int
        L.oracle_mx_quantize.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
        L.oracle_mx_quantize.restype = ctypes.c_int
        L.oracle_mx_dequantize.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
        L.oracle_mx_dequantize.restype = ctypes.c_int
        L.oracle_nv_tensor_scale.argtypes = [P, ctypes.c_longlong]
        L.oracle_nv_tensor_scale.restype = ctypes.c_float
        L.oracle_nv_quantize.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_float, P, P]
        L.oracle_nv_quantize.restype = ctypes.c_int
        L.oracle_nv_dequantize.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_float, P]
        L.oracle_nv_dequantize.restype = ctypes.c_int
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_set_num_threads.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


def _cfg(cfg) -> _Cfg:
    return _Cfg(cfg.d, cfg.latent, cfg.m, cfg.n_ffn, cfg.top_k, cfg.act, cfg.n_zero, cfg.n_copy, cfg.n_const,
                cfg.has_proj, cfg.latent_router, getattr(cfg, "shared_m", 0), getattr(cfg, "expert_fmt", 0))


def _bits(t: Optional[torch.Tensor]):
    """bf16 tensor -> contiguous uint16 numpy array of its bit patterns (or None)."""
    if t is None:
        return None
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _ptr(a) -> Optional[int]:
    return None if a is None else a.ctypes.data


def forward(cfg, layer: Dict[str, torch.Tensor], x: Optional[torch.Tensor] = None,
            idx: Optional[np.ndarray] = None, want: tuple = ("y", "idx", "w")) -> Dict[str, np.ndarray]:
    """Layer forward in fp64 for the rows of ``x`` (default ``layer['x']``).

    ``idx`` ([T,K'] int32), if given, replaces the router's own selection (the
    weights are still the renormalised softmax of the router logits at those
    ids).  ``want`` names the outputs to return among y, idx, w, z, yl, logits.
    """
    x = layer["x"] if x is None else x
    T = int(x.shape[0])
    K, Nt, L = cfg.top_k, cfg.n_total, cfg.latent
    keep = []
    xb = _bits(x)
    wr = _bits(layer["w_router"])
    wd = _bits(layer.get("w_down"))
    wu = _bits(layer.get("w_up"))
    w1 = _bits(layer["w1"])
    w2 = _bits(layer["w2"])
    cv = _bits(layer.get("const_vecs"))
    ws1 = _bits(layer.get("w_shared1"))
    ws2 = _bits(layer.get("w_shared2"))
    bias = layer.get("bias")
    bias_np = None if bias is None else bias.detach().cpu().to(torch.float32).contiguous().numpy()
    keep += [xb, wr, wd, wu, w1, w2, cv, ws1, ws2, bias_np]
    idx_in = None if idx is None else np.ascontiguousarray(idx, dtype=np.int32)
    out = {"y": np.empty((T, cfg.d), np.float64), "idx": np.empty((T, K), np.int32), "w": np.empty((T, K), np.float64)}
    if "z" in want:
        out["z"] = np.empty((T, L), np.float64)
    if "yl" in want:
        out["yl"] = np.empty((T, L), np.float64)
    if "logits" in want:
        out["logits"] = np.empty((T, Nt), np.float64)
    c = _cfg(cfg)
    rc = lib().oracle_forward(ctypes.byref(c), T, _ptr(xb), _ptr(wr), _ptr(bias_np), _ptr(wd), _ptr(wu), _ptr(w1),
                              _ptr(w2), _ptr(cv), _ptr(ws1), _ptr(ws2), _ptr(idx_in), _ptr(out["y"]), _ptr(out["idx"]),
                              _ptr(out["w"]),
                              _ptr(out.get("z")), _ptr(out.get("yl")), _ptr(out.get("logits")))
    if rc != 0:
        raise ValueError("oracle_forward rejected its arguments")
    del keep
    return {k: v for k, v in out.items() if k in want}


def route(logits: np.ndarray, top_k: int):
    """Top-K' selection (ties to the lower id) and renormalised softmax, per row."""
    lg = np.ascontiguousarray(logits, dtype=np.float64)
    T, Nt = lg.shape
    idx = np.empty((T, top_k), np.int32)
    w = np.empty((T, top_k), np.float64)
    if lib().oracle_route(T, Nt, top_k, lg.ctypes.data, idx.ctypes.data, w.ctypes.data) != 0:
        raise ValueError("oracle_route rejected its arguments")
    return idx, w


def dispatch(idx: np.ndarray, n_total: int):
    """Stable counting sort of the flat slots by expert: counts, offsets, perm, inv."""
    ix = np.ascontiguousarray(idx, dtype=np.int32)
    T, K = ix.shape
    counts = np.empty(n_total, np.int32)
    offsets = np.empty(n_total + 1, np.int32)
    perm = np.empty(T * K, np.int32)
    inv = np.empty(T * K, np.int32)
    rc = lib().oracle_dispatch(T, K, n_total, ix.ctypes.data, counts.ctypes.data, offsets.ctypes.data,
                               perm.ctypes.data, inv.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_dispatch: expert id out of range")
    return counts, offsets, perm, inv


#: block-scaled formats of the expert weights (``expert_fmt``)
FMT_BF16, FMT_MXFP8, FMT_MXFP4, FMT_NVFP4 = 0, 1, 2, 3


def mx_quantize(w: torch.Tensor, fmt: int):
    """MX encoding of a bf16 matrix [rows, K] (K a multiple of 32).

    Returns ``(codes, scales)``: uint8 [rows, K] element codes, one per byte
    (E4M3 for MXFP8; E2M1 in the low nibble for MXFP4), and uint8
    [rows, K/32] E8M0 scale bytes (value 2^(byte - 127)).
    """
    w2 = w.reshape(-1, w.shape[-1])
    rows, K = int(w2.shape[0]), int(w2.shape[1])
    wb = _bits(w2)
    codes = np.empty((rows, K), np.uint8)
    scales = np.empty((rows, max(K // 32, 1)), np.uint8)
    if lib().oracle_mx_quantize(wb.ctypes.data, rows, K, int(fmt), codes.ctypes.data, scales.ctypes.data) != 0:
        raise ValueError("oracle_mx_quantize rejected its arguments")
    return codes, scales


def mx_dequantize(codes: np.ndarray, scales: np.ndarray, fmt: int) -> np.ndarray:
    """The fp64 values an MX encoding from :func:`mx_quantize` stands for."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, K = c.shape
    out = np.empty((rows, K), np.float64)
    if lib().oracle_mx_dequantize(c.ctypes.data, s.ctypes.data, rows, K, int(fmt), out.ctypes.data) != 0:
        raise ValueError("oracle_mx_dequantize rejected its arguments")
    return out


def nv_tensor_scale(w: torch.Tensor) -> float:
    """NVFP4 fp32 tensor scale of a bf16 tensor: amax / (6 * 448), 1 when all zero."""
    wb = _bits(w.reshape(-1))
    return float(lib().oracle_nv_tensor_scale(wb.ctypes.data, wb.size))


def nv_quantize(w: torch.Tensor, g: float):
    """NVFP4 encoding of a bf16 matrix [rows, K] (K a multiple of 16) with tensor scale ``g``.

    Returns ``(codes, scales)``: uint8 [rows, K] E2M1 codes, one per byte, and
    uint8 [rows, K/16] E4M3 block-scale bytes.
    """
    w2 = w.reshape(-1, w.shape[-1])
    rows, K = int(w2.shape[0]), int(w2.shape[1])
    wb = _bits(w2)
    codes = np.empty((rows, K), np.uint8)
    scales = np.empty((rows, max(K // 16, 1)), np.uint8)
    if lib().oracle_nv_quantize(wb.ctypes.data, rows, K, float(g), codes.ctypes.data, scales.ctypes.data) != 0:
        raise ValueError("oracle_nv_quantize rejected its arguments")
    return codes, scales


def nv_dequantize(codes: np.ndarray, scales: np.ndarray, g: float) -> np.ndarray:
    """The fp64 values an NVFP4 encoding from :func:`nv_quantize` stands for."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, K = c.shape
    out = np.empty((rows, K), np.float64)
    if lib().oracle_nv_dequantize(c.ctypes.data, s.ctypes.data, rows, K, float(g), out.ctypes.data) != 0:
        raise ValueError("oracle_nv_dequantize rejected its arguments")
    return out
