"""ctypes binding of ``liblmoe.so`` (the C ABI in ``include/lmoe.h``).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch provides device memory and streams.  If the library is
missing this module raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblmoe.so")

LMOE_OK = 0
#: device error bits of lmoe_dispatch_noalloc's error word
LMOE_DEVERR_BAD_INDEX = 2
LMOE_DEVERR_REPEATED_INDEX = 8
LMOE_FMT_BF16, LMOE_FMT_MXFP8, LMOE_FMT_MXFP4, LMOE_FMT_NVFP4 = 0, 1, 2, 3
STATUS = {0: "LMOE_OK", -1: "LMOE_ERR_INVALID_ARG", -2: "LMOE_ERR_UNSUPPORTED_SHAPE", -3: "LMOE_ERR_TOO_MANY_TOKENS",
          -4: "LMOE_ERR_CUDA", -5: "LMOE_ERR_TIMEOUT", -6: "LMOE_ERR_BAD_INDEX", -7: "LMOE_ERR_WORKSPACE",
          -8: "LMOE_ERR_BAD_COUNTS"}

P = ctypes.c_void_p
I32 = ctypes.c_int32


class lmoe_config(ctypes.Structure):
    _fields_ = [(n, I32) for n in ("d", "latent", "m", "n_experts", "top_k", "max_tokens", "act", "n_zero", "n_copy",
                                   "n_const", "has_proj", "latent_router", "shared_m", "expert_fmt", "ep_size",
                                   "ep_rank")]


class lmoe_weights(ctypes.Structure):
    _fields_ = [("w_router", P), ("router_bias", P), ("w_down", P), ("w_up", P), ("w1", P), ("w2", P),
                ("const_vecs", P), ("w_shared1", P), ("w_shared2", P), ("w1_scales", P), ("w2_scales", P),
                ("w1_gscale", P), ("w2_gscale", P)]


class lmoe_debug(ctypes.Structure):
    _fields_ = [("topk_idx", P), ("topk_w", P), ("counts", P), ("offsets", P), ("perm", P), ("z", P), ("yl", P),
                ("logits", P)]


class LmoeError(RuntimeError):
    def __init__(self, call: str, status: int):
        super().__init__(f"{call} failed: {STATUS.get(status, status)} ({_text(status)})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load the CUDA library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing (run __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        L.lmoe_workspace_bytes.argtypes = [ctypes.POINTER(lmoe_config)]
        L.lmoe_workspace_bytes.restype = ctypes.c_size_t
        L.lmoe_create.argtypes = [ctypes.POINTER(lmoe_config), ctypes.POINTER(lmoe_weights), P, ctypes.c_size_t,
                                  ctypes.POINTER(P)]
        L.lmoe_forward.argtypes = [P, P, P, I32, P, ctypes.POINTER(lmoe_debug)]
        L.lmoe_forward_host.argtypes = [P, P, P, I32, P]
        L.lmoe_last_error.argtypes = [P]
        L.lmoe_destroy.argtypes = [P]
        L.lmoe_destroy.restype = None
        L.lmoe_status_string.argtypes = [ctypes.c_int]
        L.lmoe_status_string.restype = ctypes.c_char_p
        L.lmoe_set_profiling.argtypes = [P, ctypes.c_int, ctypes.c_int]
        L.lmoe_phase_times.argtypes = [P, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(I32)]
        L.lmoe_num_phases.argtypes = []
        L.lmoe_phase_name.argtypes = [ctypes.c_int]
        L.lmoe_phase_name.restype = ctypes.c_char_p
        L.lmoe_routing_stats.argtypes = [P, ctypes.POINTER(I32)]
        L.lmoe_set_small_rows.argtypes = [P, I32]
        L.lmoe_set_wait_timeout.argtypes = [P, ctypes.c_uint64]
        L.lmoe_set_graph_launch.argtypes = [P, ctypes.c_int]
        L.lmoe_set_grouped_gemm.argtypes = [P, ctypes.c_int]
        L.lmoe_gemm_bf16.argtypes = [P, P, P, I32, I32, I32, P, P]
        L.lmoe_dispatch_noalloc.argtypes = [P, I32, I32, I32, P, P, P, P, P, P]
        L.lmoe_selftest_wait.argtypes = [P, ctypes.c_uint64, P]
        L.lmoe_mx_encode_weights.argtypes = [P, ctypes.c_int64, I32, I32, P, P, P]
        L.lmoe_nvfp4_encode_weights.argtypes = [P, I32, ctypes.c_int64, I32, P, P, P, P]
        L.lmoe_ep_dispatch.argtypes = [P, P, I32, P, P, P]
        L.lmoe_ep_experts.argtypes = [P, P, P, I32, I32, P, P]
        L.lmoe_ep_combine.argtypes = [P, P, P, P]
        L.lmoe_ep_block_rows.argtypes = [P]
        L.lmoe_ep_block_rows.restype = ctypes.c_int64
        L.lmoe_ep_dispatch_blocks.argtypes = [P, P, I32, P, I32, P, P]
        L.lmoe_ep_experts_blocks.argtypes = [P, P, I32, P, I32, P, P]
        L.lmoe_ep_combine_blocks.argtypes = [P, P, P, P]
        _lib = L
    return _lib


def _text(status: int) -> str:
    try:
        return lib().lmoe_status_string(int(status)).decode()
    except Exception:  # pragma: no cover - only while reporting another error
        return "?"


def _check(call: str, status: int) -> None:
    if status != LMOE_OK:
        raise LmoeError(call, status)


def _p(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ------------------------------------------------------------------ C-ABI calls, same names
def lmoe_workspace_bytes(cfg: lmoe_config) -> int:
    return int(lib().lmoe_workspace_bytes(ctypes.byref(cfg)))


def lmoe_create(cfg: lmoe_config, weights: lmoe_weights, workspace: int, nbytes: int) -> int:
    h = P()
    _check("lmoe_create", lib().lmoe_create(ctypes.byref(cfg), ctypes.byref(weights), workspace, nbytes,
                                            ctypes.byref(h)))
    return h.value


def lmoe_forward(h: int, x: int, y: int, T: int, stream: Optional[int], dbg: Optional[lmoe_debug] = None) -> None:
    _check("lmoe_forward", lib().lmoe_forward(h, x, y, T, stream, ctypes.byref(dbg) if dbg is not None else None))


def lmoe_forward_host(h: int, x_host: int, y_host: int, T: int, stream: Optional[int]) -> None:
    _check("lmoe_forward_host", lib().lmoe_forward_host(h, x_host, y_host, T, stream))


def lmoe_last_error(h: int) -> int:
    return int(lib().lmoe_last_error(h))


def lmoe_destroy(h: int) -> None:
    lib().lmoe_destroy(h)


def lmoe_status_string(status: int) -> str:
    return _text(status)


def lmoe_set_profiling(h: int, enable: bool, max_forwards: int = 1) -> None:
    _check("lmoe_set_profiling", lib().lmoe_set_profiling(h, int(enable), int(max_forwards)))


def lmoe_num_phases() -> int:
    return int(lib().lmoe_num_phases())


def lmoe_phase_name(i: int) -> str:
    return lib().lmoe_phase_name(i).decode()


def lmoe_phase_times(h: int) -> Dict[str, tuple]:
    n = lmoe_num_phases()
    ms = (ctypes.c_float * n)()
    nl = (I32 * n)()
    _check("lmoe_phase_times", lib().lmoe_phase_times(h, ms, nl))
    return {lmoe_phase_name(i): (float(ms[i]), int(nl[i])) for i in range(n)}


def lmoe_routing_stats(h: int) -> Dict[str, int]:
    out = (I32 * 8)()
    _check("lmoe_routing_stats", lib().lmoe_routing_stats(h, out))
    return {"ffn_rows": out[0], "experts_touched": out[1], "tc_mtiles": out[2], "stream_experts": out[3],
            "stream_rows": out[4], "tc_experts": out[5], "tc_rows": out[6], "small_rows_threshold": out[7]}


def lmoe_set_small_rows(h: int, rows: int) -> None:
    _check("lmoe_set_small_rows", lib().lmoe_set_small_rows(h, rows))


def lmoe_set_wait_timeout(h: int, ns: int) -> None:
    _check("lmoe_set_wait_timeout", lib().lmoe_set_wait_timeout(h, ns))


def lmoe_set_graph_launch(h: int, enable: bool) -> None:
    """Launch each forward as one CUDA graph (default) or its kernels one by one."""
    _check("lmoe_set_graph_launch", lib().lmoe_set_graph_launch(h, 1 if enable else 0))


def lmoe_set_grouped_gemm(h: int, kind: int) -> None:
    """Grouped expert GEMM kernel: 1 (default) CTA pairs, transposed; 0 single-CTA 128-row tiles."""
    _check("lmoe_set_grouped_gemm", lib().lmoe_set_grouped_gemm(h, int(kind)))


def lmoe_selftest_wait(h: int, timeout_ns: int, stream=None) -> None:
    _check("lmoe_selftest_wait", lib().lmoe_selftest_wait(h, timeout_ns, _stream(stream)))


def lmoe_gemm_bf16(A: torch.Tensor, B: torch.Tensor, C: torch.Tensor, err: torch.Tensor, stream=None) -> None:
    """C = A @ B^T on the tensor-core kernel (bf16 in/out, fp32 accumulate)."""
    M, K = A.shape
    N = B.shape[0]
    _check("lmoe_gemm_bf16", lib().lmoe_gemm_bf16(A.data_ptr(), B.data_ptr(), C.data_ptr(), M, N, K, _stream(stream),
                                                  err.data_ptr()))


def _int32_buffer(name: str, t: torch.Tensor, device: torch.device, numel: int) -> None:
    """Raise ValueError unless ``t`` is a contiguous int32 tensor on ``device`` with at least ``numel`` elements."""
    if not isinstance(t, torch.Tensor) or t.dtype != torch.int32 or t.device != device or not t.is_contiguous():
        raise ValueError(f"{name}: a contiguous int32 tensor on {device} is required")
    if t.numel() < numel:
        raise ValueError(f"{name}: {t.numel()} elements, at least {numel} required")


def lmoe_dispatch_noalloc(idx: torch.Tensor, n_total: int, counts: torch.Tensor, offsets: torch.Tensor,
                          perm: torch.Tensor, inv: torch.Tensor, err: Optional[torch.Tensor] = None,
                          stream=None) -> None:
    """Expert counting sort of ``idx`` [T, top_k] (int32, device) into caller buffers, with no device
    allocation: the library's fixed scratch array serves as workspace (see ``include/lmoe.h``).  ``err``
    (optional, one int32 on the device) receives the call's device error bits (``LMOE_DEVERR_*``)."""
    if idx.dim() != 2 or idx.device.type != "cuda":
        raise ValueError("idx: a [T, top_k] tensor on a CUDA device is required")
    T, K = idx.shape
    _int32_buffer("idx", idx, idx.device, T * K)
    _int32_buffer("counts", counts, idx.device, n_total)
    _int32_buffer("offsets", offsets, idx.device, n_total + 1)
    _int32_buffer("perm", perm, idx.device, T * K)
    _int32_buffer("inv", inv, idx.device, T * K)
    if err is not None:
        _int32_buffer("err", err, idx.device, 1)
    _check("lmoe_dispatch_noalloc", lib().lmoe_dispatch_noalloc(
        _p(idx), T, K, n_total, _p(counts), _p(offsets), _p(perm), _p(inv), _p(err), _stream(stream)))


def lmoe_mx_encode_weights(w: torch.Tensor, fmt: int, stream=None):
    """Block-scaled (MX) encoding of a device bf16 weight tensor viewed as rows x K (K = last dimension).

    Returns ``(codes, scales)`` as new device uint8 tensors: codes [rows, K] (MXFP8) or [rows, K/2] (MXFP4,
    element 2i in the low nibble of byte i), scales rows*K/32 bytes in the tensor-core atom order that
    ``include/lmoe.h`` describes.
    """
    K = int(w.shape[-1])
    rows = w.numel() // K
    codes = torch.empty((rows, K if fmt == LMOE_FMT_MXFP8 else K // 2), dtype=torch.uint8, device=w.device)
    scales = torch.empty(rows * K // 32, dtype=torch.uint8, device=w.device)
    _check("lmoe_mx_encode_weights", lib().lmoe_mx_encode_weights(
        w.data_ptr(), rows, K, int(fmt), codes.data_ptr(), scales.data_ptr(), _stream(stream)))
    return codes, scales


def lmoe_ep_dispatch(h: int, x: torch.Tensor, send_rows: torch.Tensor, send_counts: torch.Tensor,
                     stream=None) -> None:
    """Expert-parallel stage 1 for the rows of ``x`` (device bf16 [T, d])."""
    _check("lmoe_ep_dispatch", lib().lmoe_ep_dispatch(h, x.data_ptr(), int(x.shape[0]), send_rows.data_ptr(),
                                                      send_counts.data_ptr(), _stream(stream)))


def lmoe_ep_experts(h: int, recv_rows: torch.Tensor, recv_counts: torch.Tensor, n_recv: int, rows_bound: int,
                    out_rows: torch.Tensor, stream=None) -> None:
    """Expert-parallel stage 2: this rank's experts on ``n_recv`` received rows."""
    _check("lmoe_ep_experts", lib().lmoe_ep_experts(h, recv_rows.data_ptr(), recv_counts.data_ptr(), int(n_recv),
                                                    int(rows_bound), out_rows.data_ptr(), _stream(stream)))


def lmoe_ep_combine(h: int, ret_rows: torch.Tensor, y: torch.Tensor, stream=None) -> None:
    """Expert-parallel stage 3: aggregation, W_up and residual into ``y``."""
    _check("lmoe_ep_combine", lib().lmoe_ep_combine(h, ret_rows.data_ptr(), y.data_ptr(), _stream(stream)))


def lmoe_ep_block_rows(h: int) -> int:
    """Rows of one rank-pair block of the block exchange (the most one rank can send one other rank)."""
    return int(lib().lmoe_ep_block_rows(h))


def lmoe_ep_dispatch_blocks(h: int, x: torch.Tensor, send_blocks: torch.Tensor, block_rows: int,
                            send_counts: torch.Tensor, stream=None) -> None:
    """Expert-parallel stage 1, block exchange: rank r's rows at rows r * block_rows of ``send_blocks``."""
    _check("lmoe_ep_dispatch_blocks", lib().lmoe_ep_dispatch_blocks(
        h, x.data_ptr(), int(x.shape[0]), send_blocks.data_ptr(), int(block_rows), send_counts.data_ptr(),
        _stream(stream)))


def lmoe_ep_experts_blocks(h: int, recv_blocks: torch.Tensor, block_rows: int, recv_counts: torch.Tensor,
                           rows_bound: int, out_blocks: torch.Tensor, stream=None) -> None:
    """Expert-parallel stage 2, block exchange: block s of ``recv_blocks`` holds rank s's rows."""
    _check("lmoe_ep_experts_blocks", lib().lmoe_ep_experts_blocks(
        h, recv_blocks.data_ptr(), int(block_rows), recv_counts.data_ptr(), int(rows_bound), out_blocks.data_ptr(),
        _stream(stream)))


def lmoe_ep_combine_blocks(h: int, ret_blocks: torch.Tensor, y: torch.Tensor, stream=None) -> None:
    """Expert-parallel stage 3, block exchange: the expert outputs in the layout of the send blocks."""
    _check("lmoe_ep_combine_blocks", lib().lmoe_ep_combine_blocks(h, ret_blocks.data_ptr(), y.data_ptr(),
                                                                  _stream(stream)))


def lmoe_nvfp4_encode_weights(w: torch.Tensor, stream=None):
    """NVFP4 encoding of a device bf16 tensor of matrices ``[n_mats, rows_per_mat, K]``.

    Returns ``(codes, scales, gscale)`` as new device tensors: codes uint8 [n_mats * rows_per_mat, K/2] (element
    2i in the low nibble of byte i), scales uint8 in the tensor-core atom order ``include/lmoe.h`` describes,
    gscale fp32 [n_mats].
    """
    n_mats, rows_per_mat, K = (int(v) for v in w.shape)
    codes = torch.empty((n_mats * rows_per_mat, K // 2), dtype=torch.uint8, device=w.device)
    scales = torch.empty(n_mats * rows_per_mat * K // 16, dtype=torch.uint8, device=w.device)
    gscale = torch.empty(n_mats, dtype=torch.float32, device=w.device)
    _check("lmoe_nvfp4_encode_weights", lib().lmoe_nvfp4_encode_weights(
        w.data_ptr(), n_mats, rows_per_mat, K, codes.data_ptr(), scales.data_ptr(), gscale.data_ptr(),
        _stream(stream)))
    return codes, scales, gscale


# ------------------------------------------------------------------ convenience owner of a layer
def make_config(cfg, max_tokens: int, ep_size: int = 0, ep_rank: int = 0) -> lmoe_config:
    return lmoe_config(cfg.d, cfg.latent, cfg.m, cfg.n_ffn, cfg.top_k, int(max_tokens), cfg.act, cfg.n_zero,
                       cfg.n_copy, cfg.n_const, cfg.has_proj, cfg.latent_router, getattr(cfg, "shared_m", 0),
                       getattr(cfg, "expert_fmt", 0), int(ep_size), int(ep_rank))


class LatentMoE:
    """A layer on one GPU: device copies of the weights, a workspace and a handle.

    ``cfg`` is a ``synth.LayerConfig`` (or anything with the same fields),
    ``layer`` the dict of CPU tensors from ``synth.make_layer``.  With a
    block-scaled ``cfg.expert_fmt`` the bf16 W1 / W2 are encoded on the device
    (``lmoe_mx_encode_weights``, or ``lmoe_nvfp4_encode_weights`` for NVFP4)
    and only the encodings are kept.  With
    ``ep_size`` > 1 the handle is one rank of an expert-parallel layer:
    ``layer['w1']`` / ``layer['w2']`` must then hold that rank's experts only
    (see ``expert_parallel``).
    """

    def __init__(self, cfg, layer: Dict[str, torch.Tensor], max_tokens: int, device: str = "cuda",
                 ep_size: int = 0, ep_rank: int = 0):
        self.cfg = cfg
        self.device = torch.device(device)
        self.max_tokens = int(max_tokens)
        dev = lambda t: None if t is None else t.to(self.device).contiguous()  # noqa: E731
        self.w = {k: dev(layer.get(k)) for k in ("w_router", "bias", "w_down", "w_up", "w1", "w2", "const_vecs",
                                                  "w_shared1", "w_shared2")}
        self.w["w1_scales"] = self.w["w2_scales"] = self.w["w1_gscale"] = self.w["w2_gscale"] = None
        fmt = getattr(cfg, "expert_fmt", 0)
        if fmt == LMOE_FMT_NVFP4:
            with torch.cuda.device(self.device):
                for k in ("w1", "w2"):
                    self.w[k], self.w[k + "_scales"], self.w[k + "_gscale"] = lmoe_nvfp4_encode_weights(self.w[k])
                torch.cuda.synchronize(self.device)
        elif fmt != LMOE_FMT_BF16:
            with torch.cuda.device(self.device):
                for k in ("w1", "w2"):
                    self.w[k], self.w[k + "_scales"] = lmoe_mx_encode_weights(self.w[k], fmt)
                torch.cuda.synchronize(self.device)
        self.c = make_config(cfg, self.max_tokens, ep_size, ep_rank)
        nbytes = lmoe_workspace_bytes(self.c)
        if nbytes == 0:
            raise LmoeError("lmoe_workspace_bytes", -2)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self.weights = lmoe_weights(_p(self.w["w_router"]), _p(self.w["bias"]), _p(self.w["w_down"]),
                                    _p(self.w["w_up"]), _p(self.w["w1"]), _p(self.w["w2"]), _p(self.w["const_vecs"]),
                                    _p(self.w["w_shared1"]), _p(self.w["w_shared2"]), _p(self.w["w1_scales"]),
                                    _p(self.w["w2_scales"]), _p(self.w["w1_gscale"]), _p(self.w["w2_gscale"]))
        with torch.cuda.device(self.device):
            self.h = lmoe_create(self.c, self.weights, self.workspace.data_ptr(), nbytes)

    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, debug: bool = False, stream=None):
        T = int(x.shape[0])
        if y is None:
            y = torch.empty_like(x)
        dbg = None
        out = {}
        if debug:
            K, L, nt = self.cfg.top_k, self.cfg.latent, self.cfg.n_total
            out = {"idx": torch.empty((T, K), dtype=torch.int32, device=self.device),
                   "w": torch.empty((T, K), dtype=torch.float32, device=self.device),
                   "counts": torch.empty(nt, dtype=torch.int32, device=self.device),
                   "offsets": torch.empty(nt + 1, dtype=torch.int32, device=self.device),
                   "perm": torch.empty(T * K, dtype=torch.int32, device=self.device),
                   "logits": torch.empty((T, nt), dtype=torch.float32, device=self.device)}
            if self.cfg.has_proj:
                out["z"] = torch.empty((T, L), dtype=torch.bfloat16, device=self.device)
                out["yl"] = torch.empty((T, L), dtype=torch.bfloat16, device=self.device)
            dbg = lmoe_debug(_p(out["idx"]), _p(out["w"]), _p(out["counts"]), _p(out["offsets"]), _p(out["perm"]),
                             _p(out.get("z")), _p(out.get("yl")), _p(out["logits"]))
        lmoe_forward(self.h, x.data_ptr(), y.data_ptr(), T, _stream(stream), dbg)
        return (y, out) if debug else y

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, stream=None) -> None:
        lmoe_forward_host(self.h, x_host.data_ptr(), y_host.data_ptr(), int(x_host.shape[0]), _stream(stream))

    def last_error(self) -> int:
        return lmoe_last_error(self.h)

    def close(self) -> None:
        if getattr(self, "h", None):
            lmoe_destroy(self.h)
            self.h = None

    def __del__(self):  # pragma: no cover - interpreter shutdown order varies
        try:
            self.close()
        except Exception:
            pass
