"""The C-ABI library loads and exports every entry point include/*.h declares; host-side
argument checks reject bad input before any CUDA call (these run without a GPU)."""
import ctypes
import glob
import os
import re

import pytest

from latent_mixture_experts_gemm_b200 import lmoe, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for hdr in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = re.sub(r"/\*.*?\*/", "", open(hdr).read(), flags=re.S)
        names.update(re.findall(r"LMOE_API\s+[\w\s\*]*?\b(lmoe_\w+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("lmoe_workspace_bytes", "lmoe_create", "lmoe_forward", "lmoe_forward_host", "lmoe_last_error",
                     "lmoe_destroy", "lmoe_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol():
    L = lmoe.lib()
    for name in _declared_functions():
        assert hasattr(L, name), name


def test_status_strings():
    for code in lmoe.STATUS:
        assert lmoe.lmoe_status_string(code) not in ("", "unknown status")
    assert lmoe.lmoe_status_string(12345) == "unknown status"


def test_workspace_bytes_and_shape_checks():
    ok = lmoe.make_config(synth.WORKLOADS["nemotron_prefill"], 8192)
    n = lmoe.lmoe_workspace_bytes(ok)
    assert n > 2 * 8192 * 22 * 1024 * 2   # at least the gathered rows (reused for outputs) and hidden rows
    small = lmoe.make_config(synth.WORKLOADS["tiny"], 64)
    assert 0 < lmoe.lmoe_workspace_bytes(small) < n
    bad = [dict(d=100), dict(latent=0), dict(m=32), dict(top_k=0), dict(top_k=33), dict(n_experts=0),
           dict(max_tokens=0), dict(act=7), dict(has_proj=0), dict(shared_m=100), dict(shared_m=-64)]
    for b in bad:
        c = lmoe.make_config(synth.WORKLOADS["tiny"], 64)
        for k, v in b.items():
            setattr(c, k, v)
        assert lmoe.lmoe_workspace_bytes(c) == 0, b
    c = lmoe.make_config(synth.WORKLOADS["tiny"], 64)
    c.n_experts = 1020
    c.n_zero = 5           # n_total 1025 > 1024
    assert lmoe.lmoe_workspace_bytes(c) == 0


def test_create_rejects_before_touching_the_device():
    L = lmoe.lib()
    cfg = lmoe.make_config(synth.WORKLOADS["tiny"], 64)
    w = lmoe.lmoe_weights()
    h = ctypes.c_void_p()
    assert L.lmoe_create(None, ctypes.byref(w), None, 0, ctypes.byref(h)) == -1
    bad = lmoe.make_config(synth.WORKLOADS["tiny"], 64)
    bad.d = 65
    assert L.lmoe_create(ctypes.byref(bad), ctypes.byref(w), None, 0, ctypes.byref(h)) == -2
    assert L.lmoe_create(ctypes.byref(cfg), ctypes.byref(w), None, 0, ctypes.byref(h)) == -7
    # a workspace that is large enough but misaligned, then missing weights
    big = lmoe.lmoe_workspace_bytes(cfg)
    assert L.lmoe_create(ctypes.byref(cfg), ctypes.byref(w), 0x1001, big, ctypes.byref(h)) == -1
    assert L.lmoe_create(ctypes.byref(cfg), ctypes.byref(w), 0x10000, big, ctypes.byref(h)) == -1
    assert h.value is None


def test_null_handle_calls_are_rejected():
    L = lmoe.lib()
    assert L.lmoe_forward(None, None, None, 1, None, None) == -1
    assert L.lmoe_forward_host(None, None, None, 1, None) == -1
    assert L.lmoe_last_error(None) == -1
    assert L.lmoe_set_profiling(None, 1, 1) == -1
    L.lmoe_destroy(None)
    assert L.lmoe_ep_dispatch(None, None, 1, None, None, None) == -1
    assert L.lmoe_ep_experts(None, None, None, 1, 1, None, None) == -1
    assert L.lmoe_ep_combine(None, None, None, None) == -1
    assert L.lmoe_set_graph_launch(None, 1) == -1
    assert lmoe.lmoe_num_phases() == 11
    assert lmoe.lmoe_phase_name(10) == "ep_regroup"
    assert L.lmoe_set_grouped_gemm(None, 1) == -1
    assert [lmoe.lmoe_phase_name(i) for i in range(3)] == ["router_proj_gemm", "topk_softmax", "dispatch"]


def test_gemm_shape_checks():
    L = lmoe.lib()
    assert L.lmoe_gemm_bf16(0x100, 0x100, 0x100, 128, 100, 64, None, 0x100) == -2
    assert L.lmoe_gemm_bf16(0x100, 0x100, 0x100, 128, 64, 96, None, 0x100) == -2
    assert L.lmoe_gemm_bf16(0x100, 0x100, 0x100, 128, 64, 64, None, None) == -1


def test_block_scaled_config_and_encoder_checks():
    L = lmoe.lib()
    ok = lmoe.make_config(synth.WORKLOADS["nemotron_decode_mxfp4"], 32)
    assert lmoe.lmoe_workspace_bytes(ok) > lmoe.lmoe_workspace_bytes(lmoe.make_config(synth.WORKLOADS["nemotron_decode"], 32))
    # block-scaled experts: latent and m whole 128-element stages, formats 0..3; any batch size
    big_batch = lmoe.make_config(synth.WORKLOADS["nemotron_decode_mxfp8"], 4096)
    assert lmoe.lmoe_workspace_bytes(big_batch) > 0
    for b in (dict(latent=192), dict(m=320), dict(expert_fmt=4), dict(expert_fmt=-1)):
        c = lmoe.make_config(synth.WORKLOADS["nemotron_decode_mxfp8"], 32)
        for k, v in b.items():
            setattr(c, k, v)
        assert lmoe.lmoe_workspace_bytes(c) == 0, b
    # a block-scaled layer without scale pointers, and MXFP4 codes off the 32-byte grid, are rejected
    cfg = lmoe.make_config(synth.WORKLOADS["nemotron_decode_mxfp4"], 32)
    big = lmoe.lmoe_workspace_bytes(cfg)
    h = ctypes.c_void_p()
    w = lmoe.lmoe_weights(w_router=0x10000, w_down=0x10000, w_up=0x10000, w1=0x10000, w2=0x10000)
    assert L.lmoe_create(ctypes.byref(cfg), ctypes.byref(w), 0x100000, big, ctypes.byref(h)) == -1
    w = lmoe.lmoe_weights(w_router=0x10000, w_down=0x10000, w_up=0x10000, w1=0x10010, w2=0x10000,
                          w1_scales=0x20000, w2_scales=0x20000)
    assert L.lmoe_create(ctypes.byref(cfg), ctypes.byref(w), 0x100000, big, ctypes.byref(h)) == -1
    assert h.value is None
    # the encoder checks sizes and format before anything else
    assert L.lmoe_mx_encode_weights(0x100, 100, 128, 1, 0x100, 0x100, None) == -2
    assert L.lmoe_mx_encode_weights(0x100, 128, 96, 2, 0x100, 0x100, None) == -2
    assert L.lmoe_mx_encode_weights(0x100, 128, 128, 0, 0x100, 0x100, None) == -2
    assert L.lmoe_mx_encode_weights(None, 128, 128, 1, 0x100, 0x100, None) == -1
    assert L.lmoe_mx_encode_weights(0x108, 128, 128, 1, 0x100, 0x100, None) == -1
    assert L.lmoe_mx_encode_weights(0x100, 0, 128, 1, None, None, None) == 0


def test_expert_parallel_config_checks():
    wl = synth.WORKLOADS["nemotron_prefill"]          # 512 FFN experts, top-22
    one = lmoe.lmoe_workspace_bytes(lmoe.make_config(wl, 8192))
    ep8 = lmoe.lmoe_workspace_bytes(lmoe.make_config(wl, 8192, ep_size=8, ep_rank=7))
    # the expert side holds up to 8 ranks x 8192 tokens x 22 rows, each a latent row and a hidden row
    assert ep8 > one + 7 * 8192 * 22 * (1024 + 1024) * 2
    assert lmoe.lmoe_workspace_bytes(lmoe.make_config(wl, 8192, ep_size=1)) == one
    for ep, rank in ((3, 0), (8, 8), (8, -1), (-1, 0), (0, 1), (1, 1), (2048, 0), (1024, 0)):
        assert lmoe.lmoe_workspace_bytes(lmoe.make_config(wl, 8192, ep_size=ep, ep_rank=rank)) == 0, (ep, rank)
    # block-scaled experts are not split; the expert-side capacity must stay below 2^30 rows
    assert lmoe.lmoe_workspace_bytes(lmoe.make_config(synth.WORKLOADS["nemotron_decode_mxfp8"], 32, ep_size=2)) == 0
    assert lmoe.lmoe_workspace_bytes(lmoe.make_config(wl, 1 << 25, ep_size=8)) == 0


def test_nvfp4_config_and_encoder_checks():
    L = lmoe.lib()
    ok = lmoe.make_config(synth.WORKLOADS["nemotron_decode_nvfp4"], 32)
    assert lmoe.lmoe_workspace_bytes(ok) > 0
    # NVFP4 experts stream in stages of 256 elements; no expert parallelism
    for b in (dict(latent=384), dict(m=640), dict(expert_fmt=4)):
        c = lmoe.make_config(synth.WORKLOADS["nemotron_decode_nvfp4"], 32)
        for k, v in b.items():
            setattr(c, k, v)
        assert lmoe.lmoe_workspace_bytes(c) == 0, b
    assert lmoe.lmoe_workspace_bytes(lmoe.make_config(synth.WORKLOADS["nemotron_decode_nvfp4"], 32, ep_size=2)) == 0
    # a layer without its tensor scales is rejected before any device work
    cfg = lmoe.make_config(synth.WORKLOADS["nemotron_decode_nvfp4"], 32)
    big = lmoe.lmoe_workspace_bytes(cfg)
    h = ctypes.c_void_p()
    w = lmoe.lmoe_weights(w_router=0x10000, w_down=0x10000, w_up=0x10000, w1=0x10000, w2=0x10000,
                          w1_scales=0x20000, w2_scales=0x20000)
    assert L.lmoe_create(ctypes.byref(cfg), ctypes.byref(w), 0x100000, big, ctypes.byref(h)) == -1
    assert h.value is None
    # the encoder checks sizes before pointers
    assert L.lmoe_nvfp4_encode_weights(0x100, 1, 100, 128, 0x100, 0x100, 0x100, None) == -2
    assert L.lmoe_nvfp4_encode_weights(0x100, 1, 128, 96, 0x100, 0x100, 0x100, None) == -2
    assert L.lmoe_nvfp4_encode_weights(0x100, 0, 128, 128, 0x100, 0x100, 0x100, None) == -2
    assert L.lmoe_nvfp4_encode_weights(None, 1, 128, 128, 0x100, 0x100, 0x100, None) == -1


def test_missing_library_fails_loudly():
    """Without the built CUDA library the binding raises: there is no CPU or library fallback."""
    saved_path, saved_lib = lmoe.LIB_PATH, lmoe._lib
    try:
        lmoe.LIB_PATH = os.path.join(os.path.dirname(saved_path), "no_such_liblmoe.so")
        lmoe._lib = None
        with pytest.raises(RuntimeError, match="not built"):
            lmoe.lib()
    finally:
        lmoe.LIB_PATH, lmoe._lib = saved_path, saved_lib


def test_noalloc_binding_checks_its_buffers_before_any_call():
    """The binding rejects host tensors, wrong dtypes, non-contiguous or short buffers with ValueError
    before it reaches the library (a short perm or inv would let the scatter write past its end)."""
    import torch

    idx = torch.zeros((4, 2), dtype=torch.int32)
    buf = torch.zeros(16, dtype=torch.int32)
    with pytest.raises(ValueError):
        lmoe.lmoe_dispatch_noalloc(idx, 8, buf, buf, buf, buf)       # host tensors
    with pytest.raises(ValueError):
        lmoe.lmoe_dispatch_noalloc(idx.reshape(-1), 8, buf, buf, buf, buf)  # idx not [T, top_k]
    meta = dict(dtype=torch.int32, device="meta")
    idm, ok = torch.empty((4, 2), **meta), torch.empty(16, **meta)
    # the device check runs first for anything that is not a CUDA tensor
    with pytest.raises(ValueError):
        lmoe.lmoe_dispatch_noalloc(idm, 8, ok, ok, ok, ok)
    e = lmoe._int32_buffer
    dev = torch.device("meta")
    with pytest.raises(ValueError):
        e("perm", torch.empty(7, **meta), dev, 8)                    # short
    with pytest.raises(ValueError):
        e("perm", torch.empty(8, dtype=torch.int64, device="meta"), dev, 8)  # dtype
    with pytest.raises(ValueError):
        e("perm", torch.empty((4, 4), **meta).t(), dev, 8)           # not contiguous
    e("perm", torch.empty(8, **meta), dev, 8)                         # accepted
