"""NVFP4 expert weights on the GPU, through the C ABI, against the oracle.

* The weight encoder (lmoe_nvfp4_encode_weights) against the oracle's encoder,
  bit for bit: the tensor scales (fp32), the codes, and the block scales once
  they are taken out of the tensor-core atom order.
* The layer with NVFP4 experts against the oracle's NVFP4 layer.  The oracle
  encodes the weights itself: no code or scale crosses from the GPU.  The
  contract tolerances apply.  Most cases are decode batches (T <= 32, the
  regime block-scaled experts serve); two are larger, so that experts stream
  in several 32-row entries.  The cases span one to three K stages of 256
  elements.
"""
import numpy as np
import pytest
import torch

import oracle
from latent_mixture_experts_gemm_b200 import lmoe, synth
from tests.test_gpu_layer import _run_and_check

pytestmark = pytest.mark.gpu

NV_BASE = synth.LayerConfig(name="nv_base", tokens=29, d=512, latent=256, m=256, n_ffn=16, top_k=4, seed=61,
                            expert_fmt=3)

CASES = {
    "nvfp4_relu2": NV_BASE,
    "nvfp4_swiglu_bypass_skew": NV_BASE.with_(act="swiglu", n_zero=1, n_copy=1, n_const=1, zipf=1.1, tokens=32,
                                              seed=62),
    "nvfp4_identity": NV_BASE.with_(act="identity", seed=63),
    "nvfp4_standard_moe": NV_BASE.with_(has_proj=0, latent=512, seed=64),
    "nvfp4_one_token": NV_BASE.with_(tokens=1, seed=65),
    # K = 768 for the up GEMM (three stages), 512 for the down GEMM (two)
    "nvfp4_three_stages": NV_BASE.with_(latent=768, m=512, n_ffn=24, top_k=6, tokens=31, seed=66),
    "nvfp4_shared_latent_router": NV_BASE.with_(shared_m=128, latent_router=1, seed=67),
    # more than 32 rows per expert: several 32-row entries per expert
    "nvfp4_200_tokens": NV_BASE.with_(tokens=200, seed=68),
    "nvfp4_260_tokens_swiglu_skew": NV_BASE.with_(act="swiglu", zipf=1.1, n_copy=1, tokens=260, seed=69),
    "nemotron_decode_nvfp4": synth.WORKLOADS["nemotron_decode_nvfp4"],
}


@pytest.mark.parametrize("name", list(CASES))
def test_nvfp4_layer_parity(name):
    cfg = CASES[name]
    _run_and_check(cfg, synth.make_layer(cfg), label=name)


def _detile_scales(s: np.ndarray, rows: int, K: int) -> np.ndarray:
    """[rows/128][K/64][32][16] atoms -> [rows, K/16]: byte (r, c) of atom (R, G) is row 128R + 32(c/4) + r,
    block 4G + c%4."""
    a = s.reshape(rows // 128, K // 64, 32, 4, 4)           # (R, G, r, c//4, c%4)
    return a.transpose(0, 3, 2, 1, 4).reshape(rows, K // 16)  # (R, c//4, r, G, c%4)


def test_nvfp4_encoder_matches_the_oracle_bit_for_bit():
    n_mats, rows, K = 3, 256, 320
    g = torch.Generator().manual_seed(71)
    mag = torch.pow(2.0, torch.randint(-12, 12, (n_mats, rows, 1), generator=g).float())
    w = torch.randn(n_mats, rows, K, generator=g) * mag
    w[0, 5, 64:80] = 0.0                                  # an all-zero block
    w[1, 6, :16] = torch.linspace(-1e-30, 1e-30, 16)      # tiny values: the block scale rounds to zero
    w[2] = 0.0                                            # an all-zero matrix: tensor scale 1
    w = w.to(torch.bfloat16)
    codes, scales, gs = lmoe.lmoe_nvfp4_encode_weights(w.cuda())
    torch.cuda.synchronize()
    c = codes.cpu().numpy()
    c = np.stack([c & 15, c >> 4], axis=-1).reshape(n_mats * rows, K)
    s = _detile_scales(scales.cpu().numpy(), n_mats * rows, K)
    gs = gs.cpu().numpy()
    for i in range(n_mats):
        g_ref = oracle.nv_tensor_scale(w[i])
        assert gs[i] == np.float32(g_ref), (i, gs[i], g_ref)
        ref_c, ref_s = oracle.nv_quantize(w[i], g_ref)
        sl = slice(i * rows, (i + 1) * rows)
        assert np.array_equal(s[sl], ref_s), f"matrix {i}: {np.count_nonzero(s[sl] != ref_s)} scale bytes differ"
        assert np.array_equal(c[sl], ref_c), f"matrix {i}: {np.count_nonzero(c[sl] != ref_c)} codes differ"
    assert gs[2] == 1.0


def test_nvfp4_encoder_rejects_bad_shapes():
    w = torch.zeros((2, 100, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lmoe.LmoeError) as e:
        lmoe.lmoe_nvfp4_encode_weights(w)
    assert e.value.status == -2
    w = torch.zeros((1, 128, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lmoe.LmoeError) as e:
        lmoe.lmoe_nvfp4_encode_weights(w)
    assert e.value.status == -2


def test_nvfp4_deterministic_and_host_entry_point():
    cfg = CASES["nvfp4_swiglu_bypass_skew"]
    layer = synth.make_layer(cfg)
    mod = lmoe.LatentMoE(cfg, layer, max_tokens=cfg.tokens)
    try:
        x = layer["x"].cuda()
        y1 = mod.forward(x)
        y2 = mod.forward(x)
        xh = layer["x"].pin_memory()
        yh = torch.empty_like(xh).pin_memory()
        mod.forward_host(xh, yh)
        torch.cuda.synchronize()
        assert torch.equal(y1, y2) and torch.equal(y1.cpu(), yh)
        assert mod.last_error() == 0
    finally:
        mod.close()
