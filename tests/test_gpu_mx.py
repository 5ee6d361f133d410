"""Block-scaled (MX) expert weights on the GPU, through the C ABI, against the oracle.

* The weight encoder (lmoe_mx_encode_weights) against the oracle's encoder.
  The comparison is bit for bit, both for the codes and for the scales once
  they are taken out of the tensor-core atom order.
* The layer with MXFP8 and MXFP4 experts against the oracle's MX layer.  The
  oracle encodes the weights itself: no code or scale crosses from the GPU.
  The contract tolerances apply.  Every case is a decode batch (T <= 32, the
  regime block-scaled experts serve) or a larger batch whose experts stream
  in several 32-row entries; every case covers several K stages and a ragged
  tail of token-scale blocks.
"""
import numpy as np
import pytest
import torch

import oracle
from latent_mixture_experts_gemm_b200 import lmoe, synth
from tests.test_gpu_layer import _run_and_check

pytestmark = pytest.mark.gpu

MX_BASE = synth.LayerConfig(name="mx_base", tokens=29, d=256, latent=128, m=256, n_ffn=16, top_k=4, seed=51)

CASES = {
    "mxfp8_relu2": MX_BASE.with_(expert_fmt=1),
    "mxfp4_relu2": MX_BASE.with_(expert_fmt=2, seed=52),
    "mxfp8_swiglu_bypass_skew": MX_BASE.with_(expert_fmt=1, act="swiglu", n_zero=1, n_copy=1, n_const=1, zipf=1.1,
                                              tokens=32, seed=53),
    "mxfp4_swiglu_bypass_skew": MX_BASE.with_(expert_fmt=2, act="swiglu", n_zero=1, n_copy=1, n_const=1, zipf=1.1,
                                              tokens=32, seed=54),
    "mxfp8_identity": MX_BASE.with_(expert_fmt=1, act="identity", seed=55),
    "mxfp8_standard_moe": MX_BASE.with_(expert_fmt=1, has_proj=0, latent=256, seed=56),
    "mxfp4_one_token": MX_BASE.with_(expert_fmt=2, tokens=1, seed=57),
    # K = 640 / 384: five and three stages, the second token-scale chunk only partly filled
    "mxfp8_ragged_scale_chunks": MX_BASE.with_(expert_fmt=1, d=512, latent=640, m=384, n_ffn=24, top_k=6,
                                               tokens=31, seed=58),
    "mxfp4_ragged_scale_chunks_swiglu": MX_BASE.with_(expert_fmt=2, d=512, latent=640, m=384, n_ffn=24, top_k=6,
                                                      act="swiglu", tokens=23, seed=59),
    "mxfp8_shared_latent_router": MX_BASE.with_(expert_fmt=1, shared_m=128, latent_router=1, seed=60),
    # more than 32 rows per expert: each expert streams in several 32-row entries (up to 5 with the skew)
    "mxfp8_150_tokens": MX_BASE.with_(expert_fmt=1, tokens=150, seed=62),
    "mxfp4_300_tokens_swiglu_skew": MX_BASE.with_(expert_fmt=2, act="swiglu", zipf=1.1, n_zero=1, tokens=300,
                                                  seed=63),
    "nemotron_decode_mxfp8": synth.WORKLOADS["nemotron_decode_mxfp8"],
    "nemotron_decode_mxfp4": synth.WORKLOADS["nemotron_decode_mxfp4"],
}


@pytest.mark.parametrize("name", list(CASES))
def test_mx_layer_parity(name):
    cfg = CASES[name]
    _run_and_check(cfg, synth.make_layer(cfg), label=name)


def _detile_scales(s: np.ndarray, rows: int, K: int) -> np.ndarray:
    """[rows/128][K/128][32][16] atoms -> [rows, K/32]: byte (r, c) of atom (R, G) is row 128R + 32(c/4) + r,
    block 4G + c%4."""
    a = s.reshape(rows // 128, K // 128, 32, 4, 4)          # (R, G, r, c//4, c%4)
    return a.transpose(0, 3, 2, 1, 4).reshape(rows, K // 32)  # (R, c//4, r, G, c%4)


@pytest.mark.parametrize("fmt", [oracle.FMT_MXFP8, oracle.FMT_MXFP4])
def test_weight_encoder_matches_the_oracle_bit_for_bit(fmt):
    rows, K = 384, 640
    g = torch.Generator().manual_seed(70 + fmt)
    mag = torch.pow(2.0, torch.randint(-40, 40, (rows, 1), generator=g).float())
    w = (torch.randn(rows, K, generator=g) * mag)
    w[5, 64:96] = 0.0                                # an all-zero block
    w[6, :32] = torch.linspace(-1e-30, 1e-30, 32)    # tiny values (bf16 subnormals and zero)
    w[7, 32:64] = 480.0                              # a block that saturates after scaling
    w[7, 40] = -1.9 * 256
    w = w.to(torch.bfloat16)
    codes, scales = lmoe.lmoe_mx_encode_weights(w.cuda(), fmt)
    torch.cuda.synchronize()
    c = codes.cpu().numpy()
    if fmt == oracle.FMT_MXFP4:
        c = np.stack([c & 15, c >> 4], axis=-1).reshape(rows, K)
    ref_c, ref_s = oracle.mx_quantize(w, fmt)
    s = _detile_scales(scales.cpu().numpy(), rows, K)
    assert np.array_equal(s, ref_s), f"{np.count_nonzero(s != ref_s)} scale bytes differ"
    assert np.array_equal(c, ref_c), f"{np.count_nonzero(c != ref_c)} codes differ"


def test_weight_encoder_rejects_bad_shapes():
    w = torch.zeros((100, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lmoe.LmoeError) as e:
        lmoe.lmoe_mx_encode_weights(w, lmoe.LMOE_FMT_MXFP8)
    assert e.value.status == -2
    w = torch.zeros((128, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lmoe.LmoeError) as e:
        lmoe.lmoe_mx_encode_weights(w, lmoe.LMOE_FMT_MXFP4)
    assert e.value.status == -2


def test_mx_deterministic_and_host_entry_point():
    cfg = CASES["mxfp4_swiglu_bypass_skew"]
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
