"""Pins for the oracle's NVFP4 encoding (block-scaled expert weights, 16-value blocks).

The encoding is pinned to routines that share nothing with the oracle's C code:

* E4M3 block scales: torch's float8_e4m3fn cast (round to nearest even), after
  a clamp at 448 because the cast turns larger values into NaN.
* E2M1 elements: the hand table of the eight magnitudes (ties go to the even
  code), as in the MX pins.
* The fp32 steps of the definition (g * 6, amax / that, sb * g, v / that):
  numpy float32 arithmetic, which rounds every operation correctly.

The whole layer with NVFP4 experts is then checked against a dense brute force
that uses this independent encoder.
"""
import numpy as np
import pytest
import scipy.special
import torch

import oracle
from latent_mixture_experts_gemm_b200 import synth

E2M1_MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
F32 = np.float32


def _e4m3_ref(x):
    """Nearest E4M3 value (ties to even), saturated at 448."""
    return torch.from_numpy(np.clip(np.asarray(x, np.float64), -448.0, 448.0)).to(torch.float8_e4m3fn).to(
        torch.float64).numpy()


def _e2m1_ref(q):
    """Nearest E2M1 value by search over the eight magnitudes; ties go to the even code; saturated at 6."""
    a = np.minimum(np.abs(q), 6.0)
    dist = np.abs(a[..., None] - E2M1_MAGS)
    best = dist.min(axis=-1, keepdims=True)
    cand = dist == best
    codes = np.arange(8)
    pick = np.where(cand & (codes % 2 == 0), codes, 99).min(axis=-1)
    pick = np.where(pick == 99, np.where(cand, codes, 99).min(axis=-1), pick)
    return np.sign(q) * E2M1_MAGS[pick]


def _scale_ref(w):
    """fp32 tensor scale amax / (6 * 448), 1 for an all-zero tensor."""
    amax = F32(np.abs(np.asarray(w, np.float64)).max())
    return F32(1.0) if amax == 0 else amax / F32(2688.0)


def _nv_ref(v, g):
    """Independent NVFP4 encode-then-decode of v [..., K] along its last axis with tensor scale g (fp64 out),
    plus the block scales' values."""
    v = np.asarray(v, np.float64)
    sh = v.shape
    blocks = v.reshape(*sh[:-1], sh[-1] // 16, 16)
    g = F32(g)
    amax = np.abs(blocks).max(axis=-1).astype(F32)
    x = amax / (g * F32(6.0))
    sb = _e4m3_ref(x)
    sg = sb.astype(F32) * g
    with np.errstate(divide="ignore", invalid="ignore"):
        q = blocks.astype(F32) / sg[..., None]
    el = np.where(sb[..., None] == 0, 0.0, _e2m1_ref(np.nan_to_num(q.astype(np.float64))))
    return (el * sb[..., None] * np.float64(g)).reshape(sh), sb


def _bf(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _bf16(v):
    return torch.from_numpy(np.asarray(v, np.float64)).to(torch.float32).to(torch.bfloat16).double().numpy()


def _wide_range_matrix(rows, K, seed):
    g = torch.Generator().manual_seed(seed)
    mag = torch.pow(2.0, torch.randint(-20, 20, (rows, 1), generator=g).float())
    # a few rows far below the rest, so their blocks use small and subnormal E4M3 scales
    w = torch.randn(rows, K, generator=g) * mag
    return w.to(torch.bfloat16)


# --------------------------------------------------------------------------------------------
# tensor scale, block scales, elements
# --------------------------------------------------------------------------------------------


def test_tensor_scale_closed_form():
    w = _wide_range_matrix(16, 64, seed=1)
    assert oracle.nv_tensor_scale(w) == float(_scale_ref(w.double().numpy()))
    assert oracle.nv_tensor_scale(torch.zeros(8, 32, dtype=torch.bfloat16)) == 1.0


@pytest.mark.parametrize("seed", [2, 3])
def test_encoding_matches_the_independent_encoder(seed):
    w = _wide_range_matrix(48, 128, seed)
    g = oracle.nv_tensor_scale(w)
    codes, scales = oracle.nv_quantize(w, g)
    deq = oracle.nv_dequantize(codes, scales, g)
    ref, sb = _nv_ref(w.double().numpy(), g)
    np.testing.assert_array_equal(deq, ref)
    # the scale bytes are E4M3 codes of the reference scales: decode them independently through torch
    dec = torch.from_numpy(scales.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(dec, sb)
    assert np.all(scales < 0x80)  # positive scales: the sign bit is never set


def test_the_largest_block_gets_the_largest_scale():
    w = _wide_range_matrix(8, 64, seed=4)
    g = oracle.nv_tensor_scale(w)
    _, scales = oracle.nv_quantize(w, g)
    v = np.abs(w.double().numpy()).reshape(8, 4, 16).max(-1)
    r, b = np.unravel_index(np.argmax(v), v.shape)
    assert scales[r, b] == 0x7E  # 448


def test_scale_ties_round_to_even():
    # g = 1: the scale is E4M3(amax / 6).  amax 6.375 gives 1.0625, halfway between 1.0 (mantissa 000) and
    # 1.125 (001): it goes to 1.0.  amax 7.125 gives 1.1875, halfway between 1.125 (001) and 1.25 (010): 1.25.
    w = torch.zeros(2, 16)
    w[0, 0] = 6.375
    w[1, 3] = -7.125
    codes, scales = oracle.nv_quantize(w.to(torch.bfloat16), 1.0)
    assert scales[0, 0] == 0x38 and scales[1, 0] == 0x3A
    deq = oracle.nv_dequantize(codes, scales, 1.0)
    # 6.375 / 1.0 saturates at 6; -7.125 / 1.25 = -5.7 rounds to -6 and is worth -7.5
    assert deq[0, 0] == 6.0 and deq[1, 3] == -7.5


def test_zero_and_vanishing_blocks_encode_zeros():
    w = torch.zeros(2, 32)
    w[1, :16] = 2.0 ** -14          # amax / 6 < 2^-10: the scale rounds to zero
    w[1, 16] = 1.0
    codes, scales = oracle.nv_quantize(w.to(torch.bfloat16), 1.0)
    assert scales[0].tolist() == [0, 0] and scales[1, 0] == 0
    assert not codes[0].any() and not codes[1, :16].any()
    # the second block: scale E4M3(1/6) = 0.171875 (1/6 = 1.333 * 2^-3 rounds to 1.375 * 2^-3: exponent
    # field 4, mantissa 011, byte 0x23), and 1 / 0.171875 = 5.82 rounds to 6: the element is worth 6 * 0.171875
    assert scales[1, 1] == 0x23
    assert oracle.nv_dequantize(codes, scales, 1.0)[1, 16] == 6 * 0.171875


def test_error_within_the_format_bound():
    # Each element of a block is off by at most half an E2M1 step at the block's scale (0.25, 0.5 or 1 of
    # sb * g in the binades [0, 2), [2, 4), [4, 6)), unless it saturated.  It saturates only when the scale was
    # rounded down.  A normal E4M3 scale is rounded by at most 2^-4 of itself, so |v| / (sb g) <= 6 / (1 - 2^-4)
    # = 6.4, and the error is at most 0.4 of sb * g.  (Subnormal scales round more coarsely; the comparison
    # with the independent encoder above covers them exactly.)
    g_ = torch.Generator().manual_seed(5)
    w = (torch.randn(32, 256, generator=g_) * torch.pow(2.0, torch.randint(-3, 3, (32, 1), generator=g_).float()))
    w = w.to(torch.bfloat16)
    g = oracle.nv_tensor_scale(w)
    codes, scales = oracle.nv_quantize(w, g)
    assert np.all(scales >= 0x08)  # every block scale is a normal E4M3 value
    deq = oracle.nv_dequantize(codes, scales, g)
    v = w.double().numpy()
    unit = np.repeat(torch.from_numpy(scales.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy() * g, 16,
                     axis=1)
    a = np.abs(v) / unit
    half_step = np.where(a < 2, 0.25, np.where(a < 4, 0.5, 1.0)) * unit
    err = np.abs(deq - v)
    sat = a > 6
    assert np.all(err[~sat] <= half_step[~sat] * (1 + 1e-12))
    assert np.all(a <= 6.4 * (1 + 1e-12))
    assert np.all(err[sat] <= 0.4 * unit[sat] * (1 + 1e-12))


# --------------------------------------------------------------------------------------------
# whole layer with NVFP4 experts: dense brute force with the independent encoder
# --------------------------------------------------------------------------------------------

NV_SMALL = synth.LayerConfig(d=64, latent=64, m=96, n_ffn=6, n_zero=1, n_copy=1, n_const=1, top_k=3, tokens=12,
                             seed=19, expert_fmt=oracle.FMT_NVFP4)


def _np(t):
    return None if t is None else t.to(torch.float64).numpy()


def _nv_dense_bruteforce(cfg, layer):
    x, Wr, Wd, Wu = _np(layer["x"]), _np(layer["w_router"]), _np(layer["w_down"]), _np(layer["w_up"])
    m = cfg.m
    W1 = np.stack([_nv_ref(_np(w), _scale_ref(_np(w)))[0] for w in layer["w1"]])
    W2 = np.stack([_nv_ref(_np(w), _scale_ref(_np(w)))[0] for w in layer["w2"]])
    z = x @ Wd.T if cfg.has_proj else x.copy()
    lg = x @ Wr.T
    if layer.get("bias") is not None:
        lg = lg + layer["bias"].double().numpy()
    zq = _nv_ref(_bf16(z), 1.0)[0]
    U = np.einsum("eol,tl->teo", W1, zq)
    if cfg.act == synth.ACT_RELU2:
        Hh = np.maximum(U, 0) ** 2
    else:
        Hh = scipy.special.expit(U[..., :m]) * U[..., :m] * U[..., m:]
    Hq = _nv_ref(_bf16(Hh), 1.0)[0]
    O = np.einsum("elm,tem->tel", W2, Hq)
    extra = [np.zeros_like(z)] * cfg.n_zero + [z] * cfg.n_copy
    extra += [np.broadcast_to(_np(layer["const_vecs"])[c], z.shape) for c in range(cfg.n_const)]
    O = np.concatenate([O, np.stack(extra, axis=1)], axis=1)
    order = np.argsort(-lg, axis=1, kind="stable")[:, :cfg.top_k]
    P = scipy.special.softmax(lg, axis=1)
    yl = np.zeros_like(z)
    for t in range(x.shape[0]):
        w = P[t, order[t]] / P[t, order[t]].sum()
        yl[t] = (w[:, None] * O[t, order[t]]).sum(0)
    return x + (yl @ Wu.T if cfg.has_proj else yl)


@pytest.mark.parametrize("act", ["relu2", "swiglu"])
def test_nvfp4_layer_matches_dense_bruteforce(act):
    cfg = NV_SMALL.with_(act=act)
    layer = synth.make_layer(cfg)
    out = oracle.forward(cfg, layer)
    np.testing.assert_allclose(out["y"], _nv_dense_bruteforce(cfg, layer), rtol=1e-11, atol=1e-11)


def test_nvfp4_standard_moe():
    cfg = NV_SMALL.with_(has_proj=0, latent=64, seed=20)
    layer = synth.make_layer(cfg)
    np.testing.assert_allclose(oracle.forward(cfg, layer)["y"], _nv_dense_bruteforce(cfg, layer), rtol=1e-11,
                               atol=1e-11)


def test_nvfp4_layer_stays_near_the_bf16_layer():
    """The NVFP4 layer is the bf16 layer up to the encodings: its MoE output is off by a few E2M1 steps in
    RMS, well under the output itself, and not identical to it."""
    cfg = NV_SMALL.with_(seed=21)
    layer = synth.make_layer(cfg)
    nv = oracle.forward(cfg, layer)["y"]
    bf = oracle.forward(cfg.with_(expert_fmt=0), layer)["y"]
    moe = bf - _np(layer["x"])
    ratio = np.linalg.norm(nv - bf) / np.linalg.norm(moe)
    # three encodings (W, input, hidden) of relative RMS error about 2^-4 .. 2^-3 each
    assert 0 < ratio < 0.5


def test_nvfp4_rejects_widths_that_are_not_whole_blocks():
    cfg = NV_SMALL.with_(m=40)
    with pytest.raises(ValueError):
        oracle.forward(cfg, synth.make_layer(cfg))
