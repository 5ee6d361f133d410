"""Pins for the oracle's MX block formats (block-scaled expert weights).

The encodings are pinned to routines that share nothing with the oracle's C
code:

* E4M3 elements: torch's float8_e4m3fn conversion (round to nearest even).
  That conversion turns values past the format's range into NaN where MX
  saturates, so the reference clamps to +-448 first.
* E2M1 elements: a hand table of the eight magnitudes and of the midpoints
  between them (ties go to the even mantissa).
* Block scales: numpy's frexp.  The closed form is
  s = floor(log2 amax) - emax.

The whole layer with MX experts is then checked against a dense brute force
that uses those independent encoders.
"""
import numpy as np
import pytest
import scipy.special
import torch

import oracle
from latent_mixture_experts_gemm_b200 import synth

E2M1_MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _bf(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _scale_exp(blocks, emax):
    """s = floor(log2 amax) - emax per block (numpy frexp), -127 for all-zero blocks."""
    amax = np.abs(blocks).max(axis=-1)
    _, e = np.frexp(amax)
    s = np.where(amax > 0, e - 1 - emax, -127)
    return np.clip(s, -127, 127)


def _e4m3_ref(q):
    """Nearest E4M3 value (ties to even), saturated: torch's float8 cast after a clamp."""
    return torch.from_numpy(np.clip(q, -448.0, 448.0)).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def _e2m1_ref(q):
    """Nearest E2M1 value by search over the eight magnitudes; ties go to the even code."""
    a = np.minimum(np.abs(q), 6.0)
    dist = np.abs(a[..., None] - E2M1_MAGS)
    best = dist.min(axis=-1, keepdims=True)
    cand = np.isclose(dist, best, rtol=0, atol=0)
    codes = np.arange(8)
    # among equally near magnitudes prefer the even code (mantissa bit 0)
    pick = np.where(cand & (codes % 2 == 0), codes, 99).min(axis=-1)
    pick = np.where(pick == 99, np.where(cand, codes, 99).min(axis=-1), pick)
    return np.sign(q) * E2M1_MAGS[pick]


def _mx_ref(v, fmt):
    """Independent MX encode-then-decode of v [..., K] along its last axis (fp64 values)."""
    sh = v.shape
    blocks = v.reshape(*sh[:-1], sh[-1] // 32, 32)
    emax = 8 if fmt == oracle.FMT_MXFP8 else 2
    s = _scale_exp(blocks, emax)
    X = np.ldexp(1.0, s)[..., None]
    q = blocks / X
    el = _e4m3_ref(q) if fmt == oracle.FMT_MXFP8 else _e2m1_ref(q)
    return (el * X).reshape(sh)


def _bf16(v):
    return torch.from_numpy(np.asarray(v, np.float64)).to(torch.float32).to(torch.bfloat16).double().numpy()


def _wide_range_matrix(rows, K, seed):
    g = torch.Generator().manual_seed(seed)
    mag = torch.pow(2.0, torch.randint(-30, 30, (rows, 1), generator=g).float())
    return (torch.randn(rows, K, generator=g) * mag).to(torch.bfloat16)


# --------------------------------------------------------------------------------------------
# element encodings and scales
# --------------------------------------------------------------------------------------------


def test_mxfp8_elements_match_torch_float8_e4m3fn():
    w = _wide_range_matrix(64, 256, seed=1)
    codes, scales = oracle.mx_quantize(w, oracle.FMT_MXFP8)
    v = w.double().numpy().reshape(64, 8, 32)
    s = _scale_exp(v, 8)
    assert np.array_equal(scales.astype(int) - 127, s)
    q = v / np.ldexp(1.0, s)[..., None]
    ref_codes = torch.from_numpy(np.clip(q, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes.reshape(64, 8, 32), ref_codes)
    deq = oracle.mx_dequantize(codes, scales, oracle.FMT_MXFP8)
    np.testing.assert_array_equal(deq, _mx_ref(w.double().numpy(), oracle.FMT_MXFP8))


def test_mxfp8_ties_round_to_even_and_subnormals():
    # one block with amax 256 (scale 2^0): the elements are the scaled values themselves
    vals = [256.0,
            17.0, 19.0, 21.0,          # 16 + 1 (tie between 16 and 18 -> 16), 19 -> 20 (tie -> even m), 21 -> 20
            0.0048828125,              # 2.5 subnormal quanta of 2^-9: a tie -> 2 quanta (even)
            2.0 ** -10, 3 * 2.0 ** -10,  # half a quantum -> 0 (even), 1.5 quanta -> 2 quanta
            -2.0 ** -11]               # rounds to -0
    vals += [1.0] * (32 - len(vals))
    w = _bf([vals])
    codes, scales = oracle.mx_quantize(w, oracle.FMT_MXFP8)
    assert scales[0, 0] == 127
    deq = oracle.mx_dequantize(codes, scales, oracle.FMT_MXFP8)[0]
    assert deq[0] == 256.0
    assert list(deq[1:4]) == [16.0, 20.0, 20.0]
    assert deq[4] == 2 * 2.0 ** -9                 # 0.0048828125 = 2.5 * 2^-9 -> 2 quanta
    assert deq[5] == 0.0 and deq[6] == 2 * 2.0 ** -9
    assert deq[7] == 0.0 and codes[0, 7] == 0x80   # the sign survives rounding to zero
    assert codes[0, 0] == 0x78                     # 256 = 2^8: exponent field 15, mantissa 0


def test_mxfp8_saturates_past_448():
    # amax 1.9 * 2^5 -> s = 5 - 8 = -3 -> scaled amax 486.4 > 448 -> the largest code 0x7E (and 0xFE)
    vals = [1.9 * 32, -1.9 * 32, 1.75 * 32] + [0.5] * 29
    codes, scales = oracle.mx_quantize(_bf([vals]), oracle.FMT_MXFP8)
    assert scales[0, 0] == 127 - 3
    assert codes[0, 0] == 0x7E and codes[0, 1] == 0xFE and codes[0, 2] == 0x7E


def test_mxfp4_midpoints_round_to_even():
    # amax 4 -> s = 2 - 2 = 0: the elements are the values themselves
    table = [(4.0, 4.0), (0.25, 0.0), (0.3, 0.5), (0.75, 1.0), (1.25, 1.0), (1.75, 2.0), (2.5, 2.0),
             (3.5, 4.0), (-0.75, -1.0), (0.5, 0.5), (1.5, 1.5), (3.0, 3.0), (-2.5, -2.0), (0.74, 0.5)]
    vals = [a for a, _ in table] + [0.0] * (32 - len(table))
    w = _bf([vals])
    codes, scales = oracle.mx_quantize(w, oracle.FMT_MXFP4)
    assert scales[0, 0] == 127
    deq = oracle.mx_dequantize(codes, scales, oracle.FMT_MXFP4)[0]
    expect = np.array([b for _, b in table])
    # the inputs were stored in bf16 first: 0.3 and 0.74 are not exact there, the others are
    np.testing.assert_array_equal(deq[:len(table)], expect)
    assert codes[0, 0] == 0b0110 and codes[0, 8] == 0b1010  # 4 = 1.0 * 2^2; -1 = sign | exp 1


def test_mxfp4_saturates_and_matches_the_table_encoder():
    vals = [7.0, -6.5, 5.0, 5.5] + [1.0] * 28  # amax 7 -> s = 0; 7 and -6.5 saturate to +-6; 5 -> 4; 5.5 -> 6
    codes, scales = oracle.mx_quantize(_bf([vals]), oracle.FMT_MXFP4)
    deq = oracle.mx_dequantize(codes, scales, oracle.FMT_MXFP4)[0]
    assert list(deq[:4]) == [6.0, -6.0, 4.0, 6.0]
    w = _wide_range_matrix(32, 128, seed=2)
    codes, scales = oracle.mx_quantize(w, oracle.FMT_MXFP4)
    np.testing.assert_array_equal(oracle.mx_dequantize(codes, scales, oracle.FMT_MXFP4),
                                  _mx_ref(w.double().numpy(), oracle.FMT_MXFP4))


@pytest.mark.parametrize("fmt", [oracle.FMT_MXFP8, oracle.FMT_MXFP4])
def test_encoding_is_idempotent_and_zero_blocks_get_the_smallest_scale(fmt):
    w = _wide_range_matrix(16, 128, seed=3)
    w[3, 32:64] = 0.0
    codes, scales = oracle.mx_quantize(w, fmt)
    assert scales[3, 1] == 0 and not codes[3, 32:64].any()
    deq = oracle.mx_dequantize(codes, scales, fmt)
    codes2, scales2 = oracle.mx_quantize(_bf(deq), fmt)  # decoded values are exact in bf16
    assert np.array_equal(scales, scales2) and np.array_equal(codes, codes2)


@pytest.mark.parametrize("fmt", [oracle.FMT_MXFP8, oracle.FMT_MXFP4])
def test_relative_error_within_the_format_bound(fmt):
    # With amax in [2^E, 2^(E+1)) the top binade's quantum is q = 2^(E - mantissa bits).  Rounding costs at
    # most q/2.  Saturation costs less than 2^(E+1) - max: 2q for E4M3 (512 vs 448 scaled), q for E2M1 (8 vs 6).
    w = _wide_range_matrix(32, 256, seed=4)
    codes, scales = oracle.mx_quantize(w, fmt)
    v = w.double().numpy()
    deq = oracle.mx_dequantize(codes, scales, fmt)
    blocks = np.abs(v).reshape(32, 8, 32).max(-1)
    _, e = np.frexp(blocks)
    q_top = np.ldexp(1.0, e - 1 - (3 if fmt == oracle.FMT_MXFP8 else 1))
    err = np.abs(deq - v).reshape(32, 8, 32).max(-1)
    bound = (2.0 if fmt == oracle.FMT_MXFP8 else 1.0) * q_top
    assert np.all(err <= bound)
    # and every element that did not saturate is within half a quantum of its own binade (or of the subnormals)
    el = np.abs(v).reshape(32, 8, 32)
    X = np.ldexp(1.0, scales.astype(int) - 127)[..., None]
    a = el / X
    top = 448.0 if fmt == oracle.FMT_MXFP8 else 6.0
    _, ea = np.frexp(np.maximum(a, 1e-300))
    emin = -6 if fmt == oracle.FMT_MXFP8 else 0
    mb = 3 if fmt == oracle.FMT_MXFP8 else 1
    q_el = np.ldexp(1.0, np.maximum(ea - 1, emin) - mb) * X
    ok = a < top
    assert np.all(np.abs(deq - v).reshape(32, 8, 32)[ok] <= 0.5 * q_el[ok])


# --------------------------------------------------------------------------------------------
# whole layer with MX experts: dense brute force with the independent encoders
# --------------------------------------------------------------------------------------------

MX_SMALL = synth.LayerConfig(d=64, latent=64, m=96, n_ffn=6, n_zero=1, n_copy=1, n_const=1, top_k=3, tokens=12,
                             seed=9)


def _np(t):
    return None if t is None else t.to(torch.float64).numpy()


def _mx_dense_bruteforce(cfg, layer, fmt):
    x, Wr, Wd, Wu = _np(layer["x"]), _np(layer["w_router"]), _np(layer["w_down"]), _np(layer["w_up"])
    m = cfg.m
    W1 = _mx_ref(_np(layer["w1"]), fmt)
    W2 = _mx_ref(_np(layer["w2"]), fmt)
    z = x @ Wd.T if cfg.has_proj else x.copy()
    lg = x @ Wr.T
    if layer.get("bias") is not None:
        lg = lg + layer["bias"].double().numpy()
    zq = _mx_ref(_bf16(z), oracle.FMT_MXFP8)
    U = np.einsum("eol,tl->teo", W1, zq)
    if cfg.act == synth.ACT_RELU2:
        Hh = np.maximum(U, 0) ** 2
    else:
        Hh = scipy.special.expit(U[..., :m]) * U[..., :m] * U[..., m:]
    Hq = _mx_ref(_bf16(Hh), oracle.FMT_MXFP8)
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


@pytest.mark.parametrize("fmt,act", [(oracle.FMT_MXFP8, "relu2"), (oracle.FMT_MXFP4, "relu2"),
                                     (oracle.FMT_MXFP8, "swiglu"), (oracle.FMT_MXFP4, "swiglu")])
def test_mx_layer_matches_dense_bruteforce(fmt, act):
    cfg = MX_SMALL.with_(act=act, expert_fmt=fmt)
    layer = synth.make_layer(cfg)
    out = oracle.forward(cfg, layer)
    np.testing.assert_allclose(out["y"], _mx_dense_bruteforce(cfg, layer, fmt), rtol=1e-11, atol=1e-11)


def test_mx_standard_moe_quantizes_x_itself():
    cfg = MX_SMALL.with_(has_proj=0, latent=64, expert_fmt=oracle.FMT_MXFP8, seed=10)
    layer = synth.make_layer(cfg)
    out = oracle.forward(cfg, layer)
    np.testing.assert_allclose(out["y"], _mx_dense_bruteforce(cfg, layer, oracle.FMT_MXFP8), rtol=1e-11, atol=1e-11)


def test_mx_layer_differs_from_bf16_layer_by_the_encoding_only():
    """Experts whose weights are already exact in MXFP8 leave only the activation encodings as a difference."""
    cfg = MX_SMALL.with_(expert_fmt=oracle.FMT_MXFP8, seed=11)
    layer = synth.make_layer(cfg)
    for k in ("w1", "w2"):
        c, s = oracle.mx_quantize(layer[k], oracle.FMT_MXFP8)
        layer[k] = _bf(oracle.mx_dequantize(c, s, oracle.FMT_MXFP8)).reshape(layer[k].shape)
    mx = oracle.forward(cfg, layer)["y"]
    ref = _mx_dense_bruteforce(cfg, layer, oracle.FMT_MXFP8)
    np.testing.assert_allclose(mx, ref, rtol=1e-11, atol=1e-11)
    bf = oracle.forward(cfg.with_(expert_fmt=0), layer)["y"]
    # What is left is the MXFP8 rounding of z and h.  It is not zero, and it is small against the MoE output.
    # Each encoded element is off by at most 2^-4 of its own binade, so about 2^-5 in RMS.  One more such
    # rounding passes through each expert, so the RMS ratio should stay well under 2 * 2^-4.
    moe = bf - _np(layer["x"])
    ratio = np.linalg.norm(mx - bf) / np.linalg.norm(moe)
    assert 0 < ratio < 2 * 2.0 ** -4


def test_mx_rejects_widths_that_are_not_whole_blocks():
    cfg = MX_SMALL.with_(m=40, expert_fmt=oracle.FMT_MXFP8)
    with pytest.raises(ValueError):
        oracle.forward(cfg, synth.make_layer(cfg))
