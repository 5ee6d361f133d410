"""Comparison of the CUDA path against the fp64 oracle (test helper).

Tolerances (fixed for the layer's output):
  * max |y_gpu - y_ref|                 <= 2e-2 * RMS(y_ref)
  * sum |y_gpu - y_ref| / sum |y_ref|   <= 5e-3   (mean relative error, L1 form)
  * top-K' index sets identical, except tokens whose gap between the K'-th and
    (K'+1)-th oracle logit is below 1e-4 * max|logit| (either set accepted if it
    is a valid top-K' set within that margin; such tokens are compared with the
    oracle re-run on the GPU's ids).
  * the dispatch (counts, offsets, perm) bit-exact against the oracle's counting
    sort of the GPU's own ids.

The CUDA path stores z, the expert hidden rows H, the expert outputs O, the
combined latent yl and y in bf16 (H, yl and z feed bf16 tensor-core GEMMs).  On
a few degenerate shapes (top-1 routing, where nothing averages the expert
output, or outputs of a few times RMS(y_ref), where one bf16 rounding of y is
already worth most of the bound) those roundings alone exceed the max-error
bound.  ``emulate_bf16`` evaluates the layer with exactly those storage
roundings (fp64 otherwise), and with block-scaled experts with the oracle's
encodings of their weights and inputs on top; a max-error miss is accepted only
when that emulation alone reaches at least 75% of the bound, the GPU stays
within 1.5x of the emulation's error, and the mean relative error still meets
5e-3.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

MAX_ERR_VS_RMS = 2e-2
MEAN_REL_ERR = 5e-3
NEAR_TIE = 1e-4


def metrics(got: np.ndarray, ref: np.ndarray) -> dict:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    diff = np.abs(got - ref)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    return {"max_err": float(diff.max()) if diff.size else 0.0, "rms_ref": rms,
            "mean_rel": float(diff.sum() / max(np.abs(ref).sum(), 1e-300)),
            "rel_l2": float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))}


def assert_close(got, ref, what="y", max_vs_rms=MAX_ERR_VS_RMS, mean_rel=MEAN_REL_ERR) -> dict:
    m = metrics(got, ref)
    assert m["max_err"] <= max_vs_rms * m["rms_ref"] + 1e-30, f"{what}: {m}"
    assert m["mean_rel"] <= mean_rel, f"{what}: {m}"
    return m


def _bf(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(a, np.float64)).to(torch.float32).to(torch.bfloat16).double().numpy()


def _expert_weights(cfg, layer):
    """Each expert's W1_e, W2_e at the values the layer computes with: as stored (bf16), or the oracle's
    block-scaled encoding of them decoded (MXFP8 / MXFP4 per matrix row blocks, NVFP4 per expert matrix)."""
    fmt = getattr(cfg, "expert_fmt", 0)
    W1, W2 = layer["w1"], layer["w2"]
    if fmt == 0:
        return [w.double().numpy() for w in W1], [w.double().numpy() for w in W2]
    out = []
    for W in (W1, W2):
        mats = []
        for e in range(W.shape[0]):
            if fmt == oracle.FMT_NVFP4:
                g = oracle.nv_tensor_scale(W[e])
                c, sc = oracle.nv_quantize(W[e], g)
                mats.append(oracle.nv_dequantize(c, sc, g))
            else:
                c, sc = oracle.mx_quantize(W[e], fmt)
                mats.append(oracle.mx_dequantize(c, sc, fmt))
        out.append(mats)
    return out[0], out[1]


def _expert_input(cfg, v: np.ndarray) -> np.ndarray:
    """An expert GEMM's input as the layer feeds it: bf16, then (block-scaled experts) its encoding decoded:
    MXFP8 for the MX formats, NVFP4 with tensor scale 1 for NVFP4."""
    fmt = getattr(cfg, "expert_fmt", 0)
    b = _bf(v)
    if fmt == 0:
        return b
    t = torch.from_numpy(b.reshape(1, -1)).to(torch.bfloat16)
    if fmt == oracle.FMT_NVFP4:
        c, sc = oracle.nv_quantize(t, 1.0)
        return oracle.nv_dequantize(c, sc, 1.0).reshape(-1)
    c, sc = oracle.mx_quantize(t, oracle.FMT_MXFP8)
    return oracle.mx_dequantize(c, sc, oracle.FMT_MXFP8).reshape(-1)


def emulate_bf16(cfg, layer, x: torch.Tensor, idx: np.ndarray, w: np.ndarray) -> np.ndarray:
    """y with the GPU path's bf16 storage points (z, H, O, yl, the shared expert's hidden rows and
    x + its output, y) on the given routes.  With block-scaled experts the expert weights and inputs take
    the oracle's encodings (the layer's definition) on top of those storage points."""
    f = lambda t: None if t is None else t.double().numpy()  # noqa: E731
    X = f(x)
    W1, W2 = _expert_weights(cfg, layer)
    z = _bf(X @ f(layer["w_down"]).T) if cfg.has_proj else X
    m = cfg.m
    yl = np.zeros_like(z)
    for t in range(X.shape[0]):
        acc = np.zeros(z.shape[1])
        zin = None
        for k in range(cfg.top_k):
            e = int(idx[t, k])
            if e < cfg.n_ffn:
                if zin is None:
                    zin = _expert_input(cfg, z[t])
                u = W1[e] @ zin
                if cfg.act == 0:
                    h = np.maximum(u, 0) ** 2
                elif cfg.act == 1:
                    h = u[:m] / (1 + np.exp(-u[:m])) * u[m:]
                else:
                    h = u
                o = _bf(W2[e] @ _expert_input(cfg, h))
            elif e < cfg.n_ffn + cfg.n_zero:
                o = np.zeros_like(z[t])
            elif e < cfg.n_ffn + cfg.n_zero + cfg.n_copy:
                o = z[t]
            else:
                o = f(layer["const_vecs"])[e - cfg.n_ffn - cfg.n_zero - cfg.n_copy]
            acc += float(np.float32(w[t, k])) * o
        yl[t] = acc
    base = X
    if getattr(cfg, "shared_m", 0):
        us = X @ f(layer["w_shared1"]).T
        ms = cfg.shared_m
        if cfg.act == 0:
            hs = np.maximum(us, 0) ** 2
        elif cfg.act == 1:
            hs = us[:, :ms] / (1 + np.exp(-us[:, :ms])) * us[:, ms:]
        else:
            hs = us
        base = _bf(X + _bf(hs) @ f(layer["w_shared2"]).T)   # x + shared expert, stored in bf16
    if cfg.has_proj:
        return _bf(base + _bf(yl) @ f(layer["w_up"]).T)
    return _bf(base + yl)


def assert_layer_close(got, ref, emulated, what="y") -> dict:
    """The contract bound against the fp64 oracle, with the bf16-storage allowance described above."""
    m = metrics(got, ref)
    assert m["mean_rel"] <= MEAN_REL_ERR, f"{what}: {m}"
    if m["max_err"] <= MAX_ERR_VS_RMS * m["rms_ref"]:
        return m
    assert emulated is not None, f"{what}: {m} (no bf16-storage emulation for this case)"
    me = metrics(emulated, ref)
    assert me["max_err"] >= 0.75 * MAX_ERR_VS_RMS * me["rms_ref"], f"{what}: {m} (bf16 storage alone: {me})"
    assert m["max_err"] <= 1.5 * me["max_err"], f"{what}: {m} (bf16 storage alone: {me})"
    m["bf16_storage_max_err"] = me["max_err"]
    return m


def near_tie_tokens(logits: np.ndarray, K: int) -> np.ndarray:
    """Tokens whose K'-th / (K'+1)-th largest logits are within the near-tie margin."""
    T, N = logits.shape
    if K >= N:
        return np.zeros(T, bool)
    s = -np.sort(-logits, axis=1)
    gap = s[:, K - 1] - s[:, K]
    return gap < NEAR_TIE * np.abs(logits).max(axis=1)


def check_routing(gpu_idx: np.ndarray, gpu_w: np.ndarray, ref: dict, K: int, w_atol: float = 2e-5) -> np.ndarray:
    """Index sets exact except near-ties (which must still be valid); weights close.

    Returns the mask of tokens whose GPU set differs from the oracle's."""
    lg = ref["logits"]
    tie = near_tie_tokens(lg, K)
    same = np.array([set(a) == set(b) for a, b in zip(gpu_idx.tolist(), ref["idx"].tolist())], bool)
    bad = ~same & ~tie
    assert not bad.any(), f"top-K' sets differ on non-tie tokens {np.nonzero(bad)[0][:10]}"
    margin = NEAR_TIE * np.abs(lg).max(axis=1)
    for t in np.nonzero(~same)[0]:
        sel = lg[t, gpu_idx[t]]
        rest = np.delete(lg[t], gpu_idx[t])
        assert sel.min() >= rest.max() - margin[t], f"token {t}: GPU set is not a top-K' set"
    # weights: same order where the sets agree (order by logit; allow swapped near-equal neighbours)
    for t in np.nonzero(same)[0]:
        order = {e: i for i, e in enumerate(ref["idx"][t])}
        w_ref = np.array([ref["w"][t][order[e]] for e in gpu_idx[t]])
        np.testing.assert_allclose(gpu_w[t], w_ref, atol=w_atol, rtol=1e-4)
    return ~same


def check_dispatch(gpu_idx, counts, offsets, perm, n_total):
    c, o, p, _ = oracle.dispatch(gpu_idx, n_total)
    assert np.array_equal(counts, c), "counts differ"
    assert np.array_equal(offsets, o), "offsets differ"
    assert np.array_equal(perm, p), "perm differs"


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy() if t.is_floating_point() else t.detach().cpu().numpy()
