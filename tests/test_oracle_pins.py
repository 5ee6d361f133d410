"""Pins for the fp64 oracle: checks against facts that do not come from the oracle itself.

Each test pins the oracle to something independent of its code: a hand-worked
closed form, brute force over all K'-subsets, a dense evaluation of every expert
with a full softmax, a library routine the special case reduces to, or an exact
invariant of the layer's definition.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from latent_mixture_experts_gemm_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_layer.json")


def _bf(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _layer_from_json(spec):
    c = spec["config"]
    cfg = synth.LayerConfig(d=c["d"], latent=c["latent"], m=c["m"], n_ffn=c["n_ffn"], top_k=c["top_k"],
                            act=synth._ACT_NAMES[c["act"]], n_zero=c["n_zero"], n_copy=c["n_copy"],
                            n_const=c["n_const"], has_proj=c["has_proj"])
    layer = {"x": _bf(spec["x"]), "w_router": _bf(spec["w_router"]), "w1": _bf(spec["w1"]), "w2": _bf(spec["w2"]),
             "w_down": _bf(spec["w_down"]) if "w_down" in spec else None,
             "w_up": _bf(spec["w_up"]) if "w_up" in spec else None,
             "const_vecs": _bf(spec["const_vecs"]) if "const_vecs" in spec else None, "bias": None}
    return cfg, layer


def _ev(expr, **names):
    return float(eval(expr, {"__builtins__": {}, "exp": math.exp}, names))


# --------------------------------------------------------------------------------------------
# hand-worked closed forms
# --------------------------------------------------------------------------------------------

def test_hand_worked_latent_layer():
    spec = json.load(open(GOLDEN))["latent_layer"]
    cfg, layer = _layer_from_json(spec)
    out = oracle.forward(cfg, layer, want=("y", "idx", "w"))
    x = np.asarray(spec["x"], np.float64)
    for t, ex in enumerate(spec["expected"]):
        assert list(out["idx"][t]) == ex["idx"], ex["note"]
        wu = np.array([_ev(s) for s in ex["w_unnorm"]])
        w = wu / wu.sum()
        np.testing.assert_allclose(out["w"][t], w, rtol=1e-14, atol=0)
        yl = (w[:, None] * np.asarray(ex["o"], np.float64)).sum(0)
        y = x[t] + np.array([yl[0], yl[1], yl[0] + yl[1], 0.0])
        np.testing.assert_allclose(out["y"][t], y, rtol=1e-13, atol=1e-13)


def test_hand_worked_gated_standard_layer():
    spec = json.load(open(GOLDEN))["gated_standard_layer"]
    cfg, layer = _layer_from_json(spec)
    out = oracle.forward(cfg, layer, want=("y", "idx", "w"))
    for t, ex in enumerate(spec["expected"]):
        assert list(out["idx"][t]) == ex["idx"]
        assert out["w"][t][0] == 1.0
        H = _ev(ex["h"])
        y = [_ev(s, H=H) for s in ex["y"]]
        np.testing.assert_allclose(out["y"][t], y, rtol=1e-14, atol=1e-15)


# --------------------------------------------------------------------------------------------
# routing: brute force over subsets, library softmax, ties
# --------------------------------------------------------------------------------------------

def test_route_matches_best_subset_bruteforce():
    rng = np.random.default_rng(11)
    for n_tot, K in [(7, 3), (6, 1), (8, 4), (5, 5)]:
        lg = rng.standard_normal((40, n_tot))
        idx, w = oracle.route(lg, K)
        for t in range(lg.shape[0]):
            best = max(itertools.combinations(range(n_tot), K), key=lambda s: sum(lg[t, list(s)]))
            assert set(idx[t]) == set(best)
            # slots ordered by logit, descending
            assert np.all(np.diff(lg[t, idx[t]]) < 0)
            # renormalised softmax: equals the full softmax restricted to the set and rescaled
            p = scipy.special.softmax(lg[t])
            np.testing.assert_allclose(w[t], p[idx[t]] / p[idx[t]].sum(), rtol=1e-13)
            assert abs(w[t].sum() - 1.0) < 1e-14


def test_route_full_topk_is_softmax_and_top1_is_one():
    rng = np.random.default_rng(12)
    lg = rng.standard_normal((20, 9)) * 3
    idx, w = oracle.route(lg, 9)
    for t in range(20):
        np.testing.assert_allclose(w[t], scipy.special.softmax(lg[t])[idx[t]], rtol=1e-13)
    idx1, w1 = oracle.route(lg, 1)
    assert np.all(w1 == 1.0)
    assert np.array_equal(idx1[:, 0], np.argmax(lg, axis=1))


def test_route_ties_go_to_lower_id():
    lg = np.array([[0.0, 1.0, 1.0, 0.5, 1.0, 0.5]])
    idx, w = oracle.route(lg, 4)
    assert list(idx[0]) == [1, 2, 4, 3]
    np.testing.assert_allclose(w[0], np.array([1, 1, 1, math.exp(-0.5)]) / (3 + math.exp(-0.5)), rtol=1e-15)


# --------------------------------------------------------------------------------------------
# dispatch: library stable argsort, bijection, counts
# --------------------------------------------------------------------------------------------

@pytest.mark.parametrize("T,K,n_tot", [(1, 1, 1), (37, 4, 16), (300, 6, 128), (5, 3, 1000)])
def test_dispatch_is_stable_sort(T, K, n_tot):
    rng = np.random.default_rng(T * 7 + K)
    idx = np.stack([rng.choice(n_tot, size=K, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, inv = oracle.dispatch(idx, n_tot)
    flat = idx.reshape(-1)
    assert counts.sum() == T * K
    assert np.array_equal(counts, np.bincount(flat, minlength=n_tot))
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(perm, np.argsort(flat, kind="stable"))
    assert np.array_equal(np.sort(perm), np.arange(T * K))
    assert np.array_equal(inv[perm], np.arange(T * K))


def test_dispatch_rejects_bad_ids():
    with pytest.raises(ValueError):
        oracle.dispatch(np.array([[0, 5]], np.int32), 5)


# --------------------------------------------------------------------------------------------
# whole layer: dense brute force, special cases, invariants
# --------------------------------------------------------------------------------------------

SMALL = synth.LayerConfig(d=32, latent=16, m=8, n_ffn=6, n_zero=1, n_copy=1, n_const=1, top_k=3, tokens=24, seed=5)


def _np(t):
    return None if t is None else t.to(torch.float64).numpy()


def _dense_bruteforce(cfg, layer):
    """Every expert on every token, then a full softmax masked to the best-sum K'-subset."""
    x, Wr, Wd, Wu = _np(layer["x"]), _np(layer["w_router"]), _np(layer["w_down"]), _np(layer["w_up"])
    W1, W2 = _np(layer["w1"]), _np(layer["w2"])
    T, m = x.shape[0], cfg.m
    z = x @ Wd.T if cfg.has_proj else x.copy()
    lg = (z if cfg.latent_router else x) @ Wr.T
    if layer.get("bias") is not None:
        lg = lg + layer["bias"].double().numpy()
    U = np.einsum("eol,tl->teo", W1, z)
    if cfg.act == synth.ACT_RELU2:
        Hh = np.maximum(U, 0) ** 2
    elif cfg.act == synth.ACT_SWIGLU:
        Hh = scipy.special.expit(U[..., :m]) * U[..., :m] * U[..., m:]
    else:
        Hh = U
    O = np.einsum("elm,tem->tel", W2, Hh)
    extra = [np.zeros_like(z)] * cfg.n_zero + [z] * cfg.n_copy
    extra += [np.broadcast_to(_np(layer["const_vecs"])[c], z.shape) for c in range(cfg.n_const)]
    if extra:
        O = np.concatenate([O, np.stack(extra, axis=1)], axis=1)
    P = scipy.special.softmax(lg, axis=1)
    yl = np.zeros_like(z)
    for t in range(T):
        best = max(itertools.combinations(range(cfg.n_total), cfg.top_k), key=lambda s: sum(lg[t, list(s)]))
        mask = np.zeros(cfg.n_total)
        mask[list(best)] = 1
        w = P[t] * mask / (P[t] * mask).sum()
        yl[t] = (w[:, None] * O[t]).sum(0)
    up = yl @ Wu.T if cfg.has_proj else yl
    if getattr(cfg, "shared_m", 0):
        Us = x @ _np(layer["w_shared1"]).T
        ms = cfg.shared_m
        if cfg.act == synth.ACT_RELU2:
            Hs = np.maximum(Us, 0) ** 2
        elif cfg.act == synth.ACT_SWIGLU:
            Hs = scipy.special.expit(Us[:, :ms]) * Us[:, :ms] * Us[:, ms:]
        else:
            Hs = Us
        up = up + Hs @ _np(layer["w_shared2"]).T
    return x + up


@pytest.mark.parametrize("act", ["relu2", "swiglu", "identity"])
def test_layer_matches_dense_bruteforce(act):
    cfg = SMALL.with_(act=act)
    layer = synth.make_layer(cfg)
    out = oracle.forward(cfg, layer)
    np.testing.assert_allclose(out["y"], _dense_bruteforce(cfg, layer), rtol=1e-11, atol=1e-11)


def test_layer_with_bias_matches_dense_bruteforce():
    cfg = SMALL.with_(zipf=1.1, act="swiglu")
    layer = synth.make_layer(cfg)
    assert layer["bias"] is not None
    out = oracle.forward(cfg, layer)
    np.testing.assert_allclose(out["y"], _dense_bruteforce(cfg, layer), rtol=1e-11, atol=1e-11)


def test_several_bypass_experts_of_each_kind_match_dense_bruteforce():
    cfg = SMALL.with_(n_zero=2, n_copy=2, n_const=3, top_k=4, zipf=0.8)
    layer = synth.make_layer(cfg)
    out = oracle.forward(cfg, layer)
    assert np.any(out["idx"] >= cfg.n_ffn + cfg.n_zero + cfg.n_copy + 1)   # a second constant expert is used
    np.testing.assert_allclose(out["y"], _dense_bruteforce(cfg, layer), rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("act", ["relu2", "swiglu"])
def test_shared_expert_matches_dense_bruteforce(act):
    cfg = SMALL.with_(act=act, shared_m=12, zipf=0.7)
    layer = synth.make_layer(cfg)
    assert layer["w_shared1"].shape == ((24 if act == "swiglu" else 12), cfg.d)
    out = oracle.forward(cfg, layer)
    np.testing.assert_allclose(out["y"], _dense_bruteforce(cfg, layer), rtol=1e-11, atol=1e-11)


def test_shared_expert_alone_is_a_plain_ffn_on_x():
    """Routing forced to the zero expert leaves y = x + Ws2 relu(Ws1 x)^2, and scaling Ws2 scales y - x."""
    cfg = SMALL.with_(top_k=1, shared_m=10)
    layer = synth.make_layer(cfg)
    bias = torch.full((cfg.n_total,), -100.0)
    bias[cfg.n_ffn] = 100.0                       # the zero expert
    x = _np(layer["x"])
    ffn = np.maximum(x @ _np(layer["w_shared1"]).T, 0) ** 2 @ _np(layer["w_shared2"]).T
    a = oracle.forward(cfg, dict(layer, bias=bias))
    np.testing.assert_allclose(a["y"], x + ffn, rtol=1e-12, atol=1e-12)
    b = oracle.forward(cfg, dict(layer, bias=bias, w_shared2=layer["w_shared2"] * 2))
    np.testing.assert_allclose(b["y"] - x, 2 * (a["y"] - x), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("act", ["relu2", "swiglu"])
@pytest.mark.parametrize("has_proj", [1, 0])
def test_one_expert_top1_is_a_plain_ffn(act, has_proj):
    """N' = K' = 1 (no bypass experts): the only expert gets weight 1 for every token, so the layer is
    x + W_up W2 act(W1 W_down x), or x + W2 act(W1 x) without projections, here in numpy fp64 matmuls."""
    cfg = SMALL.with_(n_ffn=1, n_zero=0, n_copy=0, n_const=0, top_k=1, act=act, has_proj=has_proj,
                      latent=SMALL.latent if has_proj else SMALL.d)
    layer = synth.make_layer(cfg, tokens=9)
    x = _np(layer["x"])
    z = x @ _np(layer["w_down"]).T if has_proj else x
    u = z @ _np(layer["w1"][0]).T
    if act == "swiglu":
        g, up = u[:, :cfg.m], u[:, cfg.m:]
        h = g / (1.0 + np.exp(-g)) * up
    else:
        h = np.maximum(u, 0.0) ** 2
    o = h @ _np(layer["w2"][0]).T
    y = x + (o @ _np(layer["w_up"]).T if has_proj else o)
    ref = oracle.forward(cfg, layer, want=("y", "idx", "w"))
    assert np.all(ref["idx"] == 0) and np.all(ref["w"] == 1.0)
    np.testing.assert_allclose(ref["y"], y, rtol=1e-12, atol=1e-12)


def test_latent_router_matches_dense_bruteforce():
    cfg = SMALL.with_(latent_router=1)
    layer = synth.make_layer(cfg)
    out = oracle.forward(cfg, layer)
    np.testing.assert_allclose(out["y"], _dense_bruteforce(cfg, layer), rtol=1e-11, atol=1e-11)


def test_latent_router_gate_reads_the_unrounded_latent():
    """The gate takes the latent at full precision ("How LatentMoE Works" step 2 says nothing of a rounding).

    z_0 = x_0 + 2^-10 x_1 = 1 + 2^-10 has no bf16 value (bf16 rounds it to 1).  Expert 0's logit is z_0,
    expert 1's is the constant bias 1 + 2^-11.  On the exact latent expert 0 wins top-1; a gate that read
    a bf16-rounded latent would pick expert 1.  The two experts differ (W2 of expert 1 is doubled), so
    the layer output tells which one ran."""
    cfg = synth.LayerConfig(d=8, latent=8, m=4, n_ffn=2, top_k=1, tokens=1, seed=12, latent_router=1)
    layer = synth.make_layer(cfg)
    x = torch.zeros(1, 8, dtype=torch.bfloat16)
    x[0, 0] = 1.0
    x[0, 1] = 1.0
    wd = torch.eye(8, dtype=torch.bfloat16)
    wd[0, 1] = 2.0 ** -10
    wr = torch.zeros(2, 8, dtype=torch.bfloat16)
    wr[0, 0] = 1.0
    bias = torch.tensor([0.0, 1.0 + 2.0 ** -11], dtype=torch.float32)
    w2 = layer["w2"].clone()
    w2[1] = layer["w2"][0] * 2
    w1 = layer["w1"].clone()
    w1[1] = layer["w1"][0]
    lay = dict(layer, x=x, w_down=wd, w_router=wr, bias=bias, w1=w1, w2=w2)
    out = oracle.forward(cfg, lay, want=("y", "idx", "w", "z", "logits"))
    assert out["z"][0, 0] == 1.0 + 2.0 ** -10
    assert float(torch.tensor(out["z"][0, 0]).to(torch.bfloat16)) == 1.0
    assert out["idx"][0, 0] == 0 and out["w"][0, 0] == 1.0
    assert out["logits"][0, 0] == 1.0 + 2.0 ** -10 and out["logits"][0, 1] == np.float32(1.0 + 2.0 ** -11)
    # expert 0's output on the exact latent (numpy fp64): y = x + W_up W2_0 relu(W1_0 z)^2
    z = _np(x) @ _np(wd).T
    h = np.maximum(z @ _np(w1[0]).T, 0) ** 2
    y = _np(x) + (h @ _np(w2[0]).T) @ _np(lay["w_up"]).T
    np.testing.assert_allclose(out["y"], y, rtol=1e-12, atol=1e-12)


def test_identity_projections_reproduce_standard_moe():
    """latent = d with W_down = W_up = I gives exactly the standard MoE (Figure 3a vs 3b)."""
    std = synth.LayerConfig(d=16, latent=16, m=8, n_ffn=5, top_k=2, has_proj=0, tokens=20, seed=6)
    layer = synth.make_layer(std)
    a = oracle.forward(std, layer)
    lat = std.with_(has_proj=1)
    eye = torch.eye(16, dtype=torch.bfloat16)
    b = oracle.forward(lat, dict(layer, w_down=eye, w_up=eye))
    assert np.array_equal(a["idx"], b["idx"])
    assert np.array_equal(a["y"], b["y"])


def test_latent_router_equals_full_width_router_on_selecting_projection():
    """W_down = [I 0] makes z = x[:latent]; a latent router R then equals the full-width router [R 0]."""
    cfg = synth.LayerConfig(d=24, latent=8, m=8, n_ffn=6, top_k=2, tokens=16, seed=9, latent_router=1)
    layer = synth.make_layer(cfg)
    wd = torch.zeros(8, 24, dtype=torch.bfloat16)
    wd[:, :8] = torch.eye(8)
    a = oracle.forward(cfg, dict(layer, w_down=wd))
    wr_full = torch.zeros(cfg.n_total, 24, dtype=torch.bfloat16)
    wr_full[:, :8] = layer["w_router"]
    b = oracle.forward(cfg.with_(latent_router=0), dict(layer, w_down=wd, w_router=wr_full))
    assert np.array_equal(a["idx"], b["idx"])
    assert np.array_equal(a["y"], b["y"])


def test_relabelling_experts_is_equivariant():
    cfg = SMALL.with_(zipf=1.1)
    layer = synth.make_layer(cfg)
    base = oracle.forward(cfg, layer)
    rng = np.random.default_rng(3)
    pi = rng.permutation(cfg.n_ffn)          # new FFN id j holds old expert pi[j]
    full = np.concatenate([pi, np.arange(cfg.n_ffn, cfg.n_total)])
    moved = dict(layer, w_router=layer["w_router"][full], w1=layer["w1"][pi], w2=layer["w2"][pi],
                 bias=layer["bias"][full])
    out = oracle.forward(cfg, moved)
    np.testing.assert_allclose(out["y"], base["y"], rtol=1e-13, atol=1e-13)
    assert np.array_equal(full[out["idx"]], base["idx"])


def test_bypass_experts_zero_copy_const():
    cfg = SMALL.with_(top_k=1)
    layer = synth.make_layer(cfg)
    x = _np(layer["x"])
    Wd, Wu = _np(layer["w_down"]), _np(layer["w_up"])
    for e, expect in [(6, lambda: x), (7, lambda: x + (x @ Wd.T) @ Wu.T),
                      (8, lambda: x + _np(layer["const_vecs"])[0] @ Wu.T)]:
        bias = torch.full((cfg.n_total,), -100.0)
        bias[e] = 100.0
        out = oracle.forward(cfg, dict(layer, bias=bias))
        assert np.all(out["idx"] == e) and np.all(out["w"] == 1.0)
        np.testing.assert_allclose(out["y"], np.broadcast_to(expect(), out["y"].shape), rtol=1e-13, atol=1e-13)
    # a zero expert in the selection lowers the others' weights (it takes its share of the softmax)
    cfg2 = SMALL.with_(top_k=2)
    bias = torch.zeros(cfg2.n_total)
    bias[6] = 100.0
    out = oracle.forward(cfg2, dict(layer, bias=bias))
    assert np.all(out["idx"][:, 0] == 6)
    assert np.all(out["w"][:, 0] > 0.999)


def test_scaling_w2_and_w1_scales_the_moe_delta():
    """Router untouched: W2 -> 2 W2 doubles y - x; W1 -> 2 W1 quadruples it under relu^2."""
    cfg = SMALL.with_(n_zero=0, n_copy=0, n_const=0)
    layer = synth.make_layer(cfg)
    x = _np(layer["x"])
    d0 = oracle.forward(cfg, layer)["y"] - x
    d2 = oracle.forward(cfg, dict(layer, w2=layer["w2"] * 2))["y"] - x
    d4 = oracle.forward(cfg, dict(layer, w1=layer["w1"] * 2))["y"] - x
    np.testing.assert_allclose(d2, 2 * d0, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(d4, 4 * d0, rtol=1e-12, atol=1e-13)


def test_identity_activation_closed_form():
    """act = identity: y = x + W_up sum_k w_k (W2_e W1_e) W_down x, with the expert product formed first."""
    cfg = SMALL.with_(act="identity", n_zero=0, n_copy=0, n_const=0)
    layer = synth.make_layer(cfg)
    out = oracle.forward(cfg, layer)
    x, Wd, Wu = _np(layer["x"]), _np(layer["w_down"]), _np(layer["w_up"])
    M = np.einsum("elm,emk->elk", _np(layer["w2"]), _np(layer["w1"]))   # [E, latent, latent]
    A = np.einsum("dl,elk,kD->edD", Wu, M, Wd)                            # [E, d, d]
    exp_y = np.stack([x[t] + sum(out["w"][t, k] * A[out["idx"][t, k]] @ x[t] for k in range(cfg.top_k))
                      for t in range(x.shape[0])])
    np.testing.assert_allclose(out["y"], exp_y, rtol=1e-11, atol=1e-11)


def test_weights_sum_to_one_and_counts_sum_to_slots():
    cfg = synth.WORKLOADS["tiny"]
    layer = synth.make_layer(cfg)
    out = oracle.forward(cfg, layer)
    np.testing.assert_allclose(out["w"].sum(1), 1.0, atol=1e-14)
    assert np.all(np.diff(out["w"], axis=1) <= 0)
    counts, offsets, perm, inv = oracle.dispatch(out["idx"], cfg.n_total)
    assert counts.sum() == cfg.tokens * cfg.top_k


def test_forced_routes_reuse_router_weights():
    """Passing the router's own selection back in reproduces the run exactly."""
    cfg = SMALL
    layer = synth.make_layer(cfg)
    a = oracle.forward(cfg, layer)
    b = oracle.forward(cfg, layer, idx=a["idx"])
    assert np.array_equal(a["y"], b["y"]) and np.array_equal(a["w"], b["w"])


def test_empty_batch():
    cfg = synth.WORKLOADS["tiny"]
    layer = synth.make_layer(cfg, tokens=0)
    out = oracle.forward(cfg, layer)
    assert out["y"].shape == (0, cfg.d)
