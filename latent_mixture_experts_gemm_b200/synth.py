"""Seeded synthetic inputs for the LatentMoE layer.

This module only draws numbers: it holds none of the layer's arithmetic.  The
CUDA path, the tests, the benchmark and the fp64 oracle all take their inputs
from here, so both sides of every parity check see the same bf16 tensors.

Recipe (one ``torch.Generator('cpu')`` per workload, seeded with its seed):

* draw order: x, router weight, W_down, W_up, W1 (expert by expert), W2
  (expert by expert), constant-expert vectors, the Zipf rank permutation, then
  the shared expert's two matrices (when the layer has one);
* every weight is ``randn * 1/sqrt(fan_in)`` in fp32, rounded to bf16 (round to
  nearest even); fan_in is the input width of the matrix (d for the router and
  W_down, latent for W_up and W1, m for W2); x and the constant vectors are
  ``randn`` (unit variance);
* with a Zipf exponent s, the router gets a bias ``b_e = -s * ln(r_e)`` where
  ``r`` is a seeded permutation of 1..N'_tot over all routed experts (bypass
  experts included), which scales each expert's routing probability by
  ``r_e^-s``: a skewed load like the one a trained router shows.

The shapes are those of the layers the pages discuss: a Nemotron-3-Super-like
layer (d=4096, latent 1024, 512 experts, top-22), its standard-MoE equal-budget
baseline (d=4096, 128 experts, top-6, no projection), and a Kimi-K3-like layer
(896 FFN experts, top-16, gated experts, MoE++ zero/copy/constant experts).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch

ACT_RELU2 = 0
ACT_SWIGLU = 1
ACT_IDENTITY = 2
_ACT_NAMES = {"relu2": ACT_RELU2, "swiglu": ACT_SWIGLU, "identity": ACT_IDENTITY}


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    """Shapes of one LatentMoE layer (plus the token count and seed of a workload)."""

    d: int
    latent: int
    m: int
    n_ffn: int
    top_k: int
    act: int = ACT_RELU2
    n_zero: int = 0
    n_copy: int = 0
    n_const: int = 0
    has_proj: int = 1
    latent_router: int = 0
    shared_m: int = 0
    expert_fmt: int = 0
    tokens: int = 0
    seed: int = 0
    zipf: float = 0.0
    name: str = ""

    @property
    def n_total(self) -> int:
        return self.n_ffn + self.n_zero + self.n_copy + self.n_const

    @property
    def gated(self) -> bool:
        return self.act == ACT_SWIGLU

    @property
    def up_rows(self) -> int:
        return 2 * self.m if self.gated else self.m

    @property
    def router_in(self) -> int:
        return self.latent if self.latent_router else self.d

    def with_(self, **kw) -> "LayerConfig":
        if "act" in kw and isinstance(kw["act"], str):
            kw["act"] = _ACT_NAMES[kw["act"]]
        return dataclasses.replace(self, **kw)


def _cfg(**kw) -> LayerConfig:
    if isinstance(kw.get("act"), str):
        kw["act"] = _ACT_NAMES[kw["act"]]
    return LayerConfig(**kw)


#: Named workloads.  ``tiny`` is small enough for the oracle to finish in well
#: under a second; the others carry the pages' layer shapes.
WORKLOADS: Dict[str, LayerConfig] = {
    "tiny": _cfg(name="tiny", tokens=64, d=256, latent=64, m=128, n_ffn=16, top_k=4, act="relu2", seed=0),
    "nemotron_decode": _cfg(name="nemotron_decode", tokens=32, d=4096, latent=1024, m=1024, n_ffn=512,
                            top_k=22, act="relu2", seed=1),
    "nemotron_prefill": _cfg(name="nemotron_prefill", tokens=8192, d=4096, latent=1024, m=1024, n_ffn=512,
                             top_k=22, act="relu2", seed=2),
    "std_prefill": _cfg(name="std_prefill", tokens=8192, d=4096, latent=4096, m=1024, n_ffn=128, top_k=6,
                        act="relu2", has_proj=0, seed=3),
    "std_decode": _cfg(name="std_decode", tokens=32, d=4096, latent=4096, m=1024, n_ffn=128, top_k=6,
                       act="relu2", has_proj=0, seed=3),
    "kimi_skew": _cfg(name="kimi_skew", tokens=4096, d=7168, latent=1792, m=1024, n_ffn=896, n_zero=4,
                      n_copy=4, n_const=4, top_k=16, act="swiglu", zipf=1.1, seed=4),
    # the Nemotron-like layer with a shared expert at the full width (hidden width 2m: the pages give none)
    "nemotron_decode_shared": _cfg(name="nemotron_decode_shared", tokens=32, d=4096, latent=1024, m=1024,
                                   n_ffn=512, top_k=22, act="relu2", shared_m=2048, seed=5),
    "nemotron_prefill_shared": _cfg(name="nemotron_prefill_shared", tokens=8192, d=4096, latent=1024, m=1024,
                                    n_ffn=512, top_k=22, act="relu2", shared_m=2048, seed=6),
    # the Nemotron-like decode batch with block-scaled expert weights (MXFP8: E4M3 elements; MXFP4: E2M1)
    "nemotron_decode_mxfp8": _cfg(name="nemotron_decode_mxfp8", tokens=32, d=4096, latent=1024, m=1024, n_ffn=512,
                                  top_k=22, act="relu2", expert_fmt=1, seed=7),
    "nemotron_decode_mxfp4": _cfg(name="nemotron_decode_mxfp4", tokens=32, d=4096, latent=1024, m=1024, n_ffn=512,
                                  top_k=22, act="relu2", expert_fmt=2, seed=8),
    "nemotron_decode_nvfp4": _cfg(name="nemotron_decode_nvfp4", tokens=32, d=4096, latent=1024, m=1024, n_ffn=512,
                                  top_k=22, act="relu2", expert_fmt=3, seed=6),
}


def _draw(g: torch.Generator, shape, scale: float) -> torch.Tensor:
    t = torch.randn(*shape, generator=g, dtype=torch.float32)
    if scale != 1.0:
        t.mul_(scale)
    return t.to(torch.bfloat16)


def make_layer(cfg: LayerConfig, tokens: Optional[int] = None, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Draw x and every weight of ``cfg`` on the CPU (bf16, plus an fp32 bias).

    Returns a dict with keys ``x, w_router, bias, w_down, w_up, w1, w2,
    const_vecs, w_shared1, w_shared2``; absent tensors (no projection, no bias,
    no constant experts, no shared expert) are ``None``.  W1 is
    ``[N', g*m, latent]`` with the gate rows first when gated; W2 is
    ``[N', latent, m]``.  The shared expert's W1 is ``[g*shared_m, d]`` (gate
    rows first when gated), its W2 ``[d, shared_m]``.
    """
    T = cfg.tokens if tokens is None else tokens
    s = cfg.seed if seed is None else seed
    g = torch.Generator(device="cpu").manual_seed(s)
    L, d, m = cfg.latent, cfg.d, cfg.m
    out: Dict[str, Optional[torch.Tensor]] = {}
    out["x"] = _draw(g, (T, d), 1.0)
    out["w_router"] = _draw(g, (cfg.n_total, cfg.router_in), 1.0 / math.sqrt(cfg.router_in))
    if cfg.has_proj:
        out["w_down"] = _draw(g, (L, d), 1.0 / math.sqrt(d))
        out["w_up"] = _draw(g, (d, L), 1.0 / math.sqrt(L))
    else:
        out["w_down"] = None
        out["w_up"] = None
    w1 = torch.empty((cfg.n_ffn, cfg.up_rows, L), dtype=torch.bfloat16)
    for e in range(cfg.n_ffn):
        w1[e] = _draw(g, (cfg.up_rows, L), 1.0 / math.sqrt(L))
    w2 = torch.empty((cfg.n_ffn, L, m), dtype=torch.bfloat16)
    for e in range(cfg.n_ffn):
        w2[e] = _draw(g, (L, m), 1.0 / math.sqrt(m))
    out["w1"] = w1
    out["w2"] = w2
    out["const_vecs"] = _draw(g, (cfg.n_const, L), 1.0) if cfg.n_const else None
    if cfg.zipf:
        ranks = torch.randperm(cfg.n_total, generator=g).to(torch.float64) + 1.0
        out["bias"] = (-cfg.zipf * torch.log(ranks)).to(torch.float32)
    else:
        out["bias"] = None
    if cfg.shared_m:
        rows = 2 * cfg.shared_m if cfg.gated else cfg.shared_m
        out["w_shared1"] = _draw(g, (rows, d), 1.0 / math.sqrt(d))
        out["w_shared2"] = _draw(g, (d, cfg.shared_m), 1.0 / math.sqrt(cfg.shared_m))
    else:
        out["w_shared1"] = out["w_shared2"] = None
    return out


def make_tokens(cfg: LayerConfig, tokens: int, seed: int) -> torch.Tensor:
    """Fresh x of ``tokens`` rows from its own seeded generator (bf16, unit variance)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    return _draw(g, (tokens, cfg.d), 1.0)
