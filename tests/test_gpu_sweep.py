"""A seeded sweep of small layer configurations, GPU against the oracle.

The named layer cases fix one feature at a time.  This sweep draws 40
configurations from a seeded generator and combines the features at random:
* widths (d, latent, m) in multiples of 64, or of 128 / 256 where the expert
  format needs it;
* 2 to 96 FFN experts, top-1 to top-12, 1 to 300 tokens (ragged tiles);
* ReLU², SwiGLU or identity activations;
* zero / copy / constant experts;
* a shared expert, the latent router, the standard MoE (no projections);
* bf16, MXFP8, MXFP4 or NVFP4 experts;
* both expert paths (the weight-streaming threshold 0, 8 or 16).

Each case is compared with the checker the named cases use: the contract's
tolerances, dispatch bit-exact, near-tie tokens against the oracle re-run on
the GPU's own routes.
"""
import random

import pytest

from latent_mixture_experts_gemm_b200 import synth
from tests.test_gpu_layer import _run_and_check

pytestmark = pytest.mark.gpu


def _draw(i: int) -> tuple:
    r = random.Random(9000 + i)
    fmt = r.choice([0, 0, 0, 1, 2, 3])
    unit = {0: 64, 1: 128, 2: 128, 3: 256}[fmt]
    has_proj = r.random() < 0.8
    d = r.choice([2, 3, 4, 6]) * max(unit, 64)
    latent = r.choice([1, 2, 3]) * unit if has_proj else d
    m = r.choice([1, 2, 3, 4]) * unit
    n_ffn = r.choice([2, 5, 8, 16, 33, 64, 96])
    n_zero, n_copy, n_const = (r.choice([0, 0, 1, 2]) for _ in range(3))
    n_total = n_ffn + n_zero + n_copy + n_const
    top_k = r.randint(1, min(12, n_total))
    tokens = r.choice([1, 7, 16, 29, 32, 77, 130, 257, 300])
    act = r.choice(["relu2", "relu2", "swiglu", "identity"])
    cfg = synth.LayerConfig(name=f"sweep{i}", tokens=tokens, d=d, latent=latent, m=m, n_ffn=n_ffn, top_k=top_k,
                            n_zero=n_zero, n_copy=n_copy, n_const=n_const, has_proj=int(has_proj),
                            latent_router=int(has_proj and r.random() < 0.25),
                            shared_m=r.choice([0, 0, 0, 64, 128]) if fmt == 0 else r.choice([0, 128]),
                            expert_fmt=fmt, zipf=r.choice([0.0, 0.0, 1.1]), seed=5000 + i)
    cfg = cfg.with_(act=act)
    small_rows = r.choice([None, 0, 8])
    return cfg, small_rows


@pytest.mark.parametrize("i", range(40))
def test_random_configuration_matches_the_oracle(i):
    cfg, small_rows = _draw(i)
    _run_and_check(cfg, synth.make_layer(cfg), small_rows=small_rows)
