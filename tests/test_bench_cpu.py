"""The benchmark's algorithmic work of a forward, on CPU.

`bench.layer_work` gives the FLOPs F and the bytes B of one forward from its
actual routing; the layer roofline is max(F / peak FLOP/s, B / HBM bandwidth).
The expected values below were derived from the layer's definition before
any code existed, for the configurations' sizes with uniform routing (every
slot on an FFN expert, the touched-expert counts stated), so they pin the
formula the benchmark reports against.
"""
import pytest

import bench
from latent_mixture_experts_gemm_b200 import synth

# (workload, ffn rows, experts touched, expected F, expected B)
EXPECTED = [
    ("nemotron_decode", 32 * 22, 386, 3.62e9, 1.642e9),
    ("nemotron_prefill", 8192 * 22, 512, 927.7e9, 2.30e9),
    ("std_prefill", 8192 * 6, 128, 833.2e9, 2.28e9),
    ("std_decode", 32 * 6, 100, 3.26e9, 1.687e9),
]


@pytest.mark.parametrize("name,rows,touched,F_exp,B_exp", EXPECTED)
def test_layer_work_matches_the_expected_work(name, rows, touched, F_exp, B_exp):
    cfg = synth.WORKLOADS[name]
    F, B, F_eff = bench.layer_work(cfg, {"ffn_rows": rows, "experts_touched": touched}, cfg.tokens)
    assert F == pytest.approx(F_exp, rel=3e-3)
    assert B == pytest.approx(B_exp, rel=1e-2)  # the expected bytes were rounded to MiB-sized weights
    assert F_eff == pytest.approx(F, rel=1e-12)  # bf16 experts run at the bf16 rate


def test_decode_is_hbm_bound_and_prefill_tensor_bound():
    """With the measured peaks (6540 GB/s, 1646 TFLOP/s): decode reads, prefill computes."""
    for name, rows, touched, _, _ in EXPECTED:
        cfg = synth.WORKLOADS[name]
        F, B, F_eff = bench.layer_work(cfg, {"ffn_rows": rows, "experts_touched": touched}, cfg.tokens)
        t_f, t_b = F_eff / 1646e12, B / 6540e9
        assert (t_b > t_f) == name.endswith("decode"), name
