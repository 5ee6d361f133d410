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


def test_grouped_expert_gemm_roofline_is_tensor_framed():
    """A prefill grouped GEMM's bytes are its touched experts' weights (the gathered and hidden rows are
    intermediates), so it is tensor-bound: 377.96 GFLOP in 0.3843 ms is 0.598 of a 1645.9 TFLOP/s peak."""
    cfg = synth.WORKLOADS["nemotron_prefill"]
    stats = {"ffn_rows": 8192 * 22, "experts_touched": 512, "tc_rows": 8192 * 22, "tc_experts": 512,
             "stream_rows": 0, "stream_experts": 0}
    peaks = {"hbm_gbs": 6540.2, "bf16_tflops": 1645.9, "source": "measured"}
    phases = {"expert_up_gemm": (0.3843, 1), "expert_down_gemm": (0.3809, 1), "combine": (0.07, 1)}
    roof, layer, launches = bench.rooflines(cfg, stats, cfg.tokens, phases, peaks, 1.09)
    assert roof["kernel"] == "expert_up_gemm" and roof["bound"] == "tensor"
    assert roof["algorithmic_per_launch"]["bytes"] == 2 * 1024 * 1024 * 512  # W1: bf16 m x latent per expert
    assert roof["frac"] == pytest.approx(377.96e9 / 0.3843e-3 / 1645.9e12, rel=1e-3)
    assert launches == 3


def test_decode_weight_stream_roofline_is_hbm_framed():
    """A decode weight stream's bytes are the touched experts' weights: 380 experts x 2 MiB in 0.1246 ms."""
    cfg = synth.WORKLOADS["nemotron_decode"]
    stats = {"ffn_rows": 704, "experts_touched": 380, "tc_rows": 0, "tc_experts": 0, "stream_rows": 704,
             "stream_experts": 380}
    peaks = {"hbm_gbs": 6540.2, "bf16_tflops": 1645.9, "source": "measured"}
    roof, _, _ = bench.rooflines(cfg, stats, 32, {"expert_up_stream": (0.1246, 1)}, peaks, 0.286)
    assert roof["bound"] == "hbm"
    assert roof["achieved"] == pytest.approx(380 * 2 * 1024 * 1024 / 0.1246e-3 / 1e9, rel=1e-9)


def test_block_scaled_expert_gemm_takes_its_own_dtype_peak():
    """An NVFP4 expert contraction that is compute-bound is framed against 4x the bf16 peak (fp4 : bf16)."""
    cfg = synth.WORKLOADS["nemotron_decode_nvfp4"].with_(tokens=8192, name="nvfp4_big")
    stats = {"ffn_rows": 8192 * 22, "experts_touched": 512, "tc_rows": 0, "tc_experts": 0,
             "stream_rows": 8192 * 22, "stream_experts": 512}
    peaks = {"hbm_gbs": 6540.2, "bf16_tflops": 1645.9, "source": "measured"}
    roof, _, _ = bench.rooflines(cfg, stats, cfg.tokens, {"expert_up_stream": (0.2, 1)}, peaks, 1.0)
    assert roof["bound"] == "tensor" and roof["peak"] == pytest.approx(4 * 1645.9)


def test_every_benchmarked_workload_has_traffic_for_its_expert_phases():
    """Each workload of the default benchmark run carries the ncu traffic of its dominant kernel: the expert
    phases (weight streams at decode, grouped GEMMs at prefill; the Kimi-like layer runs both) all have an
    entry, so a bench line never reports a null traffic for them."""
    names = [bench.DEFAULT_WORKLOAD] + list(bench.SECONDARY_WORKLOADS)
    for name in names:
        cfg = synth.WORKLOADS[name]
        phases = ["expert_up_stream", "expert_down_stream"] if cfg.tokens <= 32 else ["expert_up_gemm",
                                                                                       "expert_down_gemm"]
        for ph in phases:
            assert (name, ph) in bench.NCU_TRAFFIC, (name, ph)
            assert bench.NCU_TRAFFIC[(name, ph)] > 0

