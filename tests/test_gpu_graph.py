"""The layer forward captured in a CUDA graph and replayed, through the C ABI.

lmoe_forward enqueues kernels only: no allocation, no host synchronisation,
with the shared expert's second stream forked and joined by events.  A graph
capture of it therefore replays the same kernels, and every replay gives the
eager forward's output bit for bit, for whatever the captured input buffer
holds at replay time.  The cases cover the decode paths (split-K projections,
weight streaming, NVFP4 experts), the prefill paths (tensor-core GEMMs) and the
shared expert on its own stream.
"""
import pytest
import torch

from latent_mixture_experts_gemm_b200 import lmoe, synth

pytestmark = pytest.mark.gpu

MEDIUM = synth.LayerConfig(name="graph_medium", tokens=300, d=512, latent=128, m=256, n_ffn=64, top_k=6, seed=121)

CASES = {
    "nemotron_decode": synth.WORKLOADS["nemotron_decode"],
    "nemotron_decode_nvfp4": synth.WORKLOADS["nemotron_decode_nvfp4"],
    "medium_swiglu_shared_bypass": MEDIUM.with_(act="swiglu", shared_m=256, n_zero=1, n_copy=1, n_const=1, seed=122),
    "medium_decode_shared": MEDIUM.with_(tokens=24, shared_m=128, seed=123),
}


@pytest.mark.parametrize("name", list(CASES))
def test_graph_replay_matches_the_eager_forward(name):
    cfg = CASES[name]
    T = cfg.tokens
    layer = synth.make_layer(cfg)
    mod = lmoe.LatentMoE(cfg, layer, max_tokens=T)
    try:
        xs = [synth.make_tokens(cfg, T, seed=500 + i).cuda() for i in range(3)]
        eager = [mod.forward(x) for x in xs]
        torch.cuda.synchronize()
        static_x = xs[0].clone()
        static_y = torch.empty_like(static_x)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):  # one eager forward on the capture's stream first
            mod.forward(static_x, static_y)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            mod.forward(static_x, static_y)
        for x, ref in zip(xs, eager):
            static_x.copy_(x)
            static_y.zero_()
            g.replay()
            torch.cuda.synchronize()
            assert torch.equal(static_y, ref)
        assert mod.last_error() == 0
        del g
    finally:
        mod.close()
