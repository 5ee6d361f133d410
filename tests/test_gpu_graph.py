"""CUDA graphs, through the C ABI: the layer forward captured by the caller and replayed, and the
library's own graph launch of each forward.

lmoe_forward enqueues kernels only: no allocation, no host synchronisation,
with the shared expert's second stream forked and joined by events.  A graph
capture of it therefore replays the same kernels, and every replay gives the
eager forward's output bit for bit, for whatever the captured input buffer
holds at replay time.  The cases cover the decode paths (split-K projections,
weight streaming, NVFP4 experts), the prefill paths (tensor-core GEMMs) and the
shared expert on its own stream.
"""
import warnings

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


# lmoe_forward launches each forward as a CUDA graph of its own by default (captured on the handle's stream,
# replayed from one executable graph).  These cases check it against the kernels launched one by one.
LIB_GRAPH_CASES = dict(CASES, std_moe_medium=MEDIUM.with_(has_proj=0, latent=512, seed=124),
                       medium_latent_router=MEDIUM.with_(latent_router=1, seed=125))


@pytest.mark.parametrize("name", list(LIB_GRAPH_CASES))
def test_library_graph_launch_matches_direct_launches(name):
    cfg = LIB_GRAPH_CASES[name]
    T = cfg.tokens
    layer = synth.make_layer(cfg)
    mod = lmoe.LatentMoE(cfg, layer, max_tokens=T)
    try:
        # token counts that keep the launch sequence (graph updated in place) and change it (rebuilt)
        sizes = [T, T, max(1, T // 2), min(T, 24), T]
        xs = [synth.make_tokens(cfg, n, seed=700 + i).cuda() for i, n in enumerate(sizes)]
        lmoe.lmoe_set_graph_launch(mod.h, False)
        direct = [mod.forward(x) for x in xs]
        torch.cuda.synchronize()
        lmoe.lmoe_set_graph_launch(mod.h, True)
        graphed = [mod.forward(x) for x in xs]
        torch.cuda.synchronize()
        assert mod.last_error() == 0
        for a, b in zip(direct, graphed):
            assert torch.equal(a, b)
        # alternating between two launch sequences replays each one's kept graph
        for _ in range(3):
            for i in (0, 3):
                assert torch.equal(mod.forward(xs[i]), direct[i])
        torch.cuda.synchronize()
        assert mod.last_error() == 0
        # the host-buffer entry point takes the same graph path
        xh = xs[0].cpu().pin_memory()
        yh = torch.empty_like(xh).pin_memory()
        mod.forward_host(xh, yh)
        torch.cuda.synchronize()
        assert torch.equal(yh, direct[0].cpu())
    finally:
        mod.close()


def test_graph_launch_switch_rejects_bad_values():
    cfg = MEDIUM.with_(tokens=8)
    mod = lmoe.LatentMoE(cfg, synth.make_layer(cfg), max_tokens=8)
    try:
        assert lmoe.lib().lmoe_set_graph_launch(mod.h, 2) == -1
        lmoe.lmoe_set_graph_launch(mod.h, False)
        lmoe.lmoe_set_graph_launch(mod.h, True)
    finally:
        mod.close()


@pytest.mark.parametrize("name", ["nemotron_decode", "medium_prefill_path"])
def test_graph_launch_device_memory(name):
    """How much device memory the library's graph launch takes: the free memory the driver reports
    (cudaMemGetInfo) before and after the first graph-launched forward of a handle, after a direct-launch
    forward has loaded every kernel's module, with no other allocation in between.  Replays of the kept
    executable graph must take nothing more."""
    cfg = CASES["nemotron_decode"] if name == "nemotron_decode" else MEDIUM.with_(tokens=300, seed=124)
    layer = synth.make_layer(cfg)
    mod = lmoe.LatentMoE(cfg, layer, max_tokens=cfg.tokens)
    try:
        x = layer["x"].cuda()
        y = torch.empty_like(x)
        lmoe.lmoe_set_graph_launch(mod.h, False)
        mod.forward(x, y)          # direct launches: loads the modules of every kernel the forward uses
        ref = y.clone()
        torch.cuda.synchronize()
        lmoe.lmoe_set_graph_launch(mod.h, True)
        free0, _ = torch.cuda.mem_get_info()
        mod.forward(x, y)          # captures, instantiates and launches the handle's first executable graph
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        for _ in range(5):
            mod.forward(x, y)      # updates the kept graph in place and launches it
        torch.cuda.synchronize()
        free2, _ = torch.cuda.mem_get_info()
        assert torch.equal(y, ref)
        assert mod.last_error() == 0
        took = free0 - free1
        warnings.warn(f"graph launch, {name}: first graph-launched forward took {took} bytes of device memory "
                      f"(free {free0} -> {free1}); five more forwards took {free1 - free2}")
        assert free2 == free1, "replays of the kept executable graph took device memory"
        assert took <= 32 << 20, f"graph instantiation took {took} bytes"
    finally:
        mod.close()
