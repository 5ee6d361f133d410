"""The allocation-free expert sort (lmoe_dispatch_noalloc) against the layer's own dispatch.

lmoe_dispatch_noalloc is for callers that cannot allocate device memory, so
cannot hand the library a workspace: it keeps its scratch in a fixed device
array inside the library.  This test routes tokens with lmoe_forward (whose
debug outputs copy out the counts, offsets and permutation its dispatch step
produced), then sorts the same expert ids with lmoe_dispatch_noalloc, twice in a
row on different batches so the second call runs on the scratch the first one
left behind.  Integer results: compared bit for bit.  This file is collected
last so that, in a run stopping at the first failure, every other test has run.
"""
import numpy as np
import pytest
import torch

from latent_mixture_experts_gemm_b200 import lmoe, synth

pytestmark = pytest.mark.gpu


def _routes(cfg, tokens, seed):
    layer = synth.make_layer(cfg, tokens=tokens, seed=seed)
    mod = lmoe.LatentMoE(cfg, layer, max_tokens=tokens)
    try:
        _, dbg = mod.forward(layer["x"].cuda(), debug=True)
        torch.cuda.synchronize()
        assert mod.last_error() == 0
        return {k: dbg[k].clone() for k in ("idx", "counts", "offsets", "perm")}
    finally:
        mod.close()


def _noalloc(idx, n_total):
    T, K = idx.shape
    out = {"counts": torch.full((n_total,), -1, dtype=torch.int32, device="cuda"),
           "offsets": torch.full((n_total + 1,), -1, dtype=torch.int32, device="cuda"),
           "perm": torch.full((T * K,), -1, dtype=torch.int32, device="cuda"),
           "inv": torch.full((T * K,), -1, dtype=torch.int32, device="cuda")}
    lmoe.lmoe_dispatch_noalloc(idx, n_total, out["counts"], out["offsets"], out["perm"], out["inv"])
    return out


def test_noalloc_dispatch_matches_the_layer_dispatch_on_two_calls_in_a_row():
    # a prefill-sized batch of a 64-expert top-6 layer, then a ragged small batch of the Kimi-like shape
    # (908 routed experts incl. bypass experts, top-16) that reuses the scratch the first call wrote
    big = synth.LayerConfig(name="sort_big", d=512, latent=128, m=256, n_ffn=64, top_k=6, tokens=3000, seed=41)
    small = synth.LayerConfig(name="sort_small", d=512, latent=128, m=128, n_ffn=896, n_zero=4, n_copy=4, n_const=4,
                              top_k=16, act=synth.ACT_SWIGLU, zipf=1.1, tokens=77, seed=42)
    for cfg in (big, small):
        ref = _routes(cfg, cfg.tokens, cfg.seed)
        got = _noalloc(ref["idx"], cfg.n_total)
        torch.cuda.synchronize()
        for k in ("counts", "offsets", "perm"):
            assert torch.equal(got[k], ref[k]), f"{cfg.name}: {k} differs"
        perm = got["perm"].cpu().numpy()
        inv = got["inv"].cpu().numpy()
        assert np.array_equal(inv[perm], np.arange(perm.size))


def test_noalloc_dispatch_rejects_sizes_beyond_its_scratch():
    idx = torch.zeros((8193, 1), dtype=torch.int32, device="cuda")
    buf = torch.empty(8193, dtype=torch.int32, device="cuda")
    with pytest.raises(lmoe.LmoeError) as e:
        lmoe.lmoe_dispatch_noalloc(idx, 4, buf, buf, buf, buf)
    assert e.value.status == -3
    idx2 = torch.zeros((4, 2), dtype=torch.int32, device="cuda")
    with pytest.raises(lmoe.LmoeError) as e:
        lmoe.lmoe_dispatch_noalloc(idx2, 1025, buf, buf, buf, buf)
    assert e.value.status == -2
