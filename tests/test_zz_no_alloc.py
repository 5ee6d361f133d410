"""The allocation-free expert sort (lmoe_dispatch_noalloc), through the C ABI.

lmoe_dispatch_noalloc is for callers that cannot allocate device memory (a
plugin whose host framework owns the device-memory budget, a loop that cannot
take cudaMalloc's implicit synchronisation), so cannot hand the library a
workspace: it keeps its scratch in a fixed device array inside the library.

* Against the layer's own dispatch: lmoe_forward routes tokens (its debug
  outputs copy out the counts, offsets and permutation of its dispatch step),
  then lmoe_dispatch_noalloc sorts the same ids, twice in a row on different
  batches, so the second call runs on the scratch the first one left behind.
* Against the oracle's stable counting sort, on ids drawn here: the largest
  batch the scratch holds (8192 tokens, 1024 experts, top-32), ragged and
  single-token batches, and an empty batch, back to back on the shared scratch.
* Ids outside [0, n_total) are skipped and reported in the error word; the
  valid slots still sort as the oracle sorts them.  A row that names one expert
  twice is reported, and no write leaves the caller's buffers.

Integer results: compared bit for bit.  This file is collected last so that, in
a run stopping at the first failure, every other test has run; it also passes
on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import oracle
from latent_mixture_experts_gemm_b200 import lmoe, synth

pytestmark = pytest.mark.gpu

GUARD = 64  # sentinel elements past the end of every output buffer


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
    """One call into buffers filled with -1, each with GUARD sentinels past its end."""
    T, K = idx.shape
    full = lambda n: torch.full((n + GUARD,), -1, dtype=torch.int32, device="cuda")  # noqa: E731
    bufs = {"counts": full(n_total), "offsets": full(n_total + 1), "perm": full(T * K), "inv": full(T * K),
            "err": torch.full((1,), -7, dtype=torch.int32, device="cuda")}
    lmoe.lmoe_dispatch_noalloc(idx, n_total, bufs["counts"], bufs["offsets"], bufs["perm"], bufs["inv"], bufs["err"])
    return bufs


def _host(bufs, T, K, n_total):
    """The outputs as numpy, after checking that the sentinels past every buffer's end are untouched."""
    sizes = {"counts": n_total, "offsets": n_total + 1, "perm": T * K, "inv": T * K}
    out = {}
    for k, n in sizes.items():
        a = bufs[k].cpu().numpy()
        assert np.all(a[n:] == -1), f"{k}: written past its end"
        out[k] = a[:n]
    out["err"] = int(bufs["err"].item())
    return out


def _distinct_ids(T, K, n_total, seed, skew=0.0):
    """[T, K] int32 expert ids, distinct within each row (a top-K selection of random scores, with an
    optional per-expert Zipf-like bias that concentrates the load on a few experts)."""
    g = torch.Generator().manual_seed(seed)
    scores = torch.rand(T, n_total, generator=g)
    if skew:
        ranks = torch.randperm(n_total, generator=g).double() + 1.0
        scores = scores.double() - skew * torch.log(ranks) * 0.1
    return scores.topk(K, dim=1).indices.to(torch.int32)


def test_noalloc_dispatch_matches_the_layer_dispatch_on_two_calls_in_a_row():
    # a prefill-sized batch of a 64-expert top-6 layer, then a ragged small batch of the Kimi-like shape
    # (908 routed experts incl. bypass experts, top-16) that reuses the scratch the first call wrote
    big = synth.LayerConfig(name="sort_big", d=512, latent=128, m=256, n_ffn=64, top_k=6, tokens=3000, seed=41)
    small = synth.LayerConfig(name="sort_small", d=512, latent=128, m=128, n_ffn=896, n_zero=4, n_copy=4, n_const=4,
                              top_k=16, act=synth.ACT_SWIGLU, zipf=1.1, tokens=77, seed=42)
    for cfg in (big, small):
        ref = _routes(cfg, cfg.tokens, cfg.seed)
        got = _host(_noalloc(ref["idx"], cfg.n_total), cfg.tokens, cfg.top_k, cfg.n_total)
        torch.cuda.synchronize()
        for k in ("counts", "offsets", "perm"):
            assert np.array_equal(got[k], ref[k].cpu().numpy()), f"{cfg.name}: {k} differs"
        assert np.array_equal(got["inv"][got["perm"]], np.arange(got["perm"].size))
        assert got["err"] == 0


@pytest.mark.parametrize("shape", [(8192, 32, 1024, 0.0), (8192, 22, 512, 1.1), (4097, 16, 908, 1.1),
                                   (3000, 6, 64, 0.0), (33, 32, 32, 0.0), (1, 1, 1, 0.0), (1, 4, 1024, 0.0)],
                         ids=lambda s: f"T{s[0]}_K{s[1]}_N{s[2]}" + ("_skew" if s[3] else ""))
def test_noalloc_dispatch_matches_the_oracle(shape):
    """Two calls in a row on different ids (the second on the scratch the first left behind), each
    against the oracle's stable counting sort."""
    T, K, n_total, skew = shape
    for seed in (1, 2):
        idx = _distinct_ids(T, K, n_total, seed=100 * T + seed, skew=skew)
        got = _host(_noalloc(idx.cuda(), n_total), T, K, n_total)
        c, o, p, i = oracle.dispatch(idx.numpy(), n_total)
        assert got["err"] == 0
        assert np.array_equal(got["counts"], c)
        assert np.array_equal(got["offsets"], o)
        assert np.array_equal(got["perm"], p)
        assert np.array_equal(got["inv"], i)


def test_noalloc_dispatch_of_an_empty_batch_zeroes_counts_and_offsets():
    # a full batch first leaves non-zero scratch behind
    _host(_noalloc(_distinct_ids(500, 8, 40, seed=3).cuda(), 40), 500, 8, 40)
    bufs = _noalloc(torch.empty((0, 8), dtype=torch.int32, device="cuda"), 40)
    got = _host(bufs, 0, 8, 40)
    assert np.all(got["counts"] == 0) and np.all(got["offsets"] == 0) and got["err"] == 0


def test_noalloc_dispatch_skips_and_reports_out_of_range_ids():
    T, K, n_total = 700, 6, 50
    idx = _distinct_ids(T, K, n_total, seed=4).numpy()
    rng = np.random.default_rng(5)
    bad = rng.choice(T * K, size=37, replace=False)
    flat = idx.reshape(-1)
    flat[bad[::2]] = -1
    flat[bad[1::2]] = n_total
    got = _host(_noalloc(torch.from_numpy(idx).cuda(), n_total), T, K, n_total)
    assert got["err"] & lmoe.LMOE_DEVERR_BAD_INDEX
    assert not got["err"] & lmoe.LMOE_DEVERR_REPEATED_INDEX
    # the valid slots sort as the oracle sorts them with the bad ids moved to one extra, last expert
    remapped = np.where((idx < 0) | (idx >= n_total), n_total, idx).astype(np.int32)
    c, o, p, i = oracle.dispatch(remapped, n_total + 1)
    valid = T * K - bad.size
    assert np.array_equal(got["counts"], c[:n_total])
    assert np.array_equal(got["offsets"], o[:n_total + 1]) and got["offsets"][n_total] == valid
    assert np.array_equal(got["perm"][:valid], p[:valid])
    assert np.all(got["perm"][valid:] == -1)
    ok = np.ones(T * K, bool)
    ok[bad] = False
    assert np.array_equal(got["inv"][ok], i[ok])
    assert np.all(got["inv"][~ok] == -1)
    # the next call on clean ids reports nothing: the error bits are this call's only
    clean = _distinct_ids(T, K, n_total, seed=6)
    got2 = _host(_noalloc(clean.cuda(), n_total), T, K, n_total)
    assert got2["err"] == 0


@pytest.mark.parametrize("T", [40, 5000])
def test_noalloc_dispatch_reports_a_repeated_id_in_a_row(T):
    K, n_total = 4, 30
    idx = _distinct_ids(T, K, n_total, seed=7)
    idx[T // 2, 3] = idx[T // 2, 1]
    got = _host(_noalloc(idx.cuda(), n_total), T, K, n_total)   # also checks that nothing lands past the buffers
    assert got["err"] & lmoe.LMOE_DEVERR_REPEATED_INDEX
    assert np.all((got["perm"] >= -1) & (got["perm"] < T * K))
    assert np.all((got["inv"] >= -1) & (got["inv"] < T * K))


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
