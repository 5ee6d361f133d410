"""Expert parallelism on one GPU, through the C ABI.

* One rank: the three stages give exactly the output of ``lmoe_forward``, bit
  for bit, when called with the same expert-path threshold.
* Several ranks emulated on one GPU. Every rank runs its stages on its own
  handle, workspace, tokens and expert slice. The ranks run one stage at a time
  on one stream; tensor copies do the exchanges between stages. No kernel waits
  on another rank's kernel. Checks:
  * every rank's output meets the oracle's tolerances for its tokens;
  * with every expert on the grouped tensor-core GEMM, every rank's output is
    bit for bit the single-GPU forward of the same tokens. An expert row's
    result does not depend on which other rows share its tile.
* Counts that do not match the rows are reported as LMOE_ERR_BAD_COUNTS, and
  the stage then computes nothing; bad calls are rejected.
* The block exchange (every rank pair a fixed block of rows, the stages'
  ``*_blocks`` forms) gives the packed exchange's outputs bit for bit, on the
  same emulated ranks; with one rank it equals ``lmoe_forward``.
"""
import warnings

import numpy as np
import pytest
import torch

import oracle
from latent_mixture_experts_gemm_b200 import expert_parallel as xp
from latent_mixture_experts_gemm_b200 import lmoe, synth
from tests import _parity as P

pytestmark = pytest.mark.gpu

MEDIUM = synth.LayerConfig(name="ep_medium", tokens=0, d=512, latent=128, m=256, n_ffn=64, top_k=6, seed=91)
DECODE = synth.WORKLOADS["nemotron_decode"]

# name -> (layer shape, tokens per rank)
CASES = {
    "medium_4_ranks_ragged_empty": (MEDIUM, [300, 211, 0, 45]),
    "medium_2_ranks_swiglu_bypass_shared_skew": (
        MEDIUM.with_(act="swiglu", n_zero=1, n_copy=1, n_const=2, shared_m=128, zipf=1.1, seed=92), [257, 64]),
    "standard_moe_2_ranks": (MEDIUM.with_(has_proj=0, latent=512, seed=93), [100, 150]),
    "latent_router_2_ranks": (MEDIUM.with_(latent_router=1, seed=94), [130, 77]),
    # hundreds of rows per expert from both ranks: tiles mixing the ranks' rows, ragged ends
    "grouped_2_ranks_500_rows_per_expert": (MEDIUM.with_(n_ffn=16, top_k=4, seed=95), [1200, 900]),
    "decode_8_ranks_nemotron_shape": (DECODE.with_(seed=96), [16, 16, 9, 16, 1, 16, 16, 12]),
    "decode_2_ranks_one_token": (DECODE.with_(seed=97), [1, 1]),
}


def _split(layer, tokens):
    xs, t0 = [], 0
    for T in tokens:
        xs.append(layer["x"][t0:t0 + T])
        t0 += T
    return xs


def _emulated_forward(ranks, xs):
    """One forward of every rank: the stages in turn, the exchanges as copies on the device."""
    N = len(ranks)
    nl = ranks[0].cfg.n_ffn // N
    sends = [r.dispatch(x.cuda()) for r, x in zip(ranks, xs)]
    sc = torch.stack([c for _, c in sends]).cpu().view(N, N, nl).to(torch.int64)  # [source, destination, expert]
    per = sc.sum(2)                                                               # rows source -> destination
    outs = []
    for r in range(N):
        rc = sc[:, r, :]
        n_recv = int(rc.sum())
        bound = int(rc.sum(0).max())
        buf = ranks[r].recv_buffer(n_recv)
        if n_recv:
            torch.cat([sends[s][0][int(per[s, :r].sum()):int(per[s, :r + 1].sum())] for s in range(N)], out=buf)
        outs.append(ranks[r].experts(buf, rc.to(torch.int32).contiguous().cuda(), n_recv, bound))
    ys = []
    for s in range(N):
        n_send = int(per[s].sum())
        ret = ranks[s].ret_buffer(n_send)
        if n_send:
            torch.cat([outs[r][int(per[:s, r].sum()):int(per[:s + 1, r].sum())] for r in range(N)], out=ret)
        ys.append(ranks[s].combine(ret))
    return ys


def _emulated_forward_blocks(ranks, xs):
    """The same forward with the block exchange: block r of rank s's send blocks becomes block s of rank r's
    receive blocks, and back; no count is read on the host."""
    N = len(ranks)
    nl = ranks[0].cfg.n_ffn // N
    B = ranks[0].block_rows
    sends = [r.dispatch_blocks(x.cuda()) for r, x in zip(ranks, xs)]
    outs = []
    for r in range(N):
        recv = ranks[r].recv_blocks()
        for s in range(N):
            recv[s * B:(s + 1) * B].copy_(sends[s][0][r * B:(r + 1) * B])
        rc = torch.stack([sends[s][1][r * nl:(r + 1) * nl] for s in range(N)]).contiguous()
        outs.append(ranks[r].experts_blocks(recv, rc))
    ys = []
    for s in range(N):
        ret = ranks[s].ret_blocks()
        for r in range(N):
            ret[r * B:(r + 1) * B].copy_(outs[r][s * B:(s + 1) * B])
        ys.append(ranks[s].combine_blocks(ret))
    return ys


def _make_ranks(cfg, layer, tokens, small_rows=None):
    N = len(tokens)
    ranks = [xp.ExpertParallelLatentMoE(cfg, layer, max_tokens=max(max(tokens), 1), ep_size=N, ep_rank=r)
             for r in range(N)]
    if small_rows is not None:
        for r in ranks:
            lmoe.lmoe_set_small_rows(r.mod.h, small_rows)
    return ranks


def _close(objs):
    for o in objs:
        o.close()


@pytest.mark.parametrize("name", list(CASES))
def test_emulated_ranks_match_the_oracle(name):
    cfg, tokens = CASES[name]
    layer = synth.make_layer(cfg, tokens=sum(tokens))
    xs = _split(layer, tokens)
    ranks = _make_ranks(cfg, layer, tokens)
    single = lmoe.LatentMoE(cfg, layer, max_tokens=max(max(tokens), 1))
    try:
        ys = _emulated_forward(ranks, xs)
        torch.cuda.synchronize()
        for r, (x, y) in enumerate(zip(xs, ys)):
            assert ranks[r].last_error() == 0
            if x.shape[0] == 0:
                assert y.shape[0] == 0
                continue
            # the single-GPU forward of the same tokens routes them exactly as this rank's dispatch does
            # (same kernels on the same inputs): its ids settle the oracle's near ties
            _, dbg = single.forward(x.cuda(), debug=True)
            torch.cuda.synchronize()
            gidx, gw = dbg["idx"].cpu().numpy(), dbg["w"].cpu().numpy()
            ref = oracle.forward(cfg, layer, x=x, want=("y", "idx", "w", "logits"))
            differ = P.check_routing(gidx, gw, ref, cfg.top_k, w_atol=2e-5)
            if differ.any():
                ref2 = oracle.forward(cfg, layer, x=x, idx=gidx, want=("y",))
                ref["y"] = np.where(differ[:, None], ref2["y"], ref["y"])
            got = P.to_np(y)
            m = P.metrics(got, ref["y"])
            emulated = None
            if m["max_err"] > P.MAX_ERR_VS_RMS * m["rms_ref"]:
                emulated = P.emulate_bf16(cfg, layer, x, gidx, gw)
            m = P.assert_layer_close(got, ref["y"], emulated, f"rank {r} y")
            if "bf16_storage_max_err" in m:
                warnings.warn(f"bf16-storage allowance used by {name} rank {r}: max_err {m['max_err']:.4g}; "
                              f"bf16 storage alone {m['bf16_storage_max_err']:.4g}")
    finally:
        _close(ranks + [single])


@pytest.mark.parametrize("name", ["medium_4_ranks_ragged_empty", "medium_2_ranks_swiglu_bypass_shared_skew",
                                  "grouped_2_ranks_500_rows_per_expert", "decode_8_ranks_nemotron_shape"])
def test_emulated_ranks_bit_identical_to_single_gpu_on_the_grouped_gemm(name):
    cfg, tokens = CASES[name]
    layer = synth.make_layer(cfg, tokens=sum(tokens))
    xs = _split(layer, tokens)
    ranks = _make_ranks(cfg, layer, tokens, small_rows=0)
    single = lmoe.LatentMoE(cfg, layer, max_tokens=max(max(tokens), 1))
    lmoe.lmoe_set_small_rows(single.h, 0)
    try:
        ys = _emulated_forward(ranks, xs)
        for r, (x, y) in enumerate(zip(xs, ys)):
            if x.shape[0]:
                ref = single.forward(x.cuda())
                torch.cuda.synchronize()
                assert torch.equal(y, ref), f"rank {r}: {(y.float() - ref.float()).abs().max().item()}"
        assert all(rk.last_error() == 0 for rk in ranks)
    finally:
        _close(ranks + [single])


@pytest.mark.parametrize("name,T", [("medium", 300), ("medium", 29), ("swiglu_bypass_shared", 77),
                                    ("standard_moe", 40), ("decode", 32)])
def test_one_rank_stages_bit_identical_to_forward(name, T):
    cfg = {"medium": MEDIUM, "swiglu_bypass_shared": CASES["medium_2_ranks_swiglu_bypass_shared_skew"][0],
           "standard_moe": CASES["standard_moe_2_ranks"][0], "decode": DECODE.with_(seed=98)}[name]
    layer = synth.make_layer(cfg, tokens=T)
    mod = lmoe.LatentMoE(cfg, layer, max_tokens=T)
    try:
        x = layer["x"].cuda()
        ref = mod.forward(x)
        K, L = cfg.top_k, cfg.latent
        rows = torch.empty((T * K, L), dtype=torch.bfloat16, device="cuda")
        counts = torch.empty(cfg.n_ffn, dtype=torch.int32, device="cuda")
        lmoe.lmoe_ep_dispatch(mod.h, x, rows, counts)
        n = int(counts.sum())
        # rows_bound = T: the threshold lmoe_forward derives from T
        lmoe.lmoe_ep_experts(mod.h, rows, counts, n, T, rows)
        y = torch.empty_like(x)
        lmoe.lmoe_ep_combine(mod.h, rows, y)
        torch.cuda.synchronize()
        assert mod.last_error() == 0
        assert torch.equal(y, ref)
        # and ep_forward with one rank (no process group, the exact bound) meets the same tolerance
        one = xp.ExpertParallelLatentMoE(cfg, layer, max_tokens=T, ep_size=1, ep_rank=0)
        try:
            y1 = one.forward(x)
            torch.cuda.synchronize()
            assert one.last_error() == 0
            P.assert_close(P.to_np(y1), P.to_np(ref), "ep_forward vs forward", max_vs_rms=1e-2, mean_rel=1e-3)
        finally:
            one.close()
    finally:
        mod.close()


@pytest.mark.parametrize("name", ["medium_4_ranks_ragged_empty", "medium_2_ranks_swiglu_bypass_shared_skew",
                                  "standard_moe_2_ranks", "latent_router_2_ranks", "decode_8_ranks_nemotron_shape",
                                  "decode_2_ranks_one_token"])
def test_block_exchange_equals_the_packed_exchange(name):
    cfg, tokens = CASES[name]
    layer = synth.make_layer(cfg, tokens=sum(tokens))
    xs = _split(layer, tokens)
    ranks = _make_ranks(cfg, layer, tokens)
    try:
        assert all(r.block_exchange for r in ranks)
        packed = _emulated_forward(ranks, xs)
        blocks = _emulated_forward_blocks(ranks, xs)
        torch.cuda.synchronize()
        for r, (a, b) in enumerate(zip(packed, blocks)):
            assert torch.equal(a, b), f"rank {r}: {(a.float() - b.float()).abs().max().item()}"
        assert all(rk.last_error() == 0 for rk in ranks)
    finally:
        _close(ranks)


@pytest.mark.parametrize("T", [32, 5])
def test_one_rank_block_exchange_equals_forward(T):
    """One rank, the decode shape: the block stages (no host read of any count) give lmoe_forward's output
    bit for bit when the expert-path threshold matches (rows_bound = T)."""
    cfg = DECODE.with_(seed=99)
    layer = synth.make_layer(cfg, tokens=T)
    mod = lmoe.LatentMoE(cfg, layer, max_tokens=T)
    try:
        x = layer["x"].cuda()
        ref = mod.forward(x)
        B = lmoe.lmoe_ep_block_rows(mod.h)
        assert B == T * cfg.top_k
        blocks = torch.empty((B, cfg.latent), dtype=torch.bfloat16, device="cuda")
        counts = torch.empty(cfg.n_ffn, dtype=torch.int32, device="cuda")
        lmoe.lmoe_ep_dispatch_blocks(mod.h, x, blocks, B, counts)
        lmoe.lmoe_ep_experts_blocks(mod.h, blocks, B, counts, T, blocks)
        y = torch.empty_like(x)
        lmoe.lmoe_ep_combine_blocks(mod.h, blocks, y)
        torch.cuda.synchronize()
        assert mod.last_error() == 0
        assert torch.equal(y, ref)
        # the stages of the two exchanges do not mix within a forward
        lmoe.lmoe_ep_dispatch_blocks(mod.h, x, blocks, B, counts)
        with pytest.raises(lmoe.LmoeError):
            lmoe.lmoe_ep_combine(mod.h, blocks, y)
        lmoe.lmoe_ep_combine_blocks(mod.h, blocks, y)
        with pytest.raises(lmoe.LmoeError):  # a block smaller than T * min(K', n_local)
            lmoe.lmoe_ep_dispatch_blocks(mod.h, x, blocks, B - 1, counts)
        torch.cuda.synchronize()
    finally:
        mod.close()


def test_block_counts_over_the_block_are_reported():
    cfg = MEDIUM
    layer = synth.make_layer(cfg, tokens=4)
    rk = xp.ExpertParallelLatentMoE(cfg, layer, max_tokens=4, ep_size=2, ep_rank=1)  # 32 local experts
    try:
        B = rk.block_rows                         # 4 tokens x min(6, 32) = 24
        assert B == 24
        blocks = torch.zeros((2 * B, cfg.latent), dtype=torch.bfloat16, device="cuda")
        counts = torch.zeros(64, dtype=torch.int32)  # [2 sources][32 local experts]; rows_bound 2 x 4 = 8
        counts[0:3] = 8
        counts[3] = 1                             # source 0 sends 25 rows: more than its block
        rk.experts_blocks(blocks, counts.cuda())
        torch.cuda.synchronize()
        assert rk.last_error() == -8               # LMOE_ERR_BAD_COUNTS
        counts[3] = 0                             # 24 rows: fits
        rk.experts_blocks(blocks, counts.cuda())
        torch.cuda.synchronize()
        assert rk.last_error() == 0
    finally:
        rk.close()


def test_inconsistent_counts_are_reported_and_compute_nothing():
    cfg = MEDIUM
    layer = synth.make_layer(cfg, tokens=4)
    rk = xp.ExpertParallelLatentMoE(cfg, layer, max_tokens=16, ep_size=2, ep_rank=1)  # 32 local experts
    try:
        g = torch.Generator().manual_seed(5)
        rows = torch.randn((40, cfg.latent), generator=g).to(torch.bfloat16).cuda()
        good = torch.zeros(64, dtype=torch.int32)  # [2 sources][32 local experts], 40 rows
        good[torch.tensor([0, 5, 31, 32, 40])] = torch.tensor([7, 3, 10, 12, 8], dtype=torch.int32)
        c1 = good.clone()
        c1[5] = 4                      # sums to 41, not 40
        c2 = good.clone()
        c2[5] = -1
        c2[0] = 11                     # sums to 40 with a negative count
        for counts, n, bound in ((c1, 40, 40), (c2, 40, 40), (good, 40, 12)):  # last: expert 0 gets 19 > 12
            buf = rows.clone()
            lmoe.lmoe_ep_experts(rk.mod.h, buf, counts.cuda(), n, bound, buf)
            torch.cuda.synchronize()
            assert rk.last_error() == -8, (counts, n, bound)
            assert torch.equal(buf, rows)
        # the handle stays usable: consistent counts compute every row
        buf = rows.clone()
        lmoe.lmoe_ep_experts(rk.mod.h, buf, good.cuda(), 40, 19, buf)
        torch.cuda.synchronize()
        assert rk.last_error() == 0
        assert not torch.equal(buf, rows)
        # expert 32 + 0 of this rank (global 32) on its 7 rows from source 0: o = W2 relu(W1 z)^2
        w1 = layer["w1"][32].double()
        w2 = layer["w2"][32].double()
        z = rows[:7].cpu().double()
        ref = (torch.clamp(z @ w1.T, min=0) ** 2) @ w2.T
        P.assert_close(P.to_np(buf[:7]), ref.numpy(), "expert rows")
    finally:
        rk.close()


def test_bad_calls_are_rejected():
    cfg = MEDIUM
    layer = synth.make_layer(cfg, tokens=8)
    rk = xp.ExpertParallelLatentMoE(cfg, layer, max_tokens=8, ep_size=2, ep_rank=0)
    try:
        x = layer["x"].cuda()
        y = torch.empty_like(x)
        h = rk.mod.h
        L = lmoe.lib()
        # a rank's handle holds only its experts: the one-call forward is refused
        assert L.lmoe_forward(h, x.data_ptr(), y.data_ptr(), 8, None, None) == -1
        # combine before any dispatch
        assert L.lmoe_ep_combine(h, rk.ret_rows.data_ptr(), y.data_ptr(), None) == -1
        cap = 2 * 8 * 6
        counts = torch.zeros(64, dtype=torch.int32, device="cuda")
        assert L.lmoe_ep_experts(h, rk.recv_rows.data_ptr(), counts.data_ptr(), cap + 1, 1, rk.recv_rows.data_ptr(),
                                 None) == -3
        assert L.lmoe_ep_experts(h, rk.recv_rows.data_ptr(), counts.data_ptr(), 5, 0, rk.recv_rows.data_ptr(),
                                 None) == -1
        assert L.lmoe_ep_experts(h, rk.recv_rows.data_ptr(), counts.data_ptr(), 0, 0, None, None) == 0
        assert L.lmoe_ep_dispatch(h, x.data_ptr(), 9, rk.send_rows.data_ptr(), rk.send_counts.data_ptr(), None) == -3
        # dispatch with x and y overlapping in combine
        rk.dispatch(x)
        assert L.lmoe_ep_combine(h, rk.ret_rows.data_ptr(), x.data_ptr(), None) == -1
        torch.cuda.synchronize()
        assert rk.last_error() == 0
    finally:
        rk.close()
    # block-scaled handles have no expert-parallel stages
    mx = synth.WORKLOADS["tiny"].with_(expert_fmt=1, latent=128, m=128, tokens=4)
    mod = lmoe.LatentMoE(mx, synth.make_layer(mx), max_tokens=4)
    try:
        x = torch.zeros((4, mx.d), dtype=torch.bfloat16, device="cuda")
        rows = torch.empty((4 * mx.top_k, mx.latent), dtype=torch.bfloat16, device="cuda")
        counts = torch.empty(mx.n_ffn, dtype=torch.int32, device="cuda")
        with pytest.raises(lmoe.LmoeError) as e:
            lmoe.lmoe_ep_dispatch(mod.h, x, rows, counts)
        assert e.value.status == -2
    finally:
        mod.close()
