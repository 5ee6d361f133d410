"""The expert-parallel exchange on CPU: gloo ranks on 127.0.0.1, no GPU.

``expert_parallel.ep_forward`` moves rows between the three stages of a
forward, and the stages themselves need a GPU. Here each rank instead drives an
fp64 stand-in for the stages:
* routing, weights and latent rows come from the oracle;
* the expert FFNs and the aggregation are plain fp64 arithmetic.

Every rank's output must equal the oracle's whole-layer output for its tokens
to fp64 rounding. A row sent to the wrong rank or expert, or returned to the
wrong slot, fails this by a wide margin. Rank counts 2 and 3; uneven token
counts; a rank with no tokens; skewed routing; MoE++ bypass experts and a
shared expert.  Both exchanges: the packed one (split sizes from the counts on
the host) and the block one (equal blocks, nothing read on the host; the
stand-in fills the unused rows of every block with NaN, so a row read from
outside a block's count poisons the output).
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as tdist
import torch.multiprocessing as mp

import oracle
from latent_mixture_experts_gemm_b200 import expert_parallel as xp
from latent_mixture_experts_gemm_b200 import synth

BASE = synth.LayerConfig(name="ep_cpu", tokens=0, d=128, latent=64, m=64, n_ffn=12, top_k=4, seed=81)
CASES = {
    "relu2": BASE,
    "swiglu_bypass_shared_skew": BASE.with_(act="swiglu", n_zero=1, n_copy=1, n_const=2, shared_m=64, zipf=1.2,
                                            seed=82),
    "standard_moe": BASE.with_(has_proj=0, latent=128, seed=83),
}


def _act(cfg, u: torch.Tensor) -> torch.Tensor:
    if cfg.act == synth.ACT_RELU2:
        return torch.clamp(u, min=0.0) ** 2
    if cfg.act == synth.ACT_SWIGLU:
        g, up = u[..., :cfg.m], u[..., cfg.m:]
        return g / (1.0 + torch.exp(-g)) * up
    return u


class OracleStages:
    """fp64 stand-in for the library's three stages on one rank (test only)."""

    def __init__(self, cfg, layer, ep, rank, max_tokens=0):
        self.cfg, self.layer, self.ep, self.rank = cfg, layer, ep, rank
        self.nl = cfg.n_ffn // ep
        self.block_rows = max_tokens * min(cfg.top_k, self.nl)  # block exchange: rows per rank pair
        f = lambda t: None if t is None else t.to(torch.float64)  # noqa: E731
        loc = xp.local_experts(layer, cfg.n_ffn, ep, rank)
        self.w1, self.w2 = f(loc["w1"]), f(loc["w2"])
        self.wu, self.cv = f(layer["w_up"]), f(layer["const_vecs"])
        self.ws1, self.ws2 = f(layer["w_shared1"]), f(layer["w_shared2"])
        self.seen_bounds = []

    def dispatch(self, x):
        cfg, K = self.cfg, self.cfg.top_k
        self.x = x
        T = int(x.shape[0])
        if T:
            r = oracle.forward(cfg, self.layer, x, want=("idx", "w", "z"))
            self.idx, self.w, z = r["idx"], r["w"], torch.from_numpy(r["z"])
        else:
            self.idx = np.zeros((0, K), np.int32)
            self.w = np.zeros((0, K))
            z = torch.zeros((0, cfg.latent), dtype=torch.float64)
        self.z = z
        flat = self.idx.reshape(-1)
        order = np.argsort(flat, kind="stable")          # slots by expert id, then token, then slot
        n_send = int(np.count_nonzero(flat < cfg.n_ffn))  # FFN ids sort first
        self.pos = np.empty_like(order)
        self.pos[order] = np.arange(order.size)
        send_rows = z[torch.from_numpy(order[:n_send] // K)] if n_send else torch.zeros((0, cfg.latent), dtype=torch.float64)
        counts = np.bincount(flat[flat < cfg.n_ffn], minlength=cfg.n_ffn).astype(np.int32)
        return send_rows.contiguous(), torch.from_numpy(counts)

    def recv_buffer(self, n):
        return torch.empty((n, self.cfg.latent), dtype=torch.float64)

    ret_buffer = recv_buffer

    def experts(self, recv_rows, recv_counts, n_recv, rows_bound):
        rc = recv_counts.view(self.ep, self.nl)
        assert int(rc.sum()) == n_recv == recv_rows.shape[0]
        assert rows_bound == int(rc.sum(0).max())
        self.seen_bounds.append(rows_bound)
        e_of_row = np.concatenate([np.repeat(np.arange(self.nl), rc[s].numpy()) for s in range(self.ep)])
        out = torch.empty_like(recv_rows)
        for e in np.unique(e_of_row):
            sel = torch.from_numpy(np.nonzero(e_of_row == e)[0])
            u = recv_rows[sel] @ self.w1[e].T
            out[sel] = _act(self.cfg, u) @ self.w2[e].T
        return out

    def combine(self, ret_rows, y):
        cfg, K = self.cfg, self.cfg.top_k
        T = int(self.x.shape[0])
        xf = self.x.to(torch.float64)
        yl = torch.zeros((T, cfg.latent), dtype=torch.float64)
        for t in range(T):
            for k in range(K):
                e = int(self.idx[t, k])
                if e < cfg.n_ffn:
                    o = ret_rows[self.pos[t * K + k]]
                elif e < cfg.n_ffn + cfg.n_zero:
                    o = torch.zeros(cfg.latent, dtype=torch.float64)
                elif e < cfg.n_ffn + cfg.n_zero + cfg.n_copy:
                    o = self.z[t]
                else:
                    o = self.cv[e - cfg.n_ffn - cfg.n_zero - cfg.n_copy]
                yl[t] += float(self.w[t, k]) * o
        out = xf + (yl @ self.wu.T if cfg.has_proj else yl)
        if cfg.shared_m:
            out = out + _act(cfg, xf @ self.ws1.T) @ self.ws2.T
        return out


    # ---- block exchange: the same arithmetic on rank blocks of block_rows rows
    def _blank(self):
        return torch.full((self.ep * self.block_rows, self.cfg.latent), float("nan"), dtype=torch.float64)

    def dispatch_blocks(self, x):
        send_rows, counts = self.dispatch(x)
        per = counts.view(self.ep, self.nl).sum(1).tolist()
        self.send_per = per
        blocks, off = self._blank(), 0
        for r, n in enumerate(per):
            assert n <= self.block_rows
            blocks[r * self.block_rows:r * self.block_rows + n] = send_rows[off:off + n]
            off += n
        return blocks, counts

    def recv_blocks(self):
        return self._blank()

    ret_blocks = recv_blocks

    def experts_blocks(self, recv_blocks, recv_counts):
        B = self.block_rows
        per = recv_counts.view(self.ep, self.nl).sum(1).tolist()
        rows = torch.cat([recv_blocks[s * B:s * B + n] for s, n in enumerate(per)])
        bound = int(recv_counts.view(self.ep, self.nl).sum(0).max())
        out_rows = self.experts(rows, recv_counts, int(sum(per)), bound)
        out, off = self._blank(), 0
        for s, n in enumerate(per):
            out[s * B:s * B + n] = out_rows[off:off + n]
            off += n
        return out

    def combine_blocks(self, ret_blocks, y):
        B = self.block_rows
        ret = torch.cat([ret_blocks[r * B:r * B + n] for r, n in enumerate(self.send_per)])
        return self.combine(ret, y)


def _tokens(cfg, ep):
    """Per-rank token counts: uneven, and with three ranks one rank has none."""
    return [13, 21] if ep == 2 else [17, 0, 9]


def _rank_main(rank, world, port, name, q, blocks=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg = CASES[name]
        layer = synth.make_layer(cfg, tokens=sum(_tokens(cfg, world)))
        T = _tokens(cfg, world)
        t0 = sum(T[:rank])
        x = layer["x"][t0:t0 + T[rank]]
        st = OracleStages(cfg, layer, world, rank, max_tokens=max(T))
        y = (xp.ep_forward_blocks if blocks else xp.ep_forward)(st, xp.AllToAll(), x)
        ref = oracle.forward(cfg, layer, x)["y"] if T[rank] else np.zeros((0, cfg.d))
        err = float(np.max(np.abs(y.numpy() - ref))) if T[rank] else 0.0
        q.put((rank, err, float(np.max(np.abs(ref))) if T[rank] else 1.0, st.seen_bounds))
        tdist.barrier()
    finally:
        tdist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("exchange", ["packed", "blocks"])
@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("name", list(CASES))
def test_exchange_over_gloo_ranks_matches_the_oracle(name, world, exchange):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, name, q, exchange == "blocks"))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, err, scale, bounds in res:
        assert err <= 1e-10 * scale, f"rank {rank}: max |y - oracle| = {err} (scale {scale})"
        assert len(bounds) == 1


@pytest.mark.parametrize("exchange", ["packed", "blocks"])
def test_one_rank_needs_no_process_group(exchange):
    cfg = CASES["swiglu_bypass_shared_skew"]
    layer = synth.make_layer(cfg, tokens=19)
    st = OracleStages(cfg, layer, 1, 0, max_tokens=19)
    ex = xp.AllToAll()
    assert ex.world == 1
    y = (xp.ep_forward_blocks if exchange == "blocks" else xp.ep_forward)(st, ex, layer["x"])
    ref = oracle.forward(cfg, layer)["y"]
    assert np.max(np.abs(y.numpy() - ref)) <= 1e-10 * np.max(np.abs(ref))


def test_split_plan_by_hand():
    # 2 ranks x 3 local experts: rows this rank sends to each rank's experts, rows it receives from each rank
    send = torch.tensor([[1, 0, 2], [4, 0, 0]], dtype=torch.int32)
    recv = torch.tensor([[1, 0, 2], [0, 5, 1]], dtype=torch.int32)
    in_s, out_s, n_send, n_recv, bound = xp.split_plan(send, recv, 2)
    assert in_s == [3, 4] and out_s == [3, 6]
    assert (n_send, n_recv) == (7, 9)
    assert bound == 5  # local expert 1: 0 + 5 rows; expert 2: 2 + 1; expert 0: 1 + 0
    _, _, _, n_recv, bound = xp.split_plan(torch.zeros(6, dtype=torch.int32), torch.zeros(6, dtype=torch.int32), 2)
    assert (n_recv, bound) == (0, 0)


def test_local_experts_slices_only_the_expert_weights():
    cfg = BASE
    layer = synth.make_layer(cfg, tokens=2)
    loc = xp.local_experts(layer, cfg.n_ffn, 3, 2)
    assert torch.equal(loc["w1"], layer["w1"][8:12]) and torch.equal(loc["w2"], layer["w2"][8:12])
    assert loc["w_router"] is layer["w_router"] and loc["w_down"] is layer["w_down"]
    with pytest.raises(ValueError):
        xp.local_experts(layer, cfg.n_ffn, 5, 0)
