"""Expert parallelism for the LatentMoE layer: one process per GPU, each rank
holding ``n_ffn / ep_size`` of the FFN experts.

The pages place an all-to-all between routing and the experts and another one
back before the aggregation. In LatentMoE both carry latent-wide rows, so the
volume scales with the latent width rather than with d. Sources:
* Kimi K3 / Nemotron 3 Super article, "MoE 遇到了什么问题？";
* Nemotron-3 article, section 2.2.

Every step of the layer runs in the CUDA library's three stages:
* ``lmoe_ep_dispatch``: router, W_down, top-K', counting sort; the rows come
  out grouped by destination rank;
* ``lmoe_ep_experts``: this rank's experts on the rows it received;
* ``lmoe_ep_combine``: aggregation in the latent width, W_up, residual.

This module only moves rows between them with ``torch.distributed``: NCCL over
NVLink on GPUs, gloo on CPU in the tests. One forward on one rank:

1. dispatch;
2. all-to-all of the per-expert counts (``n_ffn`` int32 per rank);
3. one device-to-host copy of the send and receive counts, for the split sizes;
4. all-to-all of the rows;
5. experts;
6. the reverse all-to-all of the expert outputs;
7. combine.

The block exchange (``ep_forward_blocks``, the ``*_blocks`` stages) gives every
pair of ranks a fixed block of rows, so the all-to-alls have equal splits known
before the forward and step 3 disappears: no forward waits on the device. The
blocks carry unused rows, so it is the exchange for decode-size batches;
``ExpertParallelLatentMoE`` takes it when the blocks of one forward are small
(``block_limit_bytes``).
"""
from __future__ import annotations

from typing import Dict, List, Optional, Tuple

import numpy as np
import torch
import torch.distributed as dist

from . import lmoe


def split_plan(send_counts, recv_counts, ep: int) -> Tuple[List[int], List[int], int, int, int]:
    """Host-side sizes of one exchange.

    The inputs are the count matrices ``[ep, n_local]`` on the host (CPU
    tensors or arrays, any shape of ep * n_local entries): what this
    rank sends to each rank's experts, and what each rank sends to this rank's
    experts. Returns a tuple of:
    * ``in_splits``: rows sent to each rank;
    * ``out_splits``: rows received from each rank;
    * ``n_send``, ``n_recv``: their totals;
    * ``rows_bound``: the most rows any local expert receives.
    """
    sc = np.asarray(send_counts, dtype=np.int64).reshape(ep, -1)
    rc = np.asarray(recv_counts, dtype=np.int64).reshape(ep, -1)
    in_splits = sc.sum(1).tolist()
    out_splits = rc.sum(1).tolist()
    rows_bound = int(rc.sum(0).max()) if rc.size else 0
    return in_splits, out_splits, sum(in_splits), sum(out_splits), rows_bound


class AllToAll:
    """The two exchanges of a forward over a process group.

    With one rank nothing moves: the exchange returns its input.
    """

    def __init__(self, group=None):
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1

    def counts(self, send_counts: torch.Tensor) -> torch.Tensor:
        """All-to-all of the per-expert counts, ``n_local`` entries to each rank."""
        if self.world == 1:
            return send_counts
        out = torch.empty_like(send_counts)
        dist.all_to_all_single(out, send_counts, group=self.group)
        return out

    def blocks(self, out: torch.Tensor, inp: torch.Tensor) -> torch.Tensor:
        """All-to-all of equal blocks: block r of ``inp`` goes to rank r, and block s of ``out`` comes from
        rank s.  No split sizes: nothing has to be known on the host."""
        if self.world == 1:
            return inp
        dist.all_to_all_single(out, inp, group=self.group)
        return out

    def rows(self, out: torch.Tensor, inp: torch.Tensor, out_splits: List[int], in_splits: List[int]) -> torch.Tensor:
        """All-to-all of rows. ``in_splits[r]`` rows of ``inp`` go to rank r. ``out[...]`` receives
        ``out_splits[s]`` rows from each rank s, in rank order."""
        if self.world == 1:
            return inp
        dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)
        return out


def ep_forward(stages, exchange, x: torch.Tensor, y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One expert-parallel forward of ``x`` on this rank.

    ``stages`` provides:
    * ``dispatch(x) -> (send_rows, send_counts)``;
    * ``recv_buffer(n)`` and ``ret_buffer(n)``;
    * ``experts(recv_rows, recv_counts, n_recv, rows_bound) -> out_rows``;
    * ``combine(ret_rows, y) -> y``.

    ``exchange`` is an :class:`AllToAll`.
    """
    send_rows, send_counts = stages.dispatch(x)
    recv_counts = exchange.counts(send_counts)
    n = send_counts.numel()
    both = send_counts if recv_counts is send_counts else torch.cat([send_counts, recv_counts])
    host = both.cpu().numpy()  # the forward's one wait on the device
    in_splits, out_splits, n_send, n_recv, rows_bound = split_plan(host[:n], host[-n:], exchange.world)
    recv = exchange.rows(stages.recv_buffer(n_recv), send_rows[:n_send], out_splits, in_splits)
    out = stages.experts(recv, recv_counts, n_recv, rows_bound)
    ret = exchange.rows(stages.ret_buffer(n_send), out, in_splits, out_splits)
    return stages.combine(ret, y)


def ep_forward_blocks(stages, exchange, x: torch.Tensor, y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One expert-parallel forward of ``x`` on this rank with the block exchange: the same steps as
    ``ep_forward``, every rank pair moving a fixed block of rows, and no device-to-host copy.

    ``stages`` provides ``dispatch_blocks(x) -> (send_blocks, send_counts)``, ``recv_blocks()``,
    ``ret_blocks()``, ``experts_blocks(recv_blocks, recv_counts) -> out_blocks`` and
    ``combine_blocks(ret_blocks, y) -> y``.
    """
    send_blocks, send_counts = stages.dispatch_blocks(x)
    recv_counts = exchange.counts(send_counts)
    recv = exchange.blocks(stages.recv_blocks(), send_blocks)
    out = stages.experts_blocks(recv, recv_counts)
    ret = exchange.blocks(stages.ret_blocks(), out)
    return stages.combine_blocks(ret, y)


def local_experts(layer: Dict[str, torch.Tensor], n_ffn: int, ep_size: int, ep_rank: int) -> Dict[str, torch.Tensor]:
    """The layer's tensors as rank ``ep_rank`` holds them.

    W1 and W2 keep only the rank's ``n_ffn / ep_size`` experts. Every other
    tensor is whole.
    """
    if n_ffn % ep_size:
        raise ValueError(f"{n_ffn} FFN experts do not split over {ep_size} ranks")
    n_local = n_ffn // ep_size
    out = dict(layer)
    for k in ("w1", "w2"):
        out[k] = layer[k][ep_rank * n_local:(ep_rank + 1) * n_local]
    return out


class ExpertParallelLatentMoE:
    """One rank of an expert-parallel LatentMoE layer on this process's GPU.

    ``layer`` holds the whole layer, from which the rank keeps its own experts.
    The exchange buffers are allocated once, for ``max_tokens`` tokens on
    every rank:
    * ``send_rows`` and ``ret_rows``: ``[max_tokens * top_k, latent]``;
    * ``recv_rows``: ``[ep_size * max_tokens * min(top_k, n_local), latent]``,
      the most rows this rank's experts can receive.

    The experts stage writes its outputs over the received rows.

    With the block exchange (taken when ``ep_size * block_rows`` latent rows are at most
    ``block_limit_bytes``, block_rows = ``max_tokens * min(top_k, n_local)``) there are also
    ``send_blocks`` and ``ret_blocks`` of ``[ep_size * block_rows, latent]``; ``recv_rows`` has that size
    already.
    """

    def __init__(self, cfg, layer: Dict[str, torch.Tensor], max_tokens: int, ep_size: int, ep_rank: int,
                 device: str = "cuda", group=None, exchange=None, block_limit_bytes: int = 64 << 20):
        self.cfg = cfg
        self.ep_size, self.ep_rank = int(ep_size), int(ep_rank)
        self.mod = lmoe.LatentMoE(cfg, local_experts(layer, cfg.n_ffn, self.ep_size, self.ep_rank), max_tokens,
                                  device=device, ep_size=self.ep_size, ep_rank=self.ep_rank)
        self.device = self.mod.device
        n_local = cfg.n_ffn // self.ep_size
        K, L = cfg.top_k, cfg.latent
        cap = self.ep_size * int(max_tokens) * min(K, n_local)
        bf = dict(dtype=torch.bfloat16, device=self.device)
        self.send_rows = torch.empty((int(max_tokens) * K, L), **bf)
        self.ret_rows = torch.empty((int(max_tokens) * K, L), **bf)
        self.recv_rows = torch.empty((cap, L), **bf)
        self.send_counts = torch.empty(cfg.n_ffn, dtype=torch.int32, device=self.device)
        self.exchange = exchange if exchange is not None else AllToAll(group)
        self._x = None
        self.block_rows = lmoe.lmoe_ep_block_rows(self.mod.h)
        self.rows_bound = self.ep_size * int(max_tokens)  # an expert gets at most one row per token of any rank
        self.block_exchange = self.ep_size * self.block_rows * L * 2 <= block_limit_bytes
        if self.block_exchange:
            self.send_blocks = torch.empty((self.ep_size * self.block_rows, L), **bf)
            self.ret_blocks_buf = torch.empty((self.ep_size * self.block_rows, L), **bf)

    # ---- the stages (the interface ep_forward drives)
    def dispatch(self, x: torch.Tensor):
        self._x = x
        lmoe.lmoe_ep_dispatch(self.mod.h, x, self.send_rows, self.send_counts)
        return self.send_rows, self.send_counts

    def recv_buffer(self, n: int) -> torch.Tensor:
        return self.recv_rows[:n]

    def ret_buffer(self, n: int) -> torch.Tensor:
        return self.ret_rows[:n]

    def experts(self, recv_rows: torch.Tensor, recv_counts: torch.Tensor, n_recv: int, rows_bound: int):
        if n_recv:
            lmoe.lmoe_ep_experts(self.mod.h, recv_rows, recv_counts, n_recv, rows_bound, recv_rows)
        return recv_rows[:n_recv]

    def combine(self, ret_rows: torch.Tensor, y: Optional[torch.Tensor] = None) -> torch.Tensor:
        if y is None:
            y = torch.empty_like(self._x)
        # ret_rows may be empty (nothing routed to FFN experts); the stage reads no row then
        lmoe.lmoe_ep_combine(self.mod.h, ret_rows if ret_rows.numel() else self.ret_rows, y)
        self._x = None
        return y

    # ---- the block-exchange stages (the interface ep_forward_blocks drives)
    def dispatch_blocks(self, x: torch.Tensor):
        self._x = x
        lmoe.lmoe_ep_dispatch_blocks(self.mod.h, x, self.send_blocks, self.block_rows, self.send_counts)
        return self.send_blocks, self.send_counts

    def recv_blocks(self) -> torch.Tensor:
        return self.recv_rows

    def ret_blocks(self) -> torch.Tensor:
        return self.ret_blocks_buf

    def experts_blocks(self, recv_blocks: torch.Tensor, recv_counts: torch.Tensor) -> torch.Tensor:
        lmoe.lmoe_ep_experts_blocks(self.mod.h, recv_blocks, self.block_rows, recv_counts, self.rows_bound,
                                    recv_blocks)
        return recv_blocks

    def combine_blocks(self, ret_blocks: torch.Tensor, y: Optional[torch.Tensor] = None) -> torch.Tensor:
        if y is None:
            y = torch.empty_like(self._x)
        lmoe.lmoe_ep_combine_blocks(self.mod.h, ret_blocks, y)
        self._x = None
        return y

    # ---- a whole forward
    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None) -> torch.Tensor:
        if self.block_exchange:
            return ep_forward_blocks(self, self.exchange, x, y)
        return ep_forward(self, self.exchange, x, y)

    def last_error(self) -> int:
        return self.mod.last_error()

    def close(self) -> None:
        self.mod.close()
