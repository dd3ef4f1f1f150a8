"""Context-parallel decode step: one long sequence split by position across ranks.

Rank r of R holds the positions [r * shard_len, (r + 1) * shard_len) of every
sequence's K and V.  Each layer of Algorithm 1 ("Prism Attention") becomes:

  selection   every rank keeps its shard's top-k with their scores
              (prism_cp_index_local); the ranks' lists are all-gathered and
              every rank merges them into the exact global selection
              (prism_cp_merge).  A token among the k first of the sequence is
              among the k first of its shard, so nothing is lost.
  attention   every rank forms its shard's split-softmax partial (acc, m, l)
              over the selection (prism_cp_attn_local); the partials are
              all-gathered and merged (prism_cp_combine).

Anchor, refined and shared layers, the modes and the chains follow the
single-GPU step (``prism_decode_step``): a refined layer grows its proposal
from the source selection (the previous layer's, or the last anchor's with
CHAIN_ANCHOR; the anchor's pool in pool mode), a STATIC_REUSE layer copies
its source, a shared layer keeps the previous layer's selection.

``decode_step_cp`` is written over a list of rank handles and a ``gather``
function so that the same schedule runs (a) one rank per process with
``torch.distributed`` (``dist_gather``: all_gather_into_tensor, NCCL on
GPUs), and (b) all ranks in one process on one device (``local_gather``),
which is how a single GPU checks the decomposition.  Every step of the
computation runs in the library's kernels (``CudaShard``).
"""
from __future__ import annotations

from typing import Callable, List, Sequence

import torch

from . import (CHAIN_ANCHOR, MODE_DENSE_ANCHOR, MODE_POOL, MODE_STATIC_REUSE, Config, CpShard,
               cp_workspace, prism_cp_attn_local, prism_cp_combine, prism_cp_index_local,
               prism_cp_merge)

Gather = Callable[[List[torch.Tensor]], torch.Tensor]


def layer_kinds(cfg: Config) -> List[int]:
    """Kind of every layer: 1 anchor (F), 0 refined (R), 2 shared (S)."""
    N = cfg.n_layers
    if cfg.mode == MODE_DENSE_ANCHOR:
        return [1] * N
    if not cfg.anchor_mask:
        raise ValueError("the decode step needs anchor_mask unless DENSE_ANCHOR")
    kinds = [int(cfg.anchor_mask[i]) for i in range(N)]
    if kinds[0] != 1 or any(x not in (0, 1, 2) for x in kinds):
        raise ValueError("anchor_mask: layer 0 must be an anchor, kinds are 0, 1, 2")
    return kinds


def shard_rows(t: torch.Tensor, shard: CpShard) -> torch.Tensor:
    """Rows [lo, lo + shard_len) of a [B][Hkv][Lmax][d] cache as a contiguous
    shard (zero rows past Lmax)."""
    B, H, L, d = t.shape
    lo, n = shard.lo, shard.shard_len
    out = torch.zeros((B, H, n, d), dtype=t.dtype, device=t.device)
    hi = min(L, lo + n)
    if hi > lo:
        out[:, :, : hi - lo].copy_(t[:, :, lo:hi])
    return out


class CudaShard:
    """One rank's shard of a decode step: its K/V shards of every layer, the
    queries of every layer, the GLOBAL lengths, and its workspace."""

    def __init__(self, cfg: Config, shard: CpShard, q, k_layers: Sequence[torch.Tensor],
                 v_layers: Sequence[torch.Tensor], lens, ws=None):
        self.cfg, self.shard = cfg, shard
        self.q, self.k, self.v, self.lens = q, list(k_layers), list(v_layers), lens
        self.ws = cp_workspace(cfg, shard, q.device) if ws is None else ws
        self.ws_side = None      # the attention half's workspace when it trails on its own stream

    def index_local(self, layer: int, src=None):
        return prism_cp_index_local(self.cfg, self.shard, self.q[layer], self.k[layer],
                                    self.lens, src=src, ws=self.ws)

    def merge(self, pos_all, score_all):
        return prism_cp_merge(self.cfg, self.shard, pos_all, score_all, self.lens, ws=self.ws)

    def attn_local(self, layer: int, idx, side: bool = False):
        if side and self.ws_side is None:
            self.ws_side = cp_workspace(self.cfg, self.shard, self.q.device)
        return prism_cp_attn_local(self.cfg, self.shard, self.q[layer], self.k[layer],
                                   self.v[layer], self.lens, idx,
                                   ws=self.ws_side if side else self.ws)

    def combine(self, part_all):
        return prism_cp_combine(self.cfg, part_all)


def local_gather(parts: List[torch.Tensor]) -> torch.Tensor:
    """All ranks in this process: their tensors stacked in rank order."""
    return torch.stack(parts)


def dist_gather(group=None) -> Gather:
    """One rank per process: all_gather_into_tensor over `group` (NCCL), or
    the list form of all_gather where the backend lacks it (gloo)."""
    import torch.distributed as dist

    def gather(parts: List[torch.Tensor]) -> torch.Tensor:
        (x,) = parts
        x = x.contiguous()
        world = dist.get_world_size(group)
        if dist.get_backend(group) == "nccl":
            out = torch.empty((world,) + tuple(x.shape), dtype=x.dtype, device=x.device)
            dist.all_gather_into_tensor(out, x, group=group)
            return out
        bufs = [torch.empty_like(x) for _ in range(world)]
        dist.all_gather(bufs, x, group=group)
        return torch.stack(bufs)

    return gather


def decode_step_cp(cfg: Config, ranks: Sequence, gather: Gather, attn_stream=None,
                   attn_gather: Gather = None):
    """Algorithm 1 over all layers, context parallel.

    ranks: the rank handles this process runs (one per process under
    torch.distributed; all of them when emulating), each with index_local,
    merge, attn_local and combine.  attn_stream (optional, a CUDA stream):
    every layer's attention half runs there, each rank on a second workspace,
    behind the layer's merge, so the next layer's selection does not wait
    for it; attn_gather is then its exchange, which under torch.distributed
    must be a second process group (the two streams' collectives must not
    interleave on one communicator).  Returns (out [N] of [B][Hq][d], idx [N]
    of [B][Hkv][kappa]) as every rank sees them."""
    kinds = layer_kinds(cfg)
    pool_mode = cfg.mode == MODE_POOL
    lead = ranks[0]
    sel: list = [None] * cfg.n_layers
    outs: list = [None] * cfg.n_layers
    pool = None
    last_anchor = 0
    for l, kind in enumerate(kinds):
        src_layer = last_anchor if cfg.chain == CHAIN_ANCHOR else l - 1
        if kind == 2:                                   # shared: the previous selection
            sel[l] = sel[l - 1]
        elif kind == 1:                                 # anchor: Eq. (1)-(2) (and the pool, Eq. (4))
            parts = [r.index_local(l) for r in ranks]
            sel[l] = lead.merge(gather([p[0] for p in parts]), gather([p[1] for p in parts]))
            if pool_mode:
                pool = lead.merge(gather([p[2] for p in parts]), gather([p[3] for p in parts]))
        elif cfg.mode == MODE_STATIC_REUSE:             # Eq. (3): reuse without rescoring
            sel[l] = sel[src_layer]
        else:                                           # refined: Eq. (5)-(6)
            src = pool if pool_mode else sel[src_layer]
            parts = [r.index_local(l, src) for r in ranks]
            sel[l] = lead.merge(gather([p[0] for p in parts]), gather([p[1] for p in parts]))
        if attn_stream is None:
            partials = [r.attn_local(l, sel[l]) for r in ranks]
            outs[l] = lead.combine(gather(partials))
        else:
            # the attention half trails on its own stream (own workspace, own
            # exchange group), so the next layer's selection need not wait for it
            main = torch.cuda.current_stream()
            attn_stream.wait_stream(main)
            sel[l].record_stream(attn_stream)
            with torch.cuda.stream(attn_stream):
                partials = [r.attn_local(l, sel[l], side=True) for r in ranks]
                outs[l] = lead.combine((attn_gather or gather)(partials))
        if kind == 1:
            last_anchor = l
    if attn_stream is not None:
        torch.cuda.current_stream().wait_stream(attn_stream)
        for o in outs:
            o.record_stream(torch.cuda.current_stream())
    return outs, sel
