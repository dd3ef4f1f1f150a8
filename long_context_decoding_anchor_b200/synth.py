"""Seeded synthetic decode-step inputs shaped like the Prism Attention workloads.

This module draws inputs only.  It holds none of the method's arithmetic (no
scoring, no selection, no attention): it draws Q/K/V, applies a rotary position
embedding so that keys depend on their position, and plants salient token
clusters whose keys lean toward the layer's query.  The CUDA library and the
oracle both consume exactly the bf16 tensors it returns.

Recipe (per layer l of workload w, generator seed 1000*w + l):
  * Q [B][Hq][d], K and V [B][Hkv][Lmax][d] ~ N(0, 1) in fp32, drawn in that
    order from one torch.Generator;
  * with RoPE (theta 500000, rotate-half convention): keys are rotated to
    their position i, queries to the current position len[b]-1;
  * Q is rounded to bf16 (round to nearest even); qhat[b][h] is the unit
    vector of the sum of the (rounded) query heads of KV head h;
  * every cluster of w=8 consecutive tokens gets +beta*qhat added to its keys
    (beta = 3: the projection of an N(0, I) key on a unit vector has sd 1);
  * with sinks, tokens 0..3 get +6*qhat;
  * K and V are rounded to bf16.
Cluster starts are drawn per (batch, KV head) from a CPU generator seeded
1000*w + 500: uniform in [4, len-8] at layer 0, then each layer moves every
start by a uniform integer in [-D, D] and clips it back into that range.
Per-sequence lengths of the ragged workload come from a CPU generator seeded
1000*w + 777.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and salience recipe of one synthetic decode-step workload."""

    key: int                 # workload number (seeds derive from it)
    name: str
    batch: int
    max_len: int             # Lmax: padded capacity per (batch, KV head)
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    kappa: int
    radius: int
    anchor_every: int        # anchor at layers 0, anchor_every, 2*anchor_every, ...
    n_clusters: int
    cluster_width: int
    drift: int               # D: per-layer shift of cluster starts, uniform in [-D, D]
    rope: bool
    sink: bool
    ragged: Optional[tuple] = None   # (lo, hi): per-sequence lengths uniform in [lo, hi]

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def rows(self) -> int:
        return self.batch * self.n_kv_heads

    def anchor_mask(self) -> list:
        return [1 if (l % self.anchor_every) == 0 else 0 for l in range(self.n_layers)]

    def describe(self) -> str:
        lens = (f"len U[{self.ragged[0]},{self.ragged[1]}] (Lmax {self.max_len})"
                if self.ragged else f"len {self.max_len}")
        return (f"batch {self.batch}, {lens}, {self.n_layers} layers (anchor every "
                f"{self.anchor_every}), {self.n_q_heads} q / {self.n_kv_heads} kv heads, "
                f"head_dim {self.head_dim}, kappa {self.kappa}, r {self.radius}")

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    1: Workload(1, "tiny-4k", 1, 4096, 4, 8, 2, 64, 256, 4, 4, 16, 8, 16, False, False),
    2: Workload(2, "group-32k", 1, 32768, 8, 32, 8, 128, 2048, 8, 4, 64, 8, 32, True, True),
    3: Workload(3, "long-128k", 1, 131072, 32, 32, 8, 128, 2048, 8, 4, 64, 8, 32, True, True),
    4: Workload(4, "batched-ragged-32k", 16, 32768, 16, 32, 8, 128, 1024, 8, 4, 64, 8, 32,
                True, True, ragged=(8192, 32768)),
    5: Workload(5, "extreme-512k", 1, 524288, 8, 64, 8, 128, 4096, 16, 8, 256, 8, 64, True, True),
}

ROPE_THETA = 500000.0
CLUSTER_BETA = 3.0
SINK_BETA = 6.0
N_SINK = 4


def lengths(w: Workload) -> torch.Tensor:
    """Per-sequence context lengths (int32, CPU)."""
    if w.ragged is None:
        return torch.full((w.batch,), w.max_len, dtype=torch.int32)
    g = torch.Generator(device="cpu").manual_seed(1000 * w.key + 777)
    lo, hi = w.ragged
    return torch.randint(lo, hi + 1, (w.batch,), generator=g, dtype=torch.int64).to(torch.int32)


def cluster_starts(w: Workload, lens: torch.Tensor) -> torch.Tensor:
    """Cluster start positions per layer: int64 [N][B][Hkv][n_clusters] (CPU)."""
    g = torch.Generator(device="cpu").manual_seed(1000 * w.key + 500)
    B, H, M, W = w.batch, w.n_kv_heads, w.n_clusters, w.cluster_width
    lo = 4
    hi = (lens.to(torch.int64) - W).clamp(min=lo).view(B, 1, 1)     # inclusive upper bound
    span = (hi - lo + 1).to(torch.float64)
    u = torch.rand((B, H, M), generator=g, dtype=torch.float64)
    cur = lo + torch.floor(u * span).to(torch.int64)
    out = [cur.clone()]
    for _ in range(1, w.n_layers):
        step = torch.randint(-w.drift, w.drift + 1, (B, H, M), generator=g, dtype=torch.int64)
        cur = torch.minimum(torch.maximum(cur + step, torch.full_like(cur, lo)), hi.expand_as(cur))
        out.append(cur.clone())
    return torch.stack(out, 0)


def _rope_tables(positions: torch.Tensor, d: int, device) -> tuple:
    inv = ROPE_THETA ** (-torch.arange(0, d // 2, dtype=torch.float64, device=device) * 2.0 / d)
    ang = positions.to(torch.float64).unsqueeze(-1) * inv
    return torch.cos(ang).to(torch.float32), torch.sin(ang).to(torch.float32)


def _rotate(x: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor) -> torch.Tensor:
    h = x.shape[-1] // 2
    x1, x2 = x[..., :h], x[..., h:]
    return torch.cat([x1 * cos - x2 * sin, x2 * cos + x1 * sin], dim=-1)


def make_layer(w: Workload, layer: int, lens: torch.Tensor, starts: torch.Tensor,
               device="cpu"):
    """Draw (q [B][Hq][d], k, v [B][Hkv][Lmax][d]) for one layer, all bf16."""
    B, Hq, H, d, L = w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.max_len
    G = w.group
    g = torch.Generator(device=device).manual_seed(1000 * w.key + layer)
    q = torch.randn((B, Hq, d), generator=g, device=device, dtype=torch.float32)
    k = torch.randn((B, H, L, d), generator=g, device=device, dtype=torch.float32)
    v = torch.randn((B, H, L, d), generator=g, device=device, dtype=torch.float32)
    lens_d = lens.to(device=device, dtype=torch.int64)
    if w.rope:
        cos, sin = _rope_tables(torch.arange(L, device=device), d, device)
        k = _rotate(k, cos, sin)                                   # key i at position i
        qc, qs = _rope_tables(lens_d - 1, d, device)               # [B][d/2]
        q = _rotate(q, qc.unsqueeze(1), qs.unsqueeze(1))           # query at len-1
    q = q.to(torch.bfloat16)
    qsum = q.to(torch.float32).view(B, H, G, d).sum(2)
    qhat = qsum / qsum.norm(dim=-1, keepdim=True).clamp(min=1e-30)  # [B][H][d]
    W = w.cluster_width
    st = starts[layer].to(device)                                  # [B][H][M]
    offs = st.unsqueeze(-1) + torch.arange(W, device=device)       # [B][H][M][W]
    offs = offs.reshape(B, H, -1)
    cnt = torch.zeros((B, H, L), device=device, dtype=torch.float32)
    cnt.scatter_add_(2, offs, torch.ones_like(offs, dtype=torch.float32))
    bias = CLUSTER_BETA * cnt
    if w.sink:
        bias[:, :, :N_SINK] += SINK_BETA
    k = k + bias.unsqueeze(-1) * qhat.unsqueeze(2)
    return q, k.to(torch.bfloat16), v.to(torch.bfloat16)


def make_inputs(w: Workload, device="cpu", layers: Optional[Sequence[int]] = None):
    """All inputs of one decode step.

    Returns a dict with q [N][B][Hq][d] (bf16), k and v (lists of N tensors
    [B][Hkv][Lmax][d], bf16), lens [B] (int32, on ``device``), anchor_mask
    (list of N ints).  ``layers`` selects a subset of layers (their seeds and
    cluster positions are those of the full workload).
    """
    lens = lengths(w)
    starts = cluster_starts(w, lens)
    layers = list(range(w.n_layers)) if layers is None else list(layers)
    qs, ks, vs = [], [], []
    for l in layers:
        q, k, v = make_layer(w, l, lens, starts, device)
        qs.append(q)
        ks.append(k)
        vs.append(v)
    mask = w.anchor_mask()
    return {
        "q": torch.stack(qs, 0).contiguous(),
        "k": ks,
        "v": vs,
        "lens": lens.to(device),
        "anchor_mask": [mask[l] for l in layers],
        "layers": layers,
        "starts": starts,
    }


def kv_bytes(w: Workload) -> int:
    return 2 * w.n_layers * w.batch * w.n_kv_heads * w.max_len * w.head_dim * 2
