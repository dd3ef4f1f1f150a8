"""CUDA-graph replay of one prism_decode_step call.

The decode step is a fixed chain of a few kernels per layer; capturing the
whole chain once and replaying it removes the per-launch host overhead (the
paper times its kernels the same way, under CUDA graphs).  torch provides the
graph object and the capture stream; the captured work is entirely the
library's kernels.
"""
from __future__ import annotations

import torch

from . import Config, lib, prism_decode_step, prism_decode_step_kq, workspace


class DecodeStepGraph:
    def __init__(self, cfg: Config, q, k_layers, v_layers, lens, out=None, idx_out=None,
                 ws=None, kq_layers=None):
        self.cfg = cfg
        self.q, self.k, self.v, self.lens = q, list(k_layers), list(v_layers), lens
        self.kq = list(kq_layers) if kq_layers is not None else None
        self.out = out if out is not None else torch.empty(
            (cfg.n_layers, cfg.batch, cfg.n_q_heads, cfg.head_dim), dtype=torch.bfloat16,
            device=q.device)
        self.idx_out = idx_out
        self.ws = ws if ws is not None else workspace(cfg, q.device)
        side = torch.cuda.Stream(device=q.device)
        side.wait_stream(torch.cuda.current_stream(q.device))
        with torch.cuda.stream(side):          # eager warm-up (sets kernel attributes)
            self._call(side)
        torch.cuda.current_stream(q.device).wait_stream(side)
        torch.cuda.synchronize(q.device)
        self.graph = torch.cuda.CUDAGraph()
        n0 = lib().prism_launch_count()
        with torch.cuda.graph(self.graph):
            self._call(torch.cuda.current_stream(q.device))
        self.launches = int(lib().prism_launch_count() - n0)

    def _call(self, stream):
        if self.kq is not None:
            prism_decode_step_kq(self.cfg, self.q, self.k, self.v, self.kq, self.lens,
                                 out=self.out, idx_out=self.idx_out, ws=self.ws, stream=stream)
        else:
            prism_decode_step(self.cfg, self.q, self.k, self.v, self.lens, out=self.out,
                              idx_out=self.idx_out, ws=self.ws, stream=stream)

    def replay(self):
        self.graph.replay()
        return self.out
