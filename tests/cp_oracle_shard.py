"""A rank of the context-parallel decode step worked by the oracle (fp64).

Test-only stand-in for long_context_decoding_anchor_b200.cp.CudaShard: the
same four operations on one rank's shard of the positions, computed with the
oracle's scoring, top-k and expansion and a fp64 split softmax, so that the
schedule of cp.decode_step_cp and the exactness of its decomposition
(distributed top-k, split softmax) can be checked on CPU ranks."""
import numpy as np
import torch

MODE_POOL = 3


class OracleShard:
    def __init__(self, o, cfg, n_ranks, rank, shard_len, q, k_layers, v_layers, lens):
        """q: uint16 [N][B][Hq][d]; k_layers/v_layers: uint16 [B][Hkv][Lmax][d]
        (the full caches: a rank reads only its own rows of them)."""
        self.o, self.cfg = o, cfg
        self.R, self.rank, self.S = n_ranks, rank, shard_len
        self.lo = rank * shard_len
        self.q, self.k, self.v = q, k_layers, v_layers
        self.lens = np.asarray(lens)
        self.G = cfg.n_q_heads // cfg.n_kv_heads
        self.scale = cfg.scale if cfg.scale > 0 else 1.0 / np.sqrt(cfg.head_dim)
        self.agg = "max" if cfg.mode == MODE_POOL else "sum"
        self.radius = 0 if cfg.mode == MODE_POOL else cfg.radius

    def _shard_span(self, b):
        L = int(self.lens[b])
        n = max(0, min(L - self.lo, self.S))
        return L, self.lo, self.lo + n

    def _topk_pairs(self, s, pos, n):
        sel, _ = self.o.topk(s, n, pos=pos)
        score_of = dict(zip(pos.tolist(), s.tolist()))
        sc = np.array([score_of[int(i)] if i >= 0 else -np.inf for i in sel])
        return sel, sc

    def index_local(self, layer, src=None):
        cfg, G = self.cfg, self.G
        B, Hkv, kap = cfg.batch, cfg.n_kv_heads, cfg.kappa
        n_pool = cfg.pool_factor * kap
        want_pool = cfg.mode == MODE_POOL and src is None
        cp = np.full((B, Hkv, kap), -1, np.int32)
        cs = np.full((B, Hkv, kap), -np.inf)
        pp = np.full((B, Hkv, n_pool), -1, np.int32)
        ps = np.full((B, Hkv, n_pool), -np.inf)
        srch = None if src is None else src.numpy()
        for b in range(B):
            L, a, e = self._shard_span(b)
            for h in range(Hkv):
                qg = self.q[layer, b, h * G:(h + 1) * G]
                if srch is None:
                    pos = np.arange(a, e, dtype=np.int32)
                else:
                    s_row = srch[b, h]
                    prop = self.o.expand(L, s_row[s_row >= 0], self.radius)
                    pos = prop[(prop >= a) & (prop < e)].astype(np.int32)
                s = self.o.score(qg, self.k[layer][b, h], pos=pos, scale=self.scale, agg=self.agg)
                cp[b, h], cs[b, h] = self._topk_pairs(s, pos, kap)
                if want_pool:
                    pp[b, h], ps[b, h] = self._topk_pairs(s, pos, n_pool)
        out = (torch.from_numpy(cp), torch.from_numpy(cs))
        if want_pool:
            out += (torch.from_numpy(pp), torch.from_numpy(ps))
        return out

    def merge(self, pos_all, score_all):
        P, Sc = pos_all.numpy(), score_all.numpy()
        R, B, Hkv, n = P.shape
        idx = np.full((B, Hkv, n), -1, np.int32)
        for b in range(B):
            for h in range(Hkv):
                p = P[:, b, h].reshape(-1)
                s = Sc[:, b, h].reshape(-1)
                keep = p >= 0
                idx[b, h], _ = self.o.topk(s[keep], n, pos=p[keep])
        return torch.from_numpy(idx)

    def attn_local(self, layer, idx):
        cfg, G = self.cfg, self.G
        B, Hkv, d = cfg.batch, cfg.n_kv_heads, cfg.head_dim
        part = np.zeros((B, Hkv * G, d + 2))
        I = idx.numpy()
        for b in range(B):
            _, a, e = self._shard_span(b)
            for h in range(Hkv):
                sel = I[b, h]
                sel = sel[(sel >= a) & (sel < e)]
                kr = self.k[layer][b, h, sel].astype(np.uint32) << 16
                vr = self.v[layer][b, h, sel].astype(np.uint32) << 16
                kf = kr.view(np.float32).astype(np.float64)
                vf = vr.view(np.float32).astype(np.float64)
                for g in range(G):
                    j = h * G + g
                    row = part[b, j]
                    if sel.size == 0:
                        row[d] = -np.inf
                        continue
                    qf = (self.q[layer, b, j].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
                    z = self.scale * (kf @ qf)
                    m = z.max()
                    w = np.exp(z - m)
                    row[:d] = w @ vf
                    row[d], row[d + 1] = m, w.sum()
        return torch.from_numpy(part)

    def combine(self, part_all):
        P = part_all.numpy()
        d = self.cfg.head_dim
        m = P[..., d]
        M = m.max(axis=0)
        w = np.where(np.isfinite(m), np.exp(m - np.where(np.isfinite(M), M, 0.0)), 0.0)
        num = (w[..., None] * P[..., :d]).sum(axis=0)
        den = (w * P[..., d + 1]).sum(axis=0)
        out = np.where(den[..., None] > 0, num / np.where(den > 0, den, 1.0)[..., None], 0.0)
        return torch.from_numpy(out)
