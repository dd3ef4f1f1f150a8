"""Comparisons of the CUDA path with the oracle, shared by the GPU tests.

Rules (from the method's statement of the parity bar):
  * scores within 1e-2 absolute of the oracle's fp64 scores;
  * selections bit-exact against the oracle's TopK run on the GPU's own
    scores (and, for refined layers, on the GPU's own source selection);
  * recall of the GPU selection against the oracle's fp64 selection >= 0.999;
  * attention outputs within 2e-2 absolute + 1e-2 relative (bf16 outputs),
    against the oracle's attention over the GPU's own selection.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import long_context_decoding_anchor_b200 as prism
from oracle import bf16_bits

SCORE_ATOL = 1e-2
OUT_ATOL, OUT_RTOL = 2e-2, 1e-2
RECALL_MIN = 0.999


def recall(got, ref) -> float:
    g = set(int(x) for x in np.asarray(got) if x >= 0)
    r = set(int(x) for x in np.asarray(ref) if x >= 0)
    if not r:
        return 1.0 if not g else 0.0
    return len(g & r) / len(r)


def rows_of(cfg, rows=None):
    if rows is not None:
        return rows
    return [(b, h) for b in range(cfg.batch) for h in range(cfg.n_kv_heads)]


def scale_of(cfg):
    return cfg.scale if cfg.scale > 0 else 1.0 / math.sqrt(cfg.head_dim)


def check_anchor(o, cfg, q, k, lens, idx, S, rows=None, stats=None):
    """q [B][Hq][d], k [B][Hkv][Lmax][d] (device); idx/S: GPU outputs."""
    G = cfg.n_q_heads // cfg.n_kv_heads
    qh = bf16_bits(q)
    Sh = S.cpu().numpy()
    Ih = idx.cpu().numpy()
    lh = lens.cpu().numpy()
    worst = 0.0
    for b, h in rows_of(cfg, rows):
        L = int(lh[b])
        kh = bf16_bits(k[b, h, :L]) if L > 0 else np.zeros((0, cfg.head_dim), np.uint16)
        s_ref = o.score(qh[b, h * G:(h + 1) * G], kh, scale=scale_of(cfg), n=L)
        s_gpu = Sh[b, h, :L].astype(np.float64)
        if L:
            err = float(np.max(np.abs(s_gpu - s_ref)))
            worst = max(worst, err)
            assert err <= SCORE_ATOL, f"anchor scores row {(b, h)}: max err {err}"
        sel, _ = o.topk(s_gpu, cfg.kappa)
        assert np.array_equal(sel, Ih[b, h]), f"anchor selection row {(b, h)} not bit-exact"
        ref, _ = o.topk(s_ref, cfg.kappa)
        rc = recall(Ih[b, h], ref)
        assert rc >= RECALL_MIN, f"anchor recall row {(b, h)}: {rc}"
    if stats is not None:
        stats["score_err"] = max(stats.get("score_err", 0.0), worst)


def check_refine(o, cfg, q, k, lens, idx_prev, idx, cpos, cscore, ccount, rows=None, stats=None):
    G = cfg.n_q_heads // cfg.n_kv_heads
    qh = bf16_bits(q)
    Ph = idx_prev.cpu().numpy()
    Ih = idx.cpu().numpy()
    cp, cs, cc = cpos.cpu().numpy(), cscore.cpu().numpy(), ccount.cpu().numpy()
    lh = lens.cpu().numpy()
    worst = 0.0
    for b, h in rows_of(cfg, rows):
        L = int(lh[b])
        P = o.expand(L, Ph[b, h], cfg.radius)
        n = int(cc[b, h])
        assert n == len(P), f"proposal size row {(b, h)}: {n} vs {len(P)}"
        assert np.array_equal(cp[b, h, :n], P), f"proposal positions row {(b, h)}"
        kh = bf16_bits(k[b, h, :max(L, 1)])
        s_ref = o.score(qh[b, h * G:(h + 1) * G], kh, pos=P, scale=scale_of(cfg))
        s_gpu = cs[b, h, :n].astype(np.float64)
        if n:
            err = float(np.max(np.abs(s_gpu - s_ref)))
            worst = max(worst, err)
            assert err <= SCORE_ATOL, f"refine scores row {(b, h)}: max err {err}"
        sel, _ = o.topk(s_gpu, cfg.kappa, pos=P)
        assert np.array_equal(sel, Ih[b, h]), f"refine selection row {(b, h)} not bit-exact"
        ref, _ = o.topk(s_ref, cfg.kappa, pos=P)
        rc = recall(Ih[b, h], ref)
        assert rc >= RECALL_MIN, f"refine recall row {(b, h)}: {rc}"
    if stats is not None:
        stats["score_err"] = max(stats.get("score_err", 0.0), worst)


def _pool_ref_scores(o, cfg, qg, k_rows, pos, q2):
    """Eq. (9) scores in fp64: on the bf16 keys, or (q2) on the oracle's own
    2-bit quantization of them (Eq. (7)-(8))."""
    if q2:
        codes, al, be = o.quantize(k_rows)
        return o.score_q2(qg, codes, al, be, pos=pos, scale=scale_of(cfg))
    if pos is None:
        return o.score(qg, k_rows, scale=scale_of(cfg), n=k_rows.shape[0], agg="max")
    return o.score(qg, k_rows, pos=pos, scale=scale_of(cfg), agg="max")


def check_pool_anchor(o, cfg, q, k, lens, pool, idx, S, rows=None, stats=None, q2=False):
    """Pool mode proposal layer: Eq. (9) scores within 1e-2 of fp64; the pool
    (Eq. (4)) and the layer's own top-kappa bit-exact against the oracle's
    TopK on the GPU's own scores; recall of both against the fp64 scores."""
    G = cfg.n_q_heads // cfg.n_kv_heads
    n_pool = cfg.pool_factor * cfg.kappa
    qh = bf16_bits(q)
    Sh, Ph, Ih = S.cpu().numpy(), pool.cpu().numpy(), idx.cpu().numpy()
    lh = lens.cpu().numpy()
    worst = 0.0
    for b, h in rows_of(cfg, rows):
        L = int(lh[b])
        kh = bf16_bits(k[b, h, :L]) if L > 0 else np.zeros((0, cfg.head_dim), np.uint16)
        s_ref = _pool_ref_scores(o, cfg, qh[b, h * G:(h + 1) * G], kh, None, q2)
        s_gpu = Sh[b, h, :L].astype(np.float64)
        if L:
            err = float(np.max(np.abs(s_gpu - s_ref)))
            worst = max(worst, err)
            assert err <= SCORE_ATOL, f"pool scores row {(b, h)}: max err {err}"
        for got, budget, what in ((Ph[b, h], n_pool, "pool"), (Ih[b, h], cfg.kappa, "selection")):
            sel, _ = o.topk(s_gpu, budget)
            assert np.array_equal(sel, got), f"anchor {what} row {(b, h)} not bit-exact"
            ref, _ = o.topk(s_ref, budget)
            rc = recall(got, ref)
            assert rc >= RECALL_MIN, f"anchor {what} recall row {(b, h)}: {rc}"
        valid = Ih[b, h][Ih[b, h] >= 0]
        assert set(valid.tolist()) <= set(Ph[b, h].tolist()), "selection outside the pool"
    if stats is not None:
        stats["score_err"] = max(stats.get("score_err", 0.0), worst)


def check_pool_refine(o, cfg, q, k, lens, pool, idx, cpos, cscore, ccount, rows=None, stats=None,
                      q2=False):
    """Pool mode refined layer: the candidates are the pool's distinct valid
    positions (ascending), Eq. (9) scores within 1e-2, Eq. (6) bit-exact on
    the GPU's own candidate scores, recall against fp64."""
    G = cfg.n_q_heads // cfg.n_kv_heads
    qh = bf16_bits(q)
    Ph, Ih = pool.cpu().numpy(), idx.cpu().numpy()
    cp, cs, cc = cpos.cpu().numpy(), cscore.cpu().numpy(), ccount.cpu().numpy()
    lh = lens.cpu().numpy()
    worst = 0.0
    for b, h in rows_of(cfg, rows):
        L = int(lh[b])
        P = np.unique(Ph[b, h][(Ph[b, h] >= 0) & (Ph[b, h] < L)]).astype(np.int32)
        n = int(cc[b, h])
        assert n == len(P), f"pool candidates row {(b, h)}: {n} vs {len(P)}"
        assert np.array_equal(cp[b, h, :n], P), f"pool candidate positions row {(b, h)}"
        kh = bf16_bits(k[b, h, :max(L, 1)])
        s_ref = _pool_ref_scores(o, cfg, qh[b, h * G:(h + 1) * G], kh, P, q2)
        s_gpu = cs[b, h, :n].astype(np.float64)
        if n:
            err = float(np.max(np.abs(s_gpu - s_ref)))
            worst = max(worst, err)
            assert err <= SCORE_ATOL, f"pool rescoring row {(b, h)}: max err {err}"
        sel, _ = o.topk(s_gpu, cfg.kappa, pos=P)
        assert np.array_equal(sel, Ih[b, h]), f"pool refine selection row {(b, h)} not bit-exact"
        ref, _ = o.topk(s_ref, cfg.kappa, pos=P)
        rc = recall(Ih[b, h], ref)
        assert rc >= RECALL_MIN, f"pool refine recall row {(b, h)}: {rc}"
    if stats is not None:
        stats["score_err"] = max(stats.get("score_err", 0.0), worst)


def check_attention(o, cfg, q, k, v, lens, idx, out, rows=None, stats=None):
    G = cfg.n_q_heads // cfg.n_kv_heads
    qh = bf16_bits(q)
    Ih = idx.cpu().numpy()
    oh = out.float().cpu().numpy()
    lh = lens.cpu().numpy()
    worst = 0.0
    for b, h in rows_of(cfg, rows):
        L = int(lh[b])
        sel = Ih[b, h]
        if L == 0:
            assert np.all(oh[b, h * G:(h + 1) * G] == 0.0)
            continue
        kh = bf16_bits(k[b, h, :L])
        vh = bf16_bits(v[b, h, :L])
        ref, wsum = o.attention(qh[b, h * G:(h + 1) * G], kh, vh, sel, scale=scale_of(cfg))
        got = oh[b, h * G:(h + 1) * G]
        err = np.abs(got - ref) - (OUT_ATOL + OUT_RTOL * np.abs(ref))
        worst = max(worst, float(np.max(np.abs(got - ref))))
        assert np.all(err <= 0), f"attention row {(b, h)}: max abs err {np.max(np.abs(got - ref))}"
    if stats is not None:
        stats["out_err"] = max(stats.get("out_err", 0.0), worst)


def layerwise_step_check(o, cfg, inp, out, idx_all, rows=None, stats=None, layers=None):
    """Check a decode step layer by layer: every layer's selection is
    reproduced by the stage entry points on the GPU's own inputs (bit-exact),
    those stages are checked against the oracle, and every layer's output is
    checked against the oracle's attention over that layer's selection.
    `layers` restricts the check to some layers (each is checked on the
    step's own source selection, so any subset is valid)."""
    mask = list(inp["anchor_mask"])
    N = cfg.n_layers
    ws = prism.workspace(cfg)
    last_anchor = 0
    pool = None
    for l in range(N):
        anchor = cfg.mode == prism.MODE_DENSE_ANCHOR or mask[l] == 1
        shared = cfg.mode != prism.MODE_DENSE_ANCHOR and mask[l] == 2
        q, k, v, lens = inp["q"][l], inp["k"][l], inp["v"][l], inp["lens"]
        if shared:
            # Table 9's shared layer keeps the previous layer's selection
            assert torch.equal(idx_all[l], idx_all[l - 1]), f"layer {l}: shared layer changed"
            if layers is None or l in layers:
                check_attention(o, cfg, q, k, v, lens, idx_all[l], out[l], rows, stats)
            continue
        if cfg.mode == prism.MODE_POOL:
            # The pool of an anchor is not an output of the step: the stage
            # call reproduces it (bit-exact, as the selections show).  With
            # 2-bit keys the stage calls read the layer's 2-bit cache.
            q2 = bool(cfg.flags & prism.FLAG_INT2_KEYS)
            ks = inp["kq"][l] if q2 else k
            if anchor:
                S = torch.empty((cfg.batch, cfg.n_kv_heads, cfg.max_len), dtype=torch.float32,
                                device=q.device)
                pool, idx = prism.prism_index_pool(cfg, q, ks, lens, scores_out=S, ws=ws)
                assert torch.equal(idx, idx_all[l]), f"layer {l}: step selection != stage selection"
                if layers is None or l in layers:
                    check_pool_anchor(o, cfg, q, k, lens, pool, idx, S, rows, stats, q2=q2)
            elif layers is None or l in layers:
                idx, cp, cs, cc = prism.prism_index_refine(cfg, q, ks, lens, pool,
                                                           cand_cap=cfg.max_len, ws=ws)
                assert torch.equal(idx, idx_all[l]), f"layer {l}: step selection != stage selection"
                check_pool_refine(o, cfg, q, k, lens, pool, idx, cp, cs, cc, rows, stats, q2=q2)
            if layers is None or l in layers:
                check_attention(o, cfg, q, k, v, lens, idx_all[l], out[l], rows, stats)
            continue
        if layers is not None and l not in layers:
            if anchor:
                last_anchor = l
            continue
        if anchor:
            S = torch.empty((cfg.batch, cfg.n_kv_heads, cfg.max_len), dtype=torch.float32,
                            device=q.device)
            idx = prism.prism_index_anchor(cfg, q, k, lens, scores_out=S, ws=ws)
            assert torch.equal(idx, idx_all[l]), f"layer {l}: step selection != stage selection"
            check_anchor(o, cfg, q, k, lens, idx, S, rows, stats)
            last_anchor = l
        else:
            src = last_anchor if cfg.chain == prism.CHAIN_ANCHOR else l - 1
            if cfg.mode == prism.MODE_STATIC_REUSE:
                assert torch.equal(idx_all[l], idx_all[src]), f"layer {l}: static reuse"
            else:
                prev = idx_all[src].contiguous()
                idx, cp, cs, cc = prism.prism_index_refine(cfg, q, k, lens, prev,
                                                           cand_cap=cfg.max_len, ws=ws)
                assert torch.equal(idx, idx_all[l]), f"layer {l}: step selection != stage selection"
                check_refine(o, cfg, q, k, lens, prev, idx, cp, cs, cc, rows, stats)
        check_attention(o, cfg, q, k, v, lens, idx_all[l], out[l], rows, stats)
    st, detail = prism.prism_check_device_status(ws)
    assert st == 0, f"device status {st} {detail}"
