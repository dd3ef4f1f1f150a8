"""Pins of the oracle: checks against what the paper and mathematics fix.

Every pin takes an ``Oracle`` and raises AssertionError on a mismatch.  None of
them re-types the oracle's formulas: they compare against numpy/torch library
routines (einsum, lexsort, scaled_dot_product_attention), brute force over
tiny inputs, closed forms and hand-derived cases under tests/golden/.  The
planted-mistake test runs all of them against deliberately wrong builds of the
oracle and requires each build to fail at least one pin.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from helpers import (bf16_bits_to_f64, brute_expand, f32_to_bf16_bits, golden, lexsort_topk,
                     numpy_scores, numpy_scores_max, rand_bf16, sdpa_group, subset_topk)
from long_context_decoding_anchor_b200 import synth
from oracle import (CHAIN_ANCHOR, CHAIN_PREV, MODE_DENSE_ANCHOR, MODE_POOL, MODE_REFINE,
                    MODE_STATIC_REUSE, bf16_bits)


# -- Eq. (1): relevance score ---------------------------------------------------
def pin_score_bruteforce(o):
    """Scores equal numpy.einsum over group and head dim, 64-256 tokens."""
    rng = np.random.default_rng(11)
    for G, d, L in [(4, 64, 64), (2, 128, 256), (1, 16, 100), (8, 64, 128), (3, 32, 77)]:
        q = rand_bf16(rng, (G, d))
        k = rand_bf16(rng, (L, d))
        scale = 1.0 / math.sqrt(d)
        ref = numpy_scores(q, k, scale)
        got = o.score(q, k, scale=scale)
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12), "score vs einsum"
        pos = np.sort(rng.choice(L, size=L // 3, replace=False)).astype(np.int32)
        got = o.score(q, k, pos=pos, scale=scale)
        assert np.allclose(got, ref[pos], rtol=1e-12, atol=1e-12), "score on a position list"


def pin_score_hand(o):
    """Hand case: q=(1,0), k_i=(i,0): scores increase, top-kappa = last kappa."""
    g = golden("score_hand_case")
    L, kappa = g["L"], g["kappa"]
    q = f32_to_bf16_bits(np.array([[1.0, 0.0]], dtype=np.float32))
    k = f32_to_bf16_bits(np.stack([np.arange(L), np.zeros(L)], 1).astype(np.float32))
    s = o.score(q, k, scale=1.0)
    assert np.array_equal(s, np.arange(L, dtype=np.float64)), "hand scores"
    idx, keff = o.topk(s, kappa)
    assert keff == kappa and list(idx) == g["expected_topk"], "hand top-kappa"


# -- Eq. (2)/(6): exact top-kappa ------------------------------------------------
def pin_topk_golden(o):
    for c in golden("topk_cases")["cases"]:
        pos = c.get("positions")
        idx, keff = o.topk(np.array(c["scores"], dtype=np.float64), c["kappa"],
                           pos=None if pos is None else np.array(pos))
        assert list(idx) == c["expected"], f"topk golden {c}"
        assert keff == sum(1 for x in c["expected"] if x >= 0)


def pin_topk_lexsort(o):
    """Top-kappa equals numpy.lexsort on (-score, position), ties included."""
    rng = np.random.default_rng(12)
    for n, kappa, ties in [(1000, 37, False), (1000, 37, True), (300, 300, True), (50, 80, True),
                           (4096, 256, True), (1, 1, False), (257, 256, True)]:
        s = rng.integers(-5, 6, n).astype(np.float64) if ties else rng.standard_normal(n)
        if ties:
            s[rng.random(n) < 0.1] = -0.0
        pos = np.sort(rng.choice(4 * n, size=n, replace=False)).astype(np.int32)
        for p in (None, pos):
            idx, keff = o.topk(s, kappa, pos=p)
            assert np.array_equal(idx, lexsort_topk(s, kappa, p)), "topk vs lexsort"
            assert keff == min(kappa, n)


def pin_topk_all_equal(o):
    for n, kappa in [(10, 3), (4096, 256), (5, 5)]:
        idx, _ = o.topk(np.full(n, 0.25), kappa)
        assert list(idx) == list(range(kappa)), "all-equal scores select {0..kappa-1}"


def pin_topk_subsets(o):
    """Brute force over all kappa-subsets of at most 10 tokens."""
    rng = np.random.default_rng(13)
    for trial in range(40):
        n = int(rng.integers(1, 11))
        kappa = int(rng.integers(1, n + 2))
        s = rng.integers(-2, 3, n).astype(np.float64)
        ref, count = subset_topk(s, kappa)
        assert count == 1, "the tie rule makes the top-kappa subset unique"
        idx, _ = o.topk(s, kappa)
        assert np.array_equal(idx, ref), "topk vs subset brute force"


# -- positional proposal ---------------------------------------------------------
def pin_expand_golden(o):
    for c in golden("expand_cases")["cases"]:
        got = o.expand(c["L"], np.array(c["idx_prev"], dtype=np.int32), c["r"])
        assert list(got) == c["expected"], f"expand golden {c}"


def pin_expand_bruteforce(o):
    rng = np.random.default_rng(14)
    for trial in range(60):
        L = int(rng.integers(1, 300))
        r = int(rng.integers(0, 12))
        n = int(rng.integers(1, 40))
        idx = rng.integers(-3, L + 3, n).astype(np.int32)
        got = o.expand(L, idx, r)
        assert np.array_equal(got, brute_expand(L, idx, r)), "expand vs set brute force"


# -- SparseAttn -------------------------------------------------------------------
def pin_attention_sdpa(o):
    """Attention over an index set equals torch SDPA (fp64) with a mask; with
    kappa = L it is dense attention."""
    rng = np.random.default_rng(15)
    for G, d, L, nsel in [(4, 64, 96, 96), (2, 128, 200, 31), (1, 32, 64, 64), (8, 64, 150, 40)]:
        q, k, v = rand_bf16(rng, (G, d), 2.0), rand_bf16(rng, (L, d)), rand_bf16(rng, (L, d))
        idx = np.sort(rng.choice(L, size=nsel, replace=False)).astype(np.int32)
        idx = np.concatenate([idx, -np.ones(3, dtype=np.int32)])
        scale = 1.0 / math.sqrt(d)
        got, wsum = o.attention(q, k, v, idx, scale)
        ref = sdpa_group(q, k, v, idx, scale)
        assert np.allclose(got, ref, rtol=1e-10, atol=1e-12), "attention vs SDPA"
        assert np.allclose(wsum, 1.0, rtol=0, atol=1e-12), "softmax weights sum to 1"


def pin_attention_closed_forms(o):
    # Two keys, d = 2, scale 1: logits 0 and 1, weights 1/(1+e) and e/(1+e).
    q = f32_to_bf16_bits(np.array([[1.0, 0.0]], np.float32))
    k = f32_to_bf16_bits(np.array([[0.0, 0.0], [1.0, 0.0]], np.float32))
    v = f32_to_bf16_bits(np.array([[1.0, 0.0], [0.0, 1.0]], np.float32))
    got, wsum = o.attention(q, k, v, np.array([0, 1], np.int32), scale=1.0)
    e = math.e
    assert np.allclose(got[0], [1 / (1 + e), e / (1 + e)], rtol=1e-14, atol=1e-15), "two-key closed form"
    # Same keys with the default 1/sqrt(d) scale: logits 0 and 1/sqrt(2).
    got, _ = o.attention(q, k, v, np.array([0, 1], np.int32))
    w1 = 1.0 / (1.0 + math.exp(-1.0 / math.sqrt(2.0)))
    assert np.allclose(got[0], [1 - w1, w1], rtol=1e-14, atol=1e-15), "default scale"
    # All logits equal (identical key rows): the output is the mean of the V rows.
    rng = np.random.default_rng(16)
    G, d, L = 4, 64, 50
    qg = rand_bf16(rng, (G, d))
    krow = rand_bf16(rng, (1, d))
    kk = np.repeat(krow, L, 0)
    vv = rand_bf16(rng, (L, d))
    idx = np.arange(0, L, 2, dtype=np.int32)
    got, wsum = o.attention(qg, kk, vv, idx)
    mean = bf16_bits_to_f64(vv)[idx].mean(0)
    assert np.allclose(got, np.broadcast_to(mean, (G, d)), rtol=1e-13, atol=1e-14), "equal logits -> mean of V"
    # Empty selection: zero output, zero weight.
    got, wsum = o.attention(qg, kk, vv, -np.ones(4, np.int32))
    assert np.all(got == 0.0) and np.all(wsum == 0.0), "empty selection"


# -- Algorithm 1: decode step ----------------------------------------------------
def _hand_inputs():
    g = golden("decode_hand_case")
    L, N = g["L"], len(g["x"])
    q = np.zeros((N, 1, 1, 2), np.float32)
    q[..., 0] = 1.0
    ks, vs = [], []
    for l in range(N):
        k = np.zeros((1, 1, L, 2), np.float32)
        for p, x in g["x"][l].items():
            k[0, 0, int(p), 0] = x
        v = np.stack([np.arange(L), np.ones(L)], 1).astype(np.float32).reshape(1, 1, L, 2)
        ks.append(f32_to_bf16_bits(k))
        vs.append(f32_to_bf16_bits(v))
    return g, f32_to_bf16_bits(q), ks, vs, np.array([L], np.int32)


def pin_decode_hand(o):
    g, q, ks, vs, lens = _hand_inputs()
    cases = {"refine_prev": (MODE_REFINE, CHAIN_PREV), "refine_anchor": (MODE_REFINE, CHAIN_ANCHOR),
             "static_reuse": (MODE_STATIC_REUSE, CHAIN_PREV), "dense_anchor": (MODE_DENSE_ANCHOR, CHAIN_PREV)}
    for name, (mode, chain) in cases.items():
        _, idx = o.decode_step(q, ks, vs, lens, g["kappa"], g["r"], g["anchor_mask"],
                               mode=mode, chain=chain, scale=g["scale"])
        assert idx[:, 0, 0, :].tolist() == g["expected"][name], f"hand decode {name}"
    # shared (S) layers, Table 9: mask value 2
    for name, kinds in (("refine_prev_FSR", [1, 2, 0]), ("refine_prev_FRS", [1, 0, 2])):
        _, idx = o.decode_step(q, ks, vs, lens, g["kappa"], g["r"], kinds, scale=g["scale"])
        assert idx[:, 0, 0, :].tolist() == g["expected"][name], f"hand decode {name}"


def small_workloads():
    """Small synthetic workloads (64-256 tokens) with the generator's structure."""
    w1 = synth.WORKLOADS[1].replace(max_len=256, n_layers=4, kappa=16, radius=2, n_clusters=4,
                                    drift=4)
    w2 = synth.WORKLOADS[2].replace(batch=2, max_len=192, n_layers=5, n_q_heads=8, n_kv_heads=2,
                                    head_dim=64, kappa=24, radius=3, anchor_every=3, n_clusters=4,
                                    drift=5, ragged=(100, 192))
    w3 = synth.WORKLOADS[5].replace(max_len=64, n_layers=3, n_q_heads=8, n_kv_heads=1,
                                    head_dim=32, kappa=8, radius=1, anchor_every=8,
                                    n_clusters=2, drift=2)
    return [w1, w2, w3]


def _bits(inp):
    q = bf16_bits(inp["q"])
    ks = [bf16_bits(t) for t in inp["k"]]
    vs = [bf16_bits(t) for t in inp["v"]]
    return q, ks, vs, inp["lens"].cpu().numpy().astype(np.int32)


def _numpy_chain(w, q, ks, lens, mode, chain, r, mask=None):
    """The decode step's selections recomputed with numpy: einsum scores,
    lexsort top-kappa, set-based proposal.  Layer kinds: 1 anchor, 0 refined,
    2 shared (keeps the previous layer's selection)."""
    N, B, Hq, d = q.shape
    H, G = w.n_kv_heads, w.group
    scale = 1.0 / math.sqrt(d)
    mask = w.anchor_mask() if mask is None else mask
    idx = np.zeros((N, B, H, w.kappa), dtype=np.int64)
    last_anchor = 0
    for l in range(N):
        anchor = mode == MODE_DENSE_ANCHOR or mask[l] == 1
        shared = mode != MODE_DENSE_ANCHOR and mask[l] == 2
        src = last_anchor if chain == CHAIN_ANCHOR else l - 1
        for b in range(B):
            L = int(lens[b])
            for h in range(H):
                qg = q[l, b, h * G:(h + 1) * G]
                kr = ks[l][b, h, :L]
                if shared:
                    idx[l, b, h] = idx[l - 1, b, h]
                elif anchor:
                    idx[l, b, h] = lexsort_topk(numpy_scores(qg, kr, scale), w.kappa)
                elif mode == MODE_STATIC_REUSE:
                    idx[l, b, h] = idx[src, b, h]
                else:
                    P = brute_expand(L, idx[src, b, h], r)
                    idx[l, b, h] = lexsort_topk(numpy_scores(qg, kr, scale, P), w.kappa, P)
        if anchor:
            last_anchor = l
    return idx


def pin_decode_numpy_chain(o):
    """Every mode/chain of the decode step equals the numpy recomputation."""
    for w in small_workloads():
        q, ks, vs, lens = _bits(synth.make_inputs(w))
        for mode, chain in [(MODE_REFINE, CHAIN_PREV), (MODE_REFINE, CHAIN_ANCHOR),
                            (MODE_STATIC_REUSE, CHAIN_PREV), (MODE_DENSE_ANCHOR, CHAIN_PREV)]:
            _, idx = o.decode_step(q, ks, vs, lens, w.kappa, w.radius, w.anchor_mask(),
                                   mode=mode, chain=chain)
            ref = _numpy_chain(w, q, ks, lens, mode, chain, w.radius)
            assert np.array_equal(idx, ref), f"decode chain vs numpy ({w.name}, {mode}, {chain})"


def pin_decode_outputs_sdpa(o):
    """Each layer's output equals masked SDPA over that layer's selection."""
    for w in small_workloads()[:2]:
        q, ks, vs, lens = _bits(synth.make_inputs(w))
        out, idx = o.decode_step(q, ks, vs, lens, w.kappa, w.radius, w.anchor_mask())
        N, B, Hq, d = q.shape
        G = w.group
        for l in range(N):
            for b in range(B):
                L = int(lens[b])
                for h in range(w.n_kv_heads):
                    ref = sdpa_group(q[l, b, h * G:(h + 1) * G], ks[l][b, h, :L], vs[l][b, h, :L],
                                     idx[l, b, h], 1.0 / math.sqrt(d))
                    assert np.allclose(out[l, b, h * G:(h + 1) * G], ref, rtol=1e-10, atol=1e-12), \
                        "decode output vs SDPA"


def pin_decode_invariants(o):
    """Invariants the method fixes:
    r >= L: the refined selection is the exact per-layer top-kappa;
    r = 0 refinement selects the same sets as static reuse;
    static reuse repeats the anchor's selection on every layer;
    kappa = L: every layer's output is dense attention."""
    w = small_workloads()[1]
    q, ks, vs, lens = _bits(synth.make_inputs(w))
    mask = w.anchor_mask()
    _, dense = o.decode_step(q, ks, vs, lens, w.kappa, w.radius, mask, mode=MODE_DENSE_ANCHOR)
    _, wide = o.decode_step(q, ks, vs, lens, w.kappa, w.max_len, mask, mode=MODE_REFINE)
    assert np.array_equal(wide, dense), "r >= L equals per-layer exact selection"
    _, r0 = o.decode_step(q, ks, vs, lens, w.kappa, 0, mask, mode=MODE_REFINE)
    _, st = o.decode_step(q, ks, vs, lens, w.kappa, w.radius, mask, mode=MODE_STATIC_REUSE)
    assert np.array_equal(r0, st), "r = 0 refinement equals static reuse"
    last = 0
    for l in range(len(mask)):
        if mask[l]:
            last = l
            assert np.array_equal(st[l], dense[l]), "anchor layers select exactly"
        assert np.array_equal(st[l], st[last]), "static reuse repeats the anchor"
    # kappa = Lmax: sparse attention over everything = dense attention.
    out, idx = o.decode_step(q, ks, vs, lens, w.max_len, w.radius, mask, mode=MODE_REFINE)
    N, B, Hq, d = q.shape
    G = w.group
    for l in range(N):
        for b in range(B):
            L = int(lens[b])
            for h in range(w.n_kv_heads):
                assert np.array_equal(idx[l, b, h, :L], np.arange(L)), "kappa=L selects all"
                ref = sdpa_group(q[l, b, h * G:(h + 1) * G], ks[l][b, h, :L], vs[l][b, h, :L],
                                 np.arange(L), 1.0 / math.sqrt(d))
                assert np.allclose(out[l, b, h * G:(h + 1) * G], ref, rtol=1e-10, atol=1e-12), \
                    "kappa = L equals dense attention"


# -- pool variant: Eq. (9) group maximum, Eq. (4) pool, Algorithm 1 -------------
def pin_score_max_bruteforce(o):
    """Group-maximum scores equal numpy.einsum per head followed by numpy max."""
    rng = np.random.default_rng(21)
    for G, d, L in [(4, 64, 64), (2, 128, 256), (1, 16, 100), (8, 64, 128), (16, 128, 70)]:
        q = rand_bf16(rng, (G, d))
        k = rand_bf16(rng, (L, d))
        scale = 1.0 / math.sqrt(d)
        ref = numpy_scores_max(q, k, scale)
        got = o.score(q, k, scale=scale, agg="max")
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12), "max score vs einsum+max"
        pos = np.sort(rng.choice(L, size=L // 3, replace=False)).astype(np.int32)
        got = o.score(q, k, pos=pos, scale=scale, agg="max")
        assert np.allclose(got, ref[pos], rtol=1e-12, atol=1e-12), "max score on a position list"
        if G == 1:
            assert np.allclose(got, numpy_scores(q, k, scale, pos), rtol=1e-12, atol=1e-12), \
                "one head: maximum = sum"


def _pool_hand_inputs():
    g = golden("pool_hand_case")
    L, N = g["L"], len(g["keys"])
    q = np.array(g["queries"], np.float32)[None, None].repeat(N, 0)      # [N][1][2][2]
    ks, vs = [], []
    for l in range(N):
        ks.append(f32_to_bf16_bits(np.array(g["keys"][l], np.float32).reshape(1, 1, L, 2)))
        vs.append(f32_to_bf16_bits(np.stack([np.arange(L), np.ones(L)], 1)
                                   .astype(np.float32).reshape(1, 1, L, 2)))
    return g, f32_to_bf16_bits(q), ks, vs, np.array([L], np.int32)


def pin_score_max_hand(o):
    """Hand case of two heads where the group maximum and the group sum order
    the tokens differently."""
    g, q, ks, _, _ = _pool_hand_inputs()
    k0 = ks[0][0, 0]
    assert list(o.score(q[0, 0], k0, scale=1.0, agg="max")) == g["layer0_max_scores"], "hand max"
    assert list(o.score(q[0, 0], k0, scale=1.0)) == g["layer0_sum_scores"], "hand sum"


def pin_pool_hand(o):
    g, q, ks, vs, lens = _pool_hand_inputs()
    kw = dict(mode=MODE_POOL, scale=g["scale"], want_pool=True)
    _, idx, pool = o.decode_step(q, ks, vs, lens, g["kappa"], 0, g["anchor_mask"], rho=g["rho"], **kw)
    assert idx[:, 0, 0].tolist() == g["expected"]["selection"], "hand pool selections"
    assert pool[:, 0, 0].tolist() == g["expected"]["pool"], "hand pools"
    _, idx, _ = o.decode_step(q, ks, vs, lens, g["kappa"], 0, g["anchor_mask"], rho=1, **kw)
    assert idx[:, 0, 0].tolist() == g["expected"]["selection_rho1"], "hand pool, rho = 1"
    _, idx, _ = o.decode_step(q, ks, vs, lens, g["kappa"], 0, [1, 1, 1], rho=g["rho"], **kw)
    assert idx[:, 0, 0].tolist() == g["expected"]["selection_all_anchors"], "hand pool, all anchors"
    for name, kinds in (("selection_FRS", [1, 0, 2]), ("selection_FSR", [1, 2, 0])):
        _, idx, pool = o.decode_step(q, ks, vs, lens, g["kappa"], 0, kinds, rho=g["rho"], **kw)
        assert idx[:, 0, 0].tolist() == g["expected"][name], f"hand pool {name}"
        assert pool[:, 0, 0].tolist() == g["expected"]["pool"], f"hand pool {name}: pools"


def _numpy_pool_chain(w, q, ks, lens, rho, mask=None):
    """The pool variant recomputed with numpy: einsum+max scores, lexsort
    top-(rho*kappa) pool, the anchor's selection as the lexsort top-kappa of the
    pool's scores, refined layers as the lexsort top-kappa of their own scores
    over the nearest preceding anchor's pool."""
    N, B, Hq, d = q.shape
    H, G = w.n_kv_heads, w.group
    scale = 1.0 / math.sqrt(d)
    mask = w.anchor_mask() if mask is None else mask
    n = rho * w.kappa
    idx = np.zeros((N, B, H, w.kappa), dtype=np.int64)
    pool = np.zeros((N, B, H, n), dtype=np.int64)
    for l in range(N):
        for b in range(B):
            L = int(lens[b])
            for h in range(H):
                qg = q[l, b, h * G:(h + 1) * G]
                kr = ks[l][b, h, :L]
                if mask[l] == 2:
                    pool[l, b, h] = pool[l - 1, b, h]
                    idx[l, b, h] = idx[l - 1, b, h]
                elif mask[l] == 1:
                    s = numpy_scores_max(qg, kr, scale)
                    pool[l, b, h] = lexsort_topk(s, n)
                    C = pool[l, b, h][pool[l, b, h] >= 0]
                    idx[l, b, h] = lexsort_topk(s[C], w.kappa, C)
                else:
                    pool[l, b, h] = pool[l - 1, b, h]
                    C = pool[l, b, h][pool[l, b, h] >= 0]
                    idx[l, b, h] = lexsort_topk(numpy_scores_max(qg, kr, scale, C), w.kappa, C)
    return idx, pool


def pin_pool_numpy_chain(o):
    """The pool variant's selections and pools equal the numpy recomputation."""
    for w in small_workloads():
        q, ks, vs, lens = _bits(synth.make_inputs(w))
        for rho in (1, 2, 4):
            _, idx, pool = o.decode_step(q, ks, vs, lens, w.kappa, w.radius, w.anchor_mask(),
                                         mode=MODE_POOL, rho=rho, want_pool=True)
            ref_idx, ref_pool = _numpy_pool_chain(w, q, ks, lens, rho)
            assert np.array_equal(pool, ref_pool), f"pools vs numpy ({w.name}, rho {rho})"
            assert np.array_equal(idx, ref_idx), f"pool selections vs numpy ({w.name}, rho {rho})"


def pin_pool_invariants(o):
    """Invariants of the pool variant:
    rho*kappa >= L: every refined layer selects its exact per-layer top-kappa;
    rho = 1: every refined layer keeps its anchor's selection (static reuse);
    an anchor's selection lies inside its pool, which lies inside [0, L);
    one query head per KV head: the pool variant with every layer an anchor is
    the dense-anchor mode (maximum = sum);
    every output is SDPA over its layer's selection."""
    w = small_workloads()[1]
    q, ks, vs, lens = _bits(synth.make_inputs(w))
    mask = w.anchor_mask()
    N = len(mask)
    everywhere = [1] * N
    rho_all = -(-w.max_len // w.kappa)
    _, exact, _ = o.decode_step(q, ks, vs, lens, w.kappa, 0, everywhere, mode=MODE_POOL, rho=2,
                                want_pool=True)
    _, wide, _ = o.decode_step(q, ks, vs, lens, w.kappa, 0, mask, mode=MODE_POOL, rho=rho_all,
                               want_pool=True)
    assert np.array_equal(wide, exact), "rho*kappa >= L equals per-layer exact selection"
    out, r1, pool1 = o.decode_step(q, ks, vs, lens, w.kappa, 0, mask, mode=MODE_POOL, rho=1,
                                   want_pool=True)
    last = 0
    for l in range(N):
        if mask[l]:
            last = l
        assert np.array_equal(r1[l], r1[last]), "rho = 1 keeps the anchor's selection"
    _, idx, pool = o.decode_step(q, ks, vs, lens, w.kappa, 0, mask, mode=MODE_POOL, rho=3,
                                 want_pool=True)
    B, H = w.batch, w.n_kv_heads
    for l in range(N):
        for b in range(B):
            L = int(lens[b])
            for h in range(H):
                P = pool[l, b, h]
                P = P[P >= 0]
                assert len(P) == min(L, 3 * w.kappa) and np.all(P < L), "pool size and range"
                S = idx[l, b, h]
                assert set(S[S >= 0].tolist()) <= set(P.tolist()), "selection inside the pool"
    # one query head per KV head: group maximum = group sum
    w1 = w.replace(n_q_heads=w.n_kv_heads)
    q1 = q[:, :, ::w.group].copy()
    _, dense = o.decode_step(q1, ks, vs, lens, w1.kappa, 0, mask, mode=MODE_DENSE_ANCHOR)
    _, pooled = o.decode_step(q1, ks, vs, lens, w1.kappa, 0, everywhere, mode=MODE_POOL, rho=2)
    assert np.array_equal(dense, pooled), "G = 1: pool variant with anchors everywhere = dense"
    d = q.shape[-1]
    G = w.group
    for l in range(N):
        for b in range(B):
            L = int(lens[b])
            for h in range(H):
                ref = sdpa_group(q[l, b, h * G:(h + 1) * G], ks[l][b, h, :L], vs[l][b, h, :L],
                                 r1[l, b, h], 1.0 / math.sqrt(d))
                assert np.allclose(out[l, b, h * G:(h + 1) * G], ref, rtol=1e-10, atol=1e-12), \
                    "pool-mode output vs SDPA"


# Table 9 layer kinds -- 'F' anchor (1), 'R' refined (0), 'S' shared (2) --
# the 10F11R57S hybrid pattern of the paper's GLM experiment (78 layers)
TABLE9_10F11R57S = ("FFRSSSRSSSRSSSFSSSFSSSRSSSFSSSRSSSFSSSRSSSFSSSRSSSRSSSRSSSRSSSFSSSRSSSFSSSFSSS")
KIND = {"F": 1, "R": 0, "S": 2}


def kinds_of(pattern):
    return [KIND[c] for c in pattern]


def pin_shared_numpy(o):
    """Patterns mixing F, R and S layers, in refine and pool modes, equal the
    numpy recomputations; Table 9's 78-layer hybrid pattern on a small row."""
    rng = np.random.default_rng(22)
    w = small_workloads()[1].replace(n_layers=8)
    q, ks, vs, lens = _bits(synth.make_inputs(w))
    for trial in range(3):
        kinds = [1] + [int(x) for x in rng.integers(0, 3, w.n_layers - 1)]
        for chain in (CHAIN_PREV, CHAIN_ANCHOR):
            _, idx = o.decode_step(q, ks, vs, lens, w.kappa, w.radius, kinds, chain=chain)
            ref = _numpy_chain(w, q, ks, lens, MODE_REFINE, chain, w.radius, mask=kinds)
            assert np.array_equal(idx, ref), f"refine F/R/S chain vs numpy {kinds}"
        _, idx, pool = o.decode_step(q, ks, vs, lens, w.kappa, 0, kinds, mode=MODE_POOL, rho=2,
                                     want_pool=True)
        ref_idx, ref_pool = _numpy_pool_chain(w, q, ks, lens, 2, mask=kinds)
        assert np.array_equal(idx, ref_idx) and np.array_equal(pool, ref_pool), \
            f"pool F/R/S chain vs numpy {kinds}"
    # the paper's hybrid pattern, 78 layers, on a tiny row
    wt = small_workloads()[2].replace(n_layers=len(TABLE9_10F11R57S), max_len=48, kappa=4)
    q, ks, vs, lens = _bits(synth.make_inputs(wt))
    kinds = kinds_of(TABLE9_10F11R57S)
    _, idx, _ = o.decode_step(q, ks, vs, lens, wt.kappa, 0, kinds, mode=MODE_POOL, rho=4,
                              want_pool=True)
    ref_idx, _ = _numpy_pool_chain(wt, q, ks, lens, 4, mask=kinds)
    assert np.array_equal(idx, ref_idx), "Table 9 pattern vs numpy"


def pin_shared_invariants(o):
    """An anchor followed only by shared layers is static reuse (Eq. (3)); a
    shared layer never changes the selection it follows."""
    w = small_workloads()[1]
    q, ks, vs, lens = _bits(synth.make_inputs(w))
    N = w.n_layers
    mask = w.anchor_mask()
    shared = [1 if m else 2 for m in mask]
    _, st = o.decode_step(q, ks, vs, lens, w.kappa, w.radius, mask, mode=MODE_STATIC_REUSE)
    _, idx = o.decode_step(q, ks, vs, lens, w.kappa, w.radius, shared)
    assert np.array_equal(idx, st), "F then S equals static reuse"
    # pool mode scores by the group maximum: its static reuse is rho = 1
    _, st_max = o.decode_step(q, ks, vs, lens, w.kappa, 0, mask, mode=MODE_POOL, rho=1)
    _, idx = o.decode_step(q, ks, vs, lens, w.kappa, 0, shared, mode=MODE_POOL, rho=2)
    assert np.array_equal(idx, st_max), "F then S equals rho = 1 in pool mode"


# -- 2-bit proposal keys: Eq. (7)-(8) quantizer, Eq. (9) on dequantized keys --
def pin_quantize_hand(o):
    g = golden("quantize_cases")
    for r in g["rows"]:
        k = f32_to_bf16_bits(np.array([r["values"]], np.float32))
        codes, alpha, beta = o.quantize(k, g=g["g"])
        assert codes[0].tolist() == r["codes"], f"hand codes: {r['note']}"
        assert float(alpha[0, 0]) == r["alpha"] and float(beta[0, 0]) == r["beta"], r["note"]


def _numpy_quantize(k_bits, g=32):
    """Eq. (7)-(8) in numpy float32 (IEEE binary32 like the oracle and the
    kernel): per group alpha = (max - min) / 3, beta = min, codes =
    clip(floor((k - beta) / alpha + 0.5), 0, 3), alpha = 0 -> code 0."""
    k = bf16_bits_to_f64(k_bits).astype(np.float32)
    n, d = k.shape
    kg = k.reshape(n, d // g, g)
    lo = kg.min(axis=2)
    hi = kg.max(axis=2)
    a = ((hi - lo) / np.float32(3.0)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        x = ((kg - lo[..., None]) / a[..., None]).astype(np.float32)
        c = np.floor((x + np.float32(0.5)).astype(np.float32))
    c = np.where(a[..., None] > 0, np.clip(c, 0, 3), 0).astype(np.uint8)
    return c.reshape(n, d), a, lo


def pin_quantize_numpy_and_bound(o):
    """The codes equal a numpy float32 recomputation; every element is
    reconstructed within alpha / 2 (round to nearest), the group's minimum
    codes to 0 and its maximum to 3."""
    rng = np.random.default_rng(23)
    for d, scale in ((128, 1.0), (64, 3.0), (128, 0.01)):
        k = rand_bf16(rng, (300, d), scale)
        codes, alpha, beta = o.quantize(k)
        c2, a2, b2 = _numpy_quantize(k)
        assert np.array_equal(codes, c2), "codes vs numpy"
        assert np.array_equal(alpha, a2) and np.array_equal(beta, b2), "alpha/beta vs numpy"
        kf = bf16_bits_to_f64(k).reshape(300, d // 32, 32)
        rec = alpha.astype(np.float64)[..., None] * codes.reshape(300, d // 32, 32) + \
            beta.astype(np.float64)[..., None]
        assert np.all(np.abs(rec - kf) <= alpha.astype(np.float64)[..., None] * (0.5 + 1e-6) + 1e-12), \
            "reconstruction within alpha/2"
        cg = codes.reshape(300, d // 32, 32)
        assert np.all(cg.min(axis=2) == 0) and np.all(cg.max(axis=2) == 3), "min -> 0, max -> 3"


def pin_score_q2_numpy(o):
    """Eq. (9) on 2-bit keys equals numpy einsum on the dequantized matrix,
    then numpy max over the group."""
    rng = np.random.default_rng(24)
    for G, d, n in ((4, 128, 200), (8, 64, 100), (1, 128, 64)):
        q = rand_bf16(rng, (G, d))
        k = rand_bf16(rng, (n, d))
        codes, alpha, beta = o.quantize(k)
        khat = np.repeat(alpha.astype(np.float64), 32, axis=1) * codes + \
            np.repeat(beta.astype(np.float64), 32, axis=1)
        ref = (np.einsum("gd,ld->gl", bf16_bits_to_f64(q), khat) / math.sqrt(d)).max(axis=0)
        got = o.score_q2(q, codes, alpha, beta)
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12), "q2 score vs numpy"
        pos = np.sort(rng.choice(n, n // 3, replace=False)).astype(np.int32)
        assert np.allclose(o.score_q2(q, codes, alpha, beta, pos=pos), ref[pos], rtol=1e-12,
                           atol=1e-12), "q2 score on a position list"


def pin_q2_decode(o):
    """The pool-mode step on 2-bit keys equals a numpy recomputation; with
    keys that the quantizer represents exactly it equals the bf16 step."""
    w = small_workloads()[1]
    q, ks, vs, lens = _bits(synth.make_inputs(w))
    N, B, Hq, d = q.shape
    H, G = w.n_kv_heads, w.group
    mask = w.anchor_mask()
    _, idx = o.decode_step(q, ks, vs, lens, w.kappa, 0, mask, mode=MODE_POOL, rho=2, qbits=2)
    n = 2 * w.kappa
    ref = np.zeros_like(idx, dtype=np.int64)
    pool = np.zeros((B, H, n), np.int64)
    for l in range(N):
        for b in range(B):
            L = int(lens[b])
            for h in range(H):
                c, a, bt = _numpy_quantize(ks[l][b, h, :L])
                khat = np.repeat(a.astype(np.float64), 32, axis=1) * c + \
                    np.repeat(bt.astype(np.float64), 32, axis=1)
                s = (np.einsum("gd,ld->gl", bf16_bits_to_f64(q[l, b, h * G:(h + 1) * G]), khat)
                     / math.sqrt(d)).max(axis=0)
                if mask[l]:
                    pool[b, h] = lexsort_topk(s, n)
                    C = pool[b, h][pool[b, h] >= 0]
                    ref[l, b, h] = lexsort_topk(s[C], w.kappa, C)
                else:
                    C = pool[b, h][pool[b, h] >= 0]
                    ref[l, b, h] = lexsort_topk(s[C], w.kappa, C)
    assert np.array_equal(idx, ref), "2-bit pool step vs numpy"
    # keys the quantizer represents exactly: every group holds beta + alpha*{0..3}
    rng = np.random.default_rng(25)
    ex = []
    for l in range(N):
        c = rng.integers(0, 4, ks[l].shape)
        c[..., 0::32] = 0
        c[..., 1::32] = 3
        a = 2.0 ** rng.integers(-3, 1, ks[l].shape[:-1] + (d // 32,))
        bt = -2.0 * a
        kv = np.repeat(a, 32, axis=-1) * c + np.repeat(bt, 32, axis=-1)
        ex.append(f32_to_bf16_bits(kv.astype(np.float32)))
    _, i16 = o.decode_step(q, ex, vs, lens, w.kappa, 0, mask, mode=MODE_POOL, rho=2)
    _, i2 = o.decode_step(q, ex, vs, lens, w.kappa, 0, mask, mode=MODE_POOL, rho=2, qbits=2)
    assert np.array_equal(i16, i2), "exactly representable keys: 2-bit step = bf16 step"


ALL_PINS = [pin_score_bruteforce, pin_score_hand, pin_topk_golden, pin_topk_lexsort,
            pin_topk_all_equal, pin_topk_subsets, pin_expand_golden, pin_expand_bruteforce,
            pin_attention_sdpa, pin_attention_closed_forms, pin_decode_hand,
            pin_decode_numpy_chain, pin_decode_outputs_sdpa, pin_decode_invariants,
            pin_score_max_bruteforce, pin_score_max_hand, pin_pool_hand, pin_pool_numpy_chain,
            pin_pool_invariants, pin_shared_numpy, pin_shared_invariants, pin_quantize_hand,
            pin_quantize_numpy_and_bound, pin_score_q2_numpy, pin_q2_decode]

__all__ = ["ALL_PINS", "small_workloads"] + [p.__name__ for p in ALL_PINS]
_ = torch  # torch is used through helpers.sdpa_group and synth
