"""CUDA path against the oracle on seeded synthetic inputs (GPU only).

Sizes span several tiles and ragged tails; the tiny and 32K workloads run at
their full sizes, the batched ragged one at reduced batch; the 128K and 512K
workloads are covered by tests/test_gpu_fullsize.py on sampled rows."""
import math

import numpy as np
import pytest
import torch

import long_context_decoding_anchor_b200 as prism
from long_context_decoding_anchor_b200 import synth
from gpu_checks import (check_anchor, check_attention, check_refine, layerwise_step_check,
                        recall)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    prism.lib()   # the library must load: no fallback


def _inputs(w, layers=None):
    return synth.make_inputs(w, device="cuda", layers=layers)


SHAPES = {
    # name: workload overrides (kept small: several tiles, ragged tails)
    "tiny-full": synth.WORKLOADS[1],
    "d128-g4": synth.WORKLOADS[2].replace(max_len=5000, n_layers=3, kappa=200, radius=3,
                                          n_clusters=8),
    "d128-g8-ragged": synth.WORKLOADS[4].replace(batch=3, max_len=3001, n_layers=3,
                                                 n_q_heads=64, kappa=128, radius=2,
                                                 ragged=(700, 3001), n_clusters=6),
    "d128-g16": synth.WORKLOADS[5].replace(max_len=2304, n_layers=2, n_q_heads=32,
                                           n_kv_heads=2, kappa=96, radius=5, n_clusters=4),
    "d64-g1": synth.WORKLOADS[1].replace(max_len=1000, n_layers=3, n_q_heads=2,
                                         n_kv_heads=2, kappa=100, radius=1),
    "d64-g2-batch": synth.WORKLOADS[1].replace(batch=4, max_len=777, n_layers=2,
                                               n_q_heads=4, n_kv_heads=2, kappa=64,
                                               radius=2, ragged=(1, 777), n_clusters=3),
    "d64-g8": synth.WORKLOADS[1].replace(max_len=1500, n_layers=2, n_q_heads=16,
                                         n_kv_heads=2, kappa=300, radius=4),
    # a budget of 9000 over 30011 tokens (the anchor's cluster selection
    # with large tie lists)
    "d64-kappa-9000": synth.WORKLOADS[1].replace(max_len=30011, n_layers=2, kappa=9000,
                                                 radius=1, n_clusters=40),
    # more rows than SMs: the rescoring's blocks cannot all be resident at
    # once, so refined rows go through the run selection kernel
    "d128-160-rows": synth.WORKLOADS[4].replace(batch=20, max_len=2000, n_layers=2, kappa=128,
                                                ragged=(500, 2000), n_clusters=4),
}


@pytest.mark.parametrize("name", list(SHAPES))
def test_anchor_refine_attention_stages(oracle, name):
    w = SHAPES[name]
    inp = _inputs(w, layers=[0, 1])
    cfg = prism.Config.from_workload(w)
    q0, k0, v0, lens = inp["q"][0], inp["k"][0], inp["v"][0], inp["lens"]
    S = torch.empty((w.batch, w.n_kv_heads, w.max_len), dtype=torch.float32, device="cuda")
    ws = prism.workspace(cfg)
    idx0 = prism.prism_index_anchor(cfg, q0, k0, lens, scores_out=S, ws=ws)
    check_anchor(oracle, cfg, q0, k0, lens, idx0, S)
    out0 = prism.prism_sparse_decode(cfg, q0, k0, v0, lens, idx0, ws=ws)
    check_attention(oracle, cfg, q0, k0, v0, lens, idx0, out0)
    q1, k1, v1 = inp["q"][1], inp["k"][1], inp["v"][1]
    idx1, cp, cs, cc = prism.prism_index_refine(cfg, q1, k1, lens, idx0, cand_cap=w.max_len, ws=ws)
    check_refine(oracle, cfg, q1, k1, lens, idx0, idx1, cp, cs, cc)
    out1 = prism.prism_sparse_decode(cfg, q1, k1, v1, lens, idx1, ws=ws)
    check_attention(oracle, cfg, q1, k1, v1, lens, idx1, out1)
    st, detail = prism.prism_check_device_status(ws)
    assert st == 0, detail


@pytest.mark.parametrize("wkey", [1, 2])
def test_decode_step_full_workload(oracle, wkey):
    """The tiny (4K) and 32K workloads at full size, every layer."""
    w = synth.WORKLOADS[wkey]
    inp = _inputs(w)
    cfg = prism.Config.from_workload(w)
    out, idx = prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"],
                                       want_idx=True)
    stats = {}
    layerwise_step_check(oracle, cfg, inp, out, idx, stats=stats)
    # End to end: recall of the GPU chain against the oracle's fp64 chain.
    from oracle import bf16_bits
    ref_out, ref_idx = oracle.decode_step(bf16_bits(inp["q"]), [bf16_bits(t) for t in inp["k"]],
                                          [bf16_bits(t) for t in inp["v"]],
                                          inp["lens"].cpu().numpy(), w.kappa, w.radius,
                                          w.anchor_mask())
    gi = idx.cpu().numpy()
    for l in range(w.n_layers):
        for b in range(w.batch):
            for h in range(w.n_kv_heads):
                assert recall(gi[l, b, h], ref_idx[l, b, h]) >= 0.999, (l, b, h)
    assert np.max(np.abs(out.float().cpu().numpy() - ref_out)) < 5e-2


def test_decode_step_batched_ragged(oracle):
    """The batched ragged workload's structure at reduced batch and length."""
    w = synth.WORKLOADS[4].replace(batch=4, max_len=6000, ragged=(1500, 6000), n_layers=6,
                                   kappa=256, n_clusters=16)
    inp = _inputs(w)
    cfg = prism.Config.from_workload(w)
    out, idx = prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"],
                                       want_idx=True)
    layerwise_step_check(oracle, cfg, inp, out, idx)


@pytest.mark.parametrize("mode,chain", [(prism.MODE_STATIC_REUSE, prism.CHAIN_PREV),
                                        (prism.MODE_DENSE_ANCHOR, prism.CHAIN_PREV),
                                        (prism.MODE_REFINE, prism.CHAIN_ANCHOR)])
def test_decode_step_modes(oracle, mode, chain):
    w = synth.WORKLOADS[1].replace(max_len=3000, n_layers=5, anchor_every=3)
    inp = _inputs(w)
    cfg = prism.Config.from_workload(w, mode=mode, chain=chain)
    out, idx = prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"],
                                       want_idx=True)
    layerwise_step_check(oracle, cfg, inp, out, idx)
    if mode == prism.MODE_STATIC_REUSE:
        assert torch.equal(idx[1], idx[0]) and torch.equal(idx[2], idx[0])


def test_decode_step_without_idx_out_matches(oracle):
    """idx_out is optional; the outputs are identical either way."""
    w = synth.WORKLOADS[1].replace(max_len=2500, n_layers=6, anchor_every=4)
    inp = _inputs(w)
    for chain in (prism.CHAIN_PREV, prism.CHAIN_ANCHOR):
        cfg = prism.Config.from_workload(w, chain=chain)
        out_a, _ = prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"],
                                           want_idx=True)
        out_b = prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"])
        assert torch.equal(out_a, out_b)


def test_invariants_on_gpu(oracle):
    """r = 0 equals static reuse; r >= L equals per-layer exact selection;
    kappa >= L is dense attention."""
    w = synth.WORKLOADS[1].replace(max_len=1200, n_layers=4, kappa=64)
    inp = _inputs(w)
    base = dict(n_layers=w.n_layers)
    run = lambda **kw: prism.prism_decode_step(prism.Config.from_workload(w, **{**base, **kw}),
                                               inp["q"], inp["k"], inp["v"], inp["lens"],
                                               want_idx=True)
    _, r0 = run(radius=0)
    _, st = run(mode=prism.MODE_STATIC_REUSE)
    assert torch.equal(r0, st)
    _, wide = run(radius=w.max_len)
    _, dense = run(mode=prism.MODE_DENSE_ANCHOR)
    assert torch.equal(wide, dense)
    out, idx = run(kappa=w.max_len)
    assert torch.equal(idx[:, 0, :, :w.max_len].cpu(),
                       torch.arange(w.max_len, dtype=torch.int32).expand(w.n_layers, 2, -1))
    from oracle import bf16_bits
    from helpers import sdpa_group
    qh = bf16_bits(inp["q"])
    G = w.group
    for l in range(w.n_layers):
        kh, vh = bf16_bits(inp["k"][l]), bf16_bits(inp["v"][l])
        for h in range(w.n_kv_heads):
            ref = sdpa_group(qh[l, 0, h * G:(h + 1) * G], kh[0, h], vh[0, h],
                             np.arange(w.max_len), 1.0 / math.sqrt(w.head_dim))
            got = out[l, 0, h * G:(h + 1) * G].float().cpu().numpy()
            assert np.all(np.abs(got - ref) <= 2e-2 + 1e-2 * np.abs(ref))


def test_dag_schedule_matches_serial_and_graph(oracle):
    """The multi-stream schedule, the single-stream schedule and a CUDA-graph
    replay of the step give bit-identical selections and outputs."""
    from long_context_decoding_anchor_b200.runner import DecodeStepGraph
    w = synth.WORKLOADS[2].replace(max_len=9000, n_layers=9, anchor_every=3, kappa=512)
    inp = _inputs(w)
    cfg = prism.Config.from_workload(w)
    out_d, idx_d = prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"],
                                           want_idx=True)
    cfg_s = prism.Config.from_workload(w, flags=prism.FLAG_SERIAL)
    out_s, idx_s = prism.prism_decode_step(cfg_s, inp["q"], inp["k"], inp["v"], inp["lens"],
                                           want_idx=True)
    assert torch.equal(idx_d, idx_s) and torch.equal(out_d, out_s)
    idx_g = torch.empty_like(idx_d)
    g = DecodeStepGraph(cfg, inp["q"], inp["k"], inp["v"], inp["lens"], idx_out=idx_g)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(idx_g, idx_d) and torch.equal(g.out, out_d)
    st, detail = prism.prism_check_device_status(g.ws)
    assert st == 0, detail


# -- pool mode: Eq. (9) group maximum, Eq. (4) pool, refined layers on the pool --
POOL_SHAPES = ["tiny-full", "d128-g4", "d128-g8-ragged", "d128-g16", "d64-g1", "d64-g2-batch"]


@pytest.mark.parametrize("name", POOL_SHAPES)
@pytest.mark.parametrize("rho", [2, 4])
def test_pool_stages(oracle, name, rho):
    w = SHAPES[name]
    inp = _inputs(w, layers=[0, 1])
    cfg = prism.Config.from_workload(w, mode=prism.MODE_POOL, pool_factor=rho)
    from gpu_checks import check_pool_anchor, check_pool_refine
    q0, k0, v0, lens = inp["q"][0], inp["k"][0], inp["v"][0], inp["lens"]
    S = torch.empty((w.batch, w.n_kv_heads, w.max_len), dtype=torch.float32, device="cuda")
    ws = prism.workspace(cfg)
    pool, idx0 = prism.prism_index_pool(cfg, q0, k0, lens, scores_out=S, ws=ws)
    check_pool_anchor(oracle, cfg, q0, k0, lens, pool, idx0, S)
    # the anchor entry point of pool mode scores with the group maximum too
    idx_a = prism.prism_index_anchor(cfg, q0, k0, lens, ws=ws)
    assert torch.equal(idx_a, idx0)
    q1, k1, v1 = inp["q"][1], inp["k"][1], inp["v"][1]
    idx1, cp, cs, cc = prism.prism_index_refine(cfg, q1, k1, lens, pool, cand_cap=w.max_len, ws=ws)
    check_pool_refine(oracle, cfg, q1, k1, lens, pool, idx1, cp, cs, cc)
    out1 = prism.prism_sparse_decode(cfg, q1, k1, v1, lens, idx1, ws=ws)
    check_attention(oracle, cfg, q1, k1, v1, lens, idx1, out1)
    # a shuffled pool with duplicates and padding is the same candidate set
    perm = torch.randperm(pool.shape[-1], device="cuda")
    messy = pool[..., perm].clone()
    messy[..., : pool.shape[-1] // 8] = messy[..., pool.shape[-1] // 8: pool.shape[-1] // 4]
    messy[..., -3:] = -1
    uniq = [[torch.unique(messy[b, h][messy[b, h] >= 0]) for h in range(w.n_kv_heads)]
            for b in range(w.batch)]
    idx_m, cp_m, cs_m, cc_m = prism.prism_index_refine(cfg, q1, k1, lens, messy,
                                                       cand_cap=w.max_len, ws=ws)
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            n = int(cc_m[b, h])
            assert torch.equal(cp_m[b, h, :n], uniq[b][h].to(torch.int32))
    check_pool_refine(oracle, cfg, q1, k1, lens, messy, idx_m, cp_m, cs_m, cc_m)
    st, detail = prism.prism_check_device_status(ws)
    assert st == 0, detail


@pytest.mark.parametrize("wkey,rho", [(1, 2), (1, 4), (2, 4)])
def test_pool_decode_step(oracle, wkey, rho):
    """The tiny (4K) and 32K workloads at full size in pool mode, every layer
    checked stage by stage, and the whole chain against the oracle's."""
    w = synth.WORKLOADS[wkey]
    inp = _inputs(w)
    cfg = prism.Config.from_workload(w, mode=prism.MODE_POOL, pool_factor=rho)
    out, idx = prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"],
                                       want_idx=True)
    layerwise_step_check(oracle, cfg, inp, out, idx)
    from oracle import MODE_POOL, bf16_bits
    ref_out, ref_idx = oracle.decode_step(bf16_bits(inp["q"]), [bf16_bits(t) for t in inp["k"]],
                                          [bf16_bits(t) for t in inp["v"]],
                                          inp["lens"].cpu().numpy(), w.kappa, 0,
                                          w.anchor_mask(), mode=MODE_POOL, rho=rho)
    gi = idx.cpu().numpy()
    for l in range(w.n_layers):
        for b in range(w.batch):
            for h in range(w.n_kv_heads):
                assert recall(gi[l, b, h], ref_idx[l, b, h]) >= 0.999, (l, b, h)
    assert np.max(np.abs(out.float().cpu().numpy() - ref_out)) < 5e-2


def test_pool_decode_step_batched_ragged(oracle):
    w = synth.WORKLOADS[4].replace(batch=4, max_len=6000, ragged=(1500, 6000), n_layers=6,
                                   kappa=256, n_clusters=16)
    inp = _inputs(w)
    cfg = prism.Config.from_workload(w, mode=prism.MODE_POOL, pool_factor=4)
    out, idx = prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"],
                                       want_idx=True)
    layerwise_step_check(oracle, cfg, inp, out, idx)


def test_pool_invariants_on_gpu(oracle):
    """rho * kappa >= L: every refined layer selects exactly (= anchors
    everywhere); rho = 1: every refined layer keeps its anchor's selection."""
    w = synth.WORKLOADS[1].replace(max_len=1200, n_layers=5, kappa=64, anchor_every=3)
    inp = _inputs(w)
    run = lambda **kw: prism.prism_decode_step(
        prism.Config.from_workload(w, mode=prism.MODE_POOL, **kw), inp["q"], inp["k"], inp["v"],
        inp["lens"], want_idx=True)
    _, wide = run(pool_factor=-(-w.max_len // w.kappa))
    _, exact = run(pool_factor=2, anchor_mask=[1] * w.n_layers)
    assert torch.equal(wide, exact)
    _, r1 = run(pool_factor=1)
    mask = w.anchor_mask()
    last = 0
    for l in range(w.n_layers):
        last = l if mask[l] else last
        assert torch.equal(r1[l], r1[last]), l


def test_pool_dag_matches_serial_and_graph(oracle):
    from long_context_decoding_anchor_b200.runner import DecodeStepGraph
    w = synth.WORKLOADS[2].replace(max_len=9000, n_layers=9, anchor_every=3, kappa=512)
    inp = _inputs(w)
    cfg = prism.Config.from_workload(w, mode=prism.MODE_POOL, pool_factor=4)
    out_d, idx_d = prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"],
                                           want_idx=True)
    cfg_s = prism.Config.from_workload(w, mode=prism.MODE_POOL, pool_factor=4,
                                       flags=prism.FLAG_SERIAL)
    out_s, idx_s = prism.prism_decode_step(cfg_s, inp["q"], inp["k"], inp["v"], inp["lens"],
                                           want_idx=True)
    assert torch.equal(idx_d, idx_s) and torch.equal(out_d, out_s)
    idx_g = torch.empty_like(idx_d)
    g = DecodeStepGraph(cfg, inp["q"], inp["k"], inp["v"], inp["lens"], idx_out=idx_g)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(idx_g, idx_d) and torch.equal(g.out, out_d)
    st, detail = prism.prism_check_device_status(g.ws)
    assert st == 0, detail


# -- Table 9's F/R/S layer kinds (shared layers keep the previous selection) --
from pins import TABLE9_10F11R57S, kinds_of   # noqa: E402


@pytest.mark.parametrize("mode", [prism.MODE_REFINE, prism.MODE_POOL])
def test_frs_pattern(oracle, mode):
    pattern = "FRSSRSFSRSRR"
    w = synth.WORKLOADS[2].replace(max_len=6000, n_layers=len(pattern), kappa=256, n_clusters=16)
    inp = _inputs(w)
    inp["anchor_mask"] = kinds_of(pattern)
    cfg = prism.Config.from_workload(w, mode=mode, pool_factor=4, anchor_mask=kinds_of(pattern))
    out, idx = prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"],
                                       want_idx=True)
    layerwise_step_check(oracle, cfg, inp, out, idx)
    from oracle import bf16_bits
    _, ref_idx = oracle.decode_step(bf16_bits(inp["q"]), [bf16_bits(t) for t in inp["k"]],
                                    [bf16_bits(t) for t in inp["v"]], inp["lens"].cpu().numpy(),
                                    w.kappa, w.radius, kinds_of(pattern), mode=mode, rho=4)
    gi = idx.cpu().numpy()
    for l in range(w.n_layers):
        for h in range(w.n_kv_heads):
            assert recall(gi[l, 0, h], ref_idx[l, 0, h]) >= 0.999, (l, h)
    # the same selections without idx_out (shared layers then alias their source)
    out_b = prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"])
    assert torch.equal(out, out_b)


def test_table9_hybrid_pattern_pool(oracle):
    """The paper's 78-layer 10F11R57S pattern in pool mode (rho 4) on a short
    context: every layer checked against the oracle, DAG = serial = graph."""
    from long_context_decoding_anchor_b200.runner import DecodeStepGraph
    kinds = kinds_of(TABLE9_10F11R57S)
    w = synth.WORKLOADS[2].replace(max_len=2048, n_layers=len(kinds), kappa=64, n_clusters=8)
    inp = _inputs(w)
    inp["anchor_mask"] = kinds
    cfg = prism.Config.from_workload(w, mode=prism.MODE_POOL, pool_factor=4, anchor_mask=kinds)
    out, idx = prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"],
                                       want_idx=True)
    layerwise_step_check(oracle, cfg, inp, out, idx)
    cfg_s = prism.Config.from_workload(w, mode=prism.MODE_POOL, pool_factor=4, anchor_mask=kinds,
                                       flags=prism.FLAG_SERIAL)
    out_s, idx_s = prism.prism_decode_step(cfg_s, inp["q"], inp["k"], inp["v"], inp["lens"],
                                           want_idx=True)
    assert torch.equal(idx, idx_s) and torch.equal(out, out_s)
    idx_g = torch.empty_like(idx)
    g = DecodeStepGraph(cfg, inp["q"], inp["k"], inp["v"], inp["lens"], idx_out=idx_g)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(idx_g, idx) and torch.equal(g.out, out)


# -- 2-bit proposal keys (Eq. (7)-(9)) in pool mode ---------------------------
from helpers import unpack_q2   # noqa: E402


@pytest.mark.parametrize("name", ["tiny-full", "d128-g8-ragged", "d64-g2-batch"])
def test_quantize_keys_bit_exact(oracle, name):
    """The 2-bit cache equals the oracle's quantization of every row, codes and
    alpha/beta bit for bit; positions outside [start, len) are left alone."""
    from oracle import bf16_bits
    w = SHAPES[name]
    inp = _inputs(w, layers=[0])
    cfg = prism.Config.from_workload(w, mode=prism.MODE_POOL, pool_factor=4)
    k, lens = inp["k"][0], inp["lens"]
    sentinel = 0xA5
    kq = torch.full((w.batch, w.n_kv_heads, w.max_len, w.head_dim // 2), sentinel,
                    dtype=torch.uint8, device="cuda")
    start = 5
    prism.prism_quantize_keys(cfg, k, lens, start=start, kq=kq)
    torch.cuda.synchronize()
    kqh = kq.cpu().numpy()
    lh = lens.cpu().numpy()
    for b in range(w.batch):
        L = int(lh[b])
        for h in range(w.n_kv_heads):
            codes, al, be = oracle.quantize(bf16_bits(k[b, h, start:L]))
            gc, ga, gb = unpack_q2(kqh[b, h, start:L], w.head_dim)
            assert np.array_equal(gc, codes), (b, h)
            assert np.array_equal(ga.view(np.uint32), al.view(np.uint32)), (b, h)
            assert np.array_equal(gb.view(np.uint32), be.view(np.uint32)), (b, h)
            assert np.all(kqh[b, h, :start] == sentinel) and np.all(kqh[b, h, L:] == sentinel)


def _q2_inputs(w, cfg, layers=None):
    inp = _inputs(w, layers=layers)
    inp["kq"] = [prism.prism_quantize_keys(cfg, k, inp["lens"]) for k in inp["k"]]
    return inp


@pytest.mark.parametrize("name", ["tiny-full", "d128-g4", "d128-g8-ragged", "d128-g16", "d64-g2-batch"])
def test_q2_pool_stages(oracle, name):
    from gpu_checks import check_pool_anchor, check_pool_refine
    w = SHAPES[name]
    cfg = prism.Config.from_workload(w, mode=prism.MODE_POOL, pool_factor=4,
                                     flags=prism.FLAG_INT2_KEYS)
    inp = _q2_inputs(w, cfg, layers=[0, 1])
    lens = inp["lens"]
    S = torch.empty((w.batch, w.n_kv_heads, w.max_len), dtype=torch.float32, device="cuda")
    ws = prism.workspace(cfg)
    pool, idx0 = prism.prism_index_pool(cfg, inp["q"][0], inp["kq"][0], lens, scores_out=S, ws=ws)
    check_pool_anchor(oracle, cfg, inp["q"][0], inp["k"][0], lens, pool, idx0, S, q2=True)
    idx1, cp, cs, cc = prism.prism_index_refine(cfg, inp["q"][1], inp["kq"][1], lens, pool,
                                                cand_cap=w.max_len, ws=ws)
    check_pool_refine(oracle, cfg, inp["q"][1], inp["k"][1], lens, pool, idx1, cp, cs, cc, q2=True)
    st, detail = prism.prism_check_device_status(ws)
    assert st == 0, detail


@pytest.mark.parametrize("wkey", [1, 2])
def test_q2_decode_step(oracle, wkey):
    """The tiny and 32K workloads in pool mode on 2-bit keys: stage-by-stage
    checks and the chain against the oracle's (qbits = 2)."""
    from long_context_decoding_anchor_b200.runner import DecodeStepGraph
    w = synth.WORKLOADS[wkey]
    cfg = prism.Config.from_workload(w, mode=prism.MODE_POOL, pool_factor=4,
                                     flags=prism.FLAG_INT2_KEYS)
    inp = _q2_inputs(w, cfg)
    out, idx = prism.prism_decode_step_kq(cfg, inp["q"], inp["k"], inp["v"], inp["kq"],
                                          inp["lens"], want_idx=True)
    layerwise_step_check(oracle, cfg, inp, out, idx)
    from oracle import MODE_POOL, bf16_bits
    _, ref_idx = oracle.decode_step(bf16_bits(inp["q"]), [bf16_bits(t) for t in inp["k"]],
                                    [bf16_bits(t) for t in inp["v"]], inp["lens"].cpu().numpy(),
                                    w.kappa, 0, w.anchor_mask(), mode=MODE_POOL, rho=4, qbits=2)
    gi = idx.cpu().numpy()
    for l in range(w.n_layers):
        for h in range(w.n_kv_heads):
            assert recall(gi[l, 0, h], ref_idx[l, 0, h]) >= 0.999, (l, h)
    idx_g = torch.empty_like(idx)
    g = DecodeStepGraph(cfg, inp["q"], inp["k"], inp["v"], inp["lens"], idx_out=idx_g,
                        kq_layers=inp["kq"])
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(idx_g, idx) and torch.equal(g.out, out)
