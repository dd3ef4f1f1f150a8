"""Context-parallel decode step on one GPU (ranks emulated in one process).

The R ranks of cp.decode_step_cp run one after another on one device, each on
its own shard copy of K/V and its own workspace, with local_gather standing
in for the all_gather (no kernel waits on another rank's).  Every selection
must equal the single-GPU step's bit for bit (same scoring kernels, exact
merge), and the step is checked against the oracle layer by layer as the
single-GPU step is.  Shards past a sequence's end (lengths down to 1), uneven
shards (R = 3), every mode, both chains and the F/R/S kinds are covered, and
one run goes through a real NCCL process group (one rank)."""
import math
import os
import socket

import pytest
import torch

import long_context_decoding_anchor_b200 as prism
from long_context_decoding_anchor_b200 import cp, synth
from gpu_checks import layerwise_step_check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    prism.lib()


SHAPES = {
    "d128-g4": synth.WORKLOADS[2].replace(max_len=5000, n_layers=5, kappa=200, radius=3,
                                          n_clusters=8),
    "d128-g8-ragged": synth.WORKLOADS[4].replace(batch=3, max_len=3001, n_layers=5,
                                                 n_q_heads=64, kappa=128, radius=2,
                                                 ragged=(700, 3001), n_clusters=6),
    "d64-g2-batch": synth.WORKLOADS[1].replace(batch=4, max_len=777, n_layers=5, n_q_heads=4,
                                               n_kv_heads=2, kappa=64, radius=2,
                                               ragged=(1, 777), n_clusters=3),
}
MODES = {
    # name: (Config overrides, layer kinds or None for the workload's mask)
    "refine": (dict(), None),
    "refine-chain-anchor": (dict(chain=prism.CHAIN_ANCHOR), None),
    "static-reuse": (dict(mode=prism.MODE_STATIC_REUSE), None),
    "dense-anchor": (dict(mode=prism.MODE_DENSE_ANCHOR), None),
    "pool": (dict(mode=prism.MODE_POOL, pool_factor=4), None),
    "frs": (dict(), [1, 2, 0, 2, 1]),
    "pool-frs": (dict(mode=prism.MODE_POOL, pool_factor=2), [1, 0, 2, 1, 2]),
}


def _setup(shape, mode):
    w = SHAPES[shape]
    kw, kinds = MODES[mode]
    inp = synth.make_inputs(w, device="cuda")
    if kinds is not None:
        inp["anchor_mask"] = list(kinds)
    cfg = prism.Config.from_workload(w, anchor_mask=inp["anchor_mask"], **kw)
    return w, cfg, inp


def _ranks(cfg, inp, R):
    shard_len = math.ceil(cfg.max_len / R)
    ranks = []
    for r in range(R):
        sh = prism.CpShard(R, r, shard_len)
        ks = [cp.shard_rows(k, sh) for k in inp["k"]]
        vs = [cp.shard_rows(v, sh) for v in inp["v"]]
        ranks.append(cp.CudaShard(cfg, sh, inp["q"], ks, vs, inp["lens"]))
    return ranks


def _check_status(ranks):
    for r in ranks:
        st, detail = prism.prism_check_device_status(r.ws)
        assert st == 0, f"device status {detail}"


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("shape", list(SHAPES))
def test_cp_step_equals_single_gpu_and_oracle(oracle, shape, mode):
    w, cfg, inp = _setup(shape, mode)
    out_s, idx_s = prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"],
                                           want_idx=True)
    for R in (2, 3):
        ranks = _ranks(cfg, inp, R)
        outs, sel = cp.decode_step_cp(cfg, ranks, cp.local_gather)
        torch.cuda.synchronize()
        _check_status(ranks)
        for l in range(cfg.n_layers):
            assert torch.equal(sel[l], idx_s[l]), f"R={R}, layer {l}: selection differs"
            # same selection, merged partials: within a bf16 rounding of the single-GPU output
            d = (outs[l].float() - out_s[l].float()).abs()
            assert float(d.max()) <= 2e-2, f"R={R}, layer {l}: output differs by {float(d.max())}"
    # the last (R = 3) step against the oracle, layer by layer
    rows = [(b, h) for b in range(cfg.batch) for h in range(cfg.n_kv_heads)][:6]
    layerwise_step_check(oracle, cfg, inp, torch.stack(outs), torch.stack(sel), rows=rows)


@pytest.mark.parametrize("R", [1, 4])
def test_cp_rank_counts(oracle, R):
    w, cfg, inp = _setup("d64-g2-batch", "refine")
    _, idx_s = prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"],
                                       want_idx=True)
    ranks = _ranks(cfg, inp, R)
    outs, sel = cp.decode_step_cp(cfg, ranks, cp.local_gather)
    torch.cuda.synchronize()
    _check_status(ranks)
    for l in range(cfg.n_layers):
        assert torch.equal(sel[l], idx_s[l]), f"R={R}, layer {l}"
    layerwise_step_check(oracle, cfg, inp, torch.stack(outs), torch.stack(sel))


@pytest.mark.parametrize("mode", ["refine", "pool-frs"])
@pytest.mark.parametrize("R", [1, 3])
def test_cp_attention_on_its_own_stream_matches(mode, R):
    """The attention half trailing on its own stream (second workspace per
    rank) gives the same selections and outputs as the one-stream schedule,
    eagerly and replayed from a CUDA graph."""
    w, cfg, inp = _setup("d128-g4", mode)
    ranks = _ranks(cfg, inp, R)
    outs0, sel0 = cp.decode_step_cp(cfg, ranks, cp.local_gather)
    side = torch.cuda.Stream()
    outs1, sel1 = cp.decode_step_cp(cfg, ranks, cp.local_gather, attn_stream=side)
    torch.cuda.synchronize()
    _check_status(ranks)
    for l in range(cfg.n_layers):
        assert torch.equal(sel1[l], sel0[l]), f"layer {l}: selection differs"
        assert torch.equal(outs1[l], outs0[l]), f"layer {l}: output differs"
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        outs2, sel2 = cp.decode_step_cp(cfg, ranks, cp.local_gather, attn_stream=side)
    g.replay()
    torch.cuda.synchronize()
    for l in range(cfg.n_layers):
        assert torch.equal(sel2[l], sel0[l]) and torch.equal(outs2[l], outs0[l]), f"graph, layer {l}"
    del g


def test_cp_local_scores_are_the_single_gpu_scores():
    """A shard's (position, score) pairs are the single-GPU anchor scores at
    those positions, bit for bit; the merge of all shards is the single-GPU
    selection."""
    w, cfg, inp = _setup("d128-g4", "refine")
    q, k, lens = inp["q"][0], inp["k"][0], inp["lens"]
    S = torch.empty((w.batch, w.n_kv_heads, w.max_len), dtype=torch.float32, device="cuda")
    idx = prism.prism_index_anchor(cfg, q, k, lens, scores_out=S)
    R = 3
    ranks = _ranks(cfg, inp, R)
    parts = [r.index_local(0) for r in ranks]
    for (pos, sc) in parts:
        valid = pos >= 0
        assert bool(valid.any())
        b, h, _ = torch.nonzero(valid, as_tuple=True)
        ref = S[b, h, pos[valid].long()]
        assert torch.equal(sc[valid], ref)
        assert bool(torch.isneginf(sc[~valid]).all())
    merged = ranks[0].merge(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    assert torch.equal(merged, idx)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_cp_through_an_nccl_group():
    """The exchange through torch.distributed (NCCL, one rank)."""
    import torch.distributed as dist
    w, cfg, inp = _setup("d128-g4", "pool")
    _, idx_s = prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"],
                                       want_idx=True)
    os.environ.setdefault("NCCL_NVLS_ENABLE", "0")
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1)
    try:
        ranks = _ranks(cfg, inp, 1)
        outs, sel = cp.decode_step_cp(cfg, ranks, cp.dist_gather())
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    _check_status(ranks)
    for l in range(cfg.n_layers):
        assert torch.equal(sel[l], idx_s[l])
