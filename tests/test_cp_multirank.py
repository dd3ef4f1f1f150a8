"""Context-parallel decode step on CPU ranks (gloo), each rank's shard worked
by the oracle.

cp.decode_step_cp runs its real schedule -- per layer the local selections,
an all_gather over the process group, the exact merge, the local split-softmax
partials, a second all_gather and the combine -- with OracleShard ranks in
place of the CUDA ones.  The result must equal the oracle's single-process
decode step: the selections exactly (the top-k of a union is the top-k of the
union of the parts' top-k), the outputs to fp64 rounding (split softmax).
Shards past a sequence's end, shards reaching past the capacity (4 x 80 >
300), every mode, both chains and the F/R/S layer kinds are covered."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.dirname(os.path.abspath(__file__))

CASES = {
    # name: (mode, chain, kinds, rho)
    "refine-prev": (0, 0, [1, 0, 0, 1, 0], 1),
    "refine-anchor": (0, 1, [1, 0, 0, 1, 0], 1),
    "static-reuse": (1, 0, [1, 0, 0, 1, 0], 1),
    "dense-anchor": (2, 0, [1, 1, 1, 1, 1], 1),
    "pool": (3, 0, [1, 0, 0, 1, 0], 3),
    "frs": (0, 0, [1, 2, 0, 2, 1], 1),
    "pool-frs": (3, 0, [1, 0, 2, 1, 2], 2),
}


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    """Seeded bf16 bits: B 2, Hkv 2, G 2, d 64, Lmax 300, lengths 300 and 131,
    5 layers (a salient cluster per row so selections are not arbitrary)."""
    from long_context_decoding_anchor_b200 import synth
    w = synth.WORKLOADS[1].replace(batch=2, max_len=300, n_layers=5, n_q_heads=4, n_kv_heads=2,
                                   kappa=24, radius=2, n_clusters=3, ragged=(120, 300))
    inp = synth.make_inputs(w)
    lens = inp["lens"].clone()
    lens[0], lens[1] = 300, 131
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    q = bits(inp["q"])
    ks = [bits(k) for k in inp["k"]]
    vs = [bits(v) for v in inp["v"]]
    return w, q, ks, vs, lens.numpy().astype(np.int32)


def _cfg(w, mode, chain, kinds, rho):
    import long_context_decoding_anchor_b200 as prism
    return prism.Config.make(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.max_len, w.kappa,
                             w.radius, len(kinds), kinds, mode=mode, chain=chain,
                             pool_factor=rho)


def _worker(rank, world, port, shard_len, names, q_out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    for p in (ROOT, TESTS):
        sys.path.insert(0, p)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        import oracle
        from cp_oracle_shard import OracleShard
        from long_context_decoding_anchor_b200 import cp
        o = oracle.load()
        w, q, ks, vs, lens = _inputs()
        gather = cp.dist_gather()
        res = {}
        for name in names:
            mode, chain, kinds, rho = CASES[name]
            cfg = _cfg(w, mode, chain, kinds, rho)
            me = OracleShard(o, cfg, world, rank, shard_len, q, ks, vs, lens)
            outs, sel = cp.decode_step_cp(cfg, [me], gather)
            res[name] = (np.stack([x.numpy() for x in outs]), np.stack([x.numpy() for x in sel]))
        q_out.put((rank, res))
    finally:
        dist.destroy_process_group()


def _run(world, shard_len, names):
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, shard_len, names, q_out))
             for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q_out.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


@pytest.mark.parametrize("world,shard_len", [(2, 150), (3, 100), (4, 80)])
def test_cp_schedule_matches_single_process(oracle, world, shard_len):
    names = list(CASES)
    res = _run(world, shard_len, names)
    w, q, ks, vs, lens = _inputs()
    for name in names:
        mode, chain, kinds, rho = CASES[name]
        ref_out, ref_idx = oracle.decode_step(q, ks, vs, lens, w.kappa, w.radius, kinds,
                                              mode=mode, chain=chain, rho=rho)
        for rank in range(world):
            out, idx = res[rank][name]
            np.testing.assert_array_equal(idx, ref_idx, err_msg=f"{name}, rank {rank}")
            np.testing.assert_allclose(out, ref_out, rtol=1e-12, atol=1e-12,
                                       err_msg=f"{name}, rank {rank}")


def test_layer_kinds_and_shard_rows():
    """Host helpers of the schedule: the layer kinds it walks and the shard
    copy of a cache (rows past the capacity are zero)."""
    import long_context_decoding_anchor_b200 as prism
    from long_context_decoding_anchor_b200 import cp
    c = prism.Config.make(1, 4, 2, 64, 300, 8, 1, 4, [1, 0, 2, 1])
    assert cp.layer_kinds(c) == [1, 0, 2, 1]
    d = prism.Config.make(1, 4, 2, 64, 300, 8, 1, 3, None, mode=prism.MODE_DENSE_ANCHOR)
    assert cp.layer_kinds(d) == [1, 1, 1]
    for bad in ([0, 1, 1, 1], [1, 3, 0, 0]):
        with pytest.raises(ValueError):
            cp.layer_kinds(prism.Config.make(1, 4, 2, 64, 300, 8, 1, 4, bad))
    with pytest.raises(ValueError):
        cp.layer_kinds(prism.Config.make(1, 4, 2, 64, 300, 8, 1, 4, None))
    t = torch.arange(2 * 3 * 10 * 2, dtype=torch.float32).reshape(2, 3, 10, 2)
    sh = prism.CpShard(3, 2, 4)                    # rows 8..11 of a capacity of 10
    part = cp.shard_rows(t, sh)
    assert part.shape == (2, 3, 4, 2)
    assert torch.equal(part[:, :, :2], t[:, :, 8:10])
    assert bool((part[:, :, 2:] == 0).all())
    assert torch.equal(cp.local_gather([t[0], t[1]]), t)


@pytest.mark.parametrize("world,shard_len", [(1, 300), (2, 151), (5, 61)])
def test_cp_schedule_emulated_ranks(oracle, world, shard_len):
    """The same schedule with every rank in one process (local_gather), as the
    one-GPU tests run it, against the oracle's single-process step."""
    from cp_oracle_shard import OracleShard
    from long_context_decoding_anchor_b200 import cp
    w, q, ks, vs, lens = _inputs()
    for name in ("refine-prev", "pool", "frs"):
        mode, chain, kinds, rho = CASES[name]
        cfg = _cfg(w, mode, chain, kinds, rho)
        ranks = [OracleShard(oracle, cfg, world, r, shard_len, q, ks, vs, lens)
                 for r in range(world)]
        outs, sel = cp.decode_step_cp(cfg, ranks, cp.local_gather)
        ref_out, ref_idx = oracle.decode_step(q, ks, vs, lens, w.kappa, w.radius, kinds,
                                              mode=mode, chain=chain, rho=rho)
        np.testing.assert_array_equal(np.stack([x.numpy() for x in sel]), ref_idx, err_msg=name)
        np.testing.assert_allclose(np.stack([x.numpy() for x in outs]), ref_out, rtol=1e-12,
                                   atol=1e-12, err_msg=name)
