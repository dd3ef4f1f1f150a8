#!/usr/bin/env python
"""Benchmark: Prism Attention decode step at 128K context on B200.

Workload (the 128K long-context decode): batch 1, context 131072, 32 layers
(anchor every 4), 32 query / 8 KV heads, head_dim 128, kappa 2048, r 8, bf16
KV cache (~17 GB) from the seeded synthetic generator.  A step is one
prism_decode_step over all 32 layers (anchor scoring + exact top-kappa on
anchor layers, +-r proposal / rescoring / top-kappa on refined layers, sparse
GQA attention on every layer), replayed from a CUDA graph with every input
already in HBM.  Every step touches ~4 GB of distinct K/V bytes, far more than
the 126 MB L2, so no flush is needed between steps.

One JSON line on rank 0.  ``--impl reference`` times the oracle (plain C,
fp64) on the host cores instead, on a bounded sample of the same workload.
Multi-GPU (torchrun): every rank runs its own replica (no collective on the
data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("decode-step µs/layer at 128K ctx; index+attn HBM GB/s as fraction of "
          "B200 peak")
UNIT = "us/layer"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["prism", "reference"], default="prism")
    ap.add_argument("--workload", type=int, default=3)
    ap.add_argument("--no-graph", action="store_true", help="time eager launches")
    ap.add_argument("--cpu-layers", type=int, default=16,
                    help="layers of the workload in the CPU-baseline sample")
    ap.add_argument("--ref-layers", type=int, default=8,
                    help="layers per step of the reference (oracle) arm")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-q2", action="store_true", help="skip the 2-bit key measurement")
    ap.add_argument("--configs", default="2,4,5",
                    help="other workloads measured into per_config ('' to skip)")
    ap.add_argument("--skip-cp", action="store_true",
                    help="skip the context-parallel measurement (512K workload)")
    ap.add_argument("--profile", action="store_true",
                    help="only run --steps eager decode steps (for ncu captures)")
    ap.add_argument("--layers", type=int, default=0,
                    help="override the workload's layer count (profiling a smaller case)")
    ap.add_argument("--pool", type=int, default=4,
                    help="rho of the pool-mode measurement (0: skip it)")
    ap.add_argument("--mode", choices=["refine", "refine-chain", "pool", "pool-int2"],
                    default="refine",
                    help="decode-step mode of a --profile run (refine-chain: one anchor at "
                         "layer 0, every other layer refined; pool uses --pool as rho; "
                         "pool-int2 scores on 2-bit keys)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.path = tempfile.mktemp(prefix="prism_clocks_", suffix=".csv")
        self.proc = None
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", gpu_id], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_id_for(dev) -> str:
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev.index or 0)


# --------------------------------------------------------------------------- ranks
def max_over_ranks(x: float, device) -> float:
    """The largest of every rank's x (a time); x itself with a single rank."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_us_per_layer(ms_per_step: float, n_layers: int, world: int) -> float:
    """Every rank runs its own replica of the step (no collective on the data
    path), so the job processes world * n_layers layers per step time."""
    return ms_per_step * 1e3 / (n_layers * world)


def barrier_if_distributed():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


# --------------------------------------------------------------------------- helpers
def anchor_bytes(w, lens):
    return int(sum(int(L) for L in lens)) * w.n_kv_heads * w.head_dim * 2


def selection_recall(sel, exact) -> list:
    """Per (batch, KV head) row: the fraction of the exact top-kappa `exact`
    (-1 padded) that the selection `sel` holds.  For a refined layer this is
    the coverage of the layer's own top-kappa by its proposal (the quantity of
    the paper's Fig. 3): an exact top-kappa token inside the proposal ranks
    among the proposal's kappa best and is selected."""
    import torch
    s_all = sel.reshape(-1, sel.shape[-1]).cpu()
    e_all = exact.reshape(-1, exact.shape[-1]).cpu()
    out = []
    for s_row, e_row in zip(s_all, e_all):
        e_row = e_row[e_row >= 0]
        s_row = s_row[s_row >= 0]
        out.append(float(torch.isin(e_row, s_row).sum()) / max(1, e_row.numel()))
    return out


def proposal_counts(prism, cfg, inp, idx, mask, ws) -> list:
    """Per refined layer: the proposal size |P| of every (batch, KV head) row
    (int tensor on the host), from the public refine call's candidate count."""
    out = []
    for l in range(cfg.n_layers):
        if mask[l]:
            continue
        _, _, _, cc = prism.prism_index_refine(cfg, inp["q"][l], inp["k"][l], inp["lens"],
                                               idx[l - 1].contiguous(), cand_cap=1, ws=ws)
        out.append(cc.flatten().cpu())
    return out


def graph_step_ms(prism, cfg, inp, reps, dev, ws=None):
    """Mean device time (CUDA events) of one CUDA-graph replay of the step."""
    import torch
    from long_context_decoding_anchor_b200.runner import DecodeStepGraph
    n = cfg.n_layers
    r = DecodeStepGraph(cfg, inp["q"][:n], inp["k"][:n], inp["v"][:n], inp["lens"], ws=ws)
    for _ in range(3):
        r.replay()
    stream = torch.cuda.current_stream(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    a.record(stream)
    for _ in range(reps):
        r.replay()
    b.record(stream)
    torch.cuda.synchronize(dev)
    launches = r.launches
    del r
    return a.elapsed_time(b) / reps, launches


def anchor_kernel_s(prism, cfg, inp, anchors, ws, reps, dev):
    """Mean seconds of one prism_score_anchor launch (a single scoring kernel),
    CUDA events around each launch on the launching stream."""
    import ctypes

    import torch
    L = prism.lib()
    stream = torch.cuda.current_stream(dev)
    S = torch.empty((cfg.batch, cfg.n_kv_heads, cfg.max_len), dtype=torch.float32, device=dev)
    cfgp = ctypes.byref(cfg)

    def launch(l):
        rc = L.prism_score_anchor(cfgp, ctypes.c_void_p(inp["q"][l].data_ptr()),
                                  ctypes.c_void_p(inp["k"][l].data_ptr()),
                                  ctypes.c_void_p(inp["lens"].data_ptr()),
                                  ctypes.c_void_p(S.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
                                  ws.numel(), ctypes.c_void_p(stream.cuda_stream))
        if rc != 0:
            raise RuntimeError(f"prism_score_anchor: {rc}")
    for i in range(3):
        launch(anchors[i % len(anchors)])
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for i in range(reps):
        evs[i][0].record(stream)
        launch(anchors[i % len(anchors)])
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    del S
    return statistics.mean(a.elapsed_time(b) for a, b in evs) * 1e-3


def kernel_table(replay, dev) -> dict:
    """Per kernel of one replay: launches, total and mean device microseconds
    (CUPTI activity records through torch.profiler; no host launch cost,
    overlapping kernels each counted in full), plus the replay's span."""
    import torch
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize(dev)
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        replay()
        torch.cuda.synchronize(dev)
    fd, fn = tempfile.mkstemp(prefix="prism_trace_", suffix=".json")
    os.close(fd)
    try:
        prof.export_chrome_trace(fn)
        with open(fn) as f:
            ev = [e for e in json.load(f)["traceEvents"] if e.get("cat") == "kernel"]
    finally:
        os.unlink(fn)
    rows = {}
    for e in ev:
        name = e["name"].replace("void ", "").replace("prism::", "").split("(")[0][:60]
        r = rows.setdefault(name, [0, 0.0])
        r[0] += 1
        r[1] += float(e["dur"])
    span = (max(e["ts"] + e["dur"] for e in ev) - min(e["ts"] for e in ev)) if ev else 0.0
    return {"span_us": round(span, 2),
            "kernels": {n: {"launches": c, "total_us": round(t, 2), "mean_us": round(t / c, 3)}
                        for n, (c, t) in sorted(rows.items(), key=lambda x: -x[1][1])}}


def measure_workload(args, prism, synth, wid, dev, peak, reps, world) -> dict:
    """One of the pages' workloads at one GPU: graph-replayed step (us/layer),
    its algorithmic HBM fraction, the anchor scoring kernel's roofline, the
    refined layers alone, and the proposal sizes |P|."""
    import torch
    w = synth.WORKLOADS[wid]
    inp = synth.make_inputs(w, device=dev)
    cfg = prism.Config.from_workload(w)
    ws = prism.workspace(cfg, dev)
    N = w.n_layers
    mask = w.anchor_mask()
    lens_h = inp["lens"].cpu().tolist()
    _, idx = prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"],
                                     want_idx=True, ws=ws)
    st, detail = prism.prism_check_device_status(ws)
    if st != 0:
        raise RuntimeError(f"{w.name}: device status {st} {detail}")
    props = proposal_counts(prism, cfg, inp, idx, mask, ws)
    n_anchor = sum(mask)
    kappa_eff = sum(min(w.kappa, int(L)) for L in lens_h) * w.n_kv_heads
    gather = kappa_eff * w.head_dim * 2 * 2
    a_bytes = anchor_bytes(w, lens_h)
    prop_total = sum(int(p.sum()) for p in props)
    step_bytes = n_anchor * a_bytes + prop_total * w.head_dim * 2 + N * gather
    ms, launches = graph_step_ms(prism, cfg, inp, reps, dev, ws=ws)
    ms = max_over_ranks(ms, dev)
    anchors = [l for l in range(N) if mask[l]]
    t_a = anchor_kernel_s(prism, cfg, inp, anchors, ws, max(8, reps), dev)
    # refined layers alone: one anchor then every other layer refined, minus the anchor layer
    cfg_r = prism.Config.from_workload(w, anchor_mask=[1] + [0] * (N - 1))
    cfg_0 = prism.Config.from_workload(w.replace(n_layers=1))
    t_r, _ = graph_step_ms(prism, cfg_r, inp, reps, dev)
    t_0, _ = graph_step_ms(prism, cfg_0, inp, reps, dev)
    _, idx_r = prism.prism_decode_step(cfg_r, inp["q"], inp["k"], inp["v"], inp["lens"],
                                       want_idx=True, ws=ws)
    props_r = proposal_counts(prism, cfg_r, inp, idx_r, [1] + [0] * (N - 1), ws)
    r_us = (t_r - t_0) * 1e3 / (N - 1)
    r_bytes = statistics.mean(int(p.sum()) for p in props_r) * w.head_dim * 2 + gather
    allp = torch.cat(props).float() if props else torch.zeros(1)
    step_gbs = step_bytes / (ms * 1e-3) / 1e9
    res = {
        "workload": f"{w.name}: {w.describe()}",
        "value": whole_job_us_per_layer(ms, N, world), "unit": UNIT, "ms_per_step": ms,
        "launches_per_step": launches,
        "anchor_kernel": {"bound": "hbm", "achieved": a_bytes / t_a / 1e9, "peak": peak,
                          "unit": "GB/s", "frac": a_bytes / t_a / 1e9 / peak,
                          "us_per_launch": t_a * 1e6, "bytes_per_launch": a_bytes},
        "proposal": {"mean_per_row": float(allp.mean()), "max_per_row": int(allp.max()),
                     "min_per_row": int(allp.min()),
                     "kappa_2r1": w.kappa * (2 * w.radius + 1)},
        "refine_attn": {"bytes_per_layer": r_bytes, "us_per_layer": r_us,
                        "frac": r_bytes / (r_us * 1e-6) / 1e9 / peak},
        "step_hbm": {"algorithmic_bytes": step_bytes, "gbs": step_gbs, "frac": step_gbs / peak},
    }
    del inp, ws, idx, idx_r
    torch.cuda.empty_cache()
    return res


def kernel_traffic(src_paths, profile_md):
    """DRAM bytes per launch of the anchor scoring kernel from a committed ncu
    summary, valid only while the kernel's sources are unchanged."""
    try:
        text = open(profile_md).read()
    except OSError:
        return None
    h = hashlib.sha256()
    for p in src_paths:
        h.update(open(p, "rb").read())
    m_sha = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    m_tr = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", text)
    if not m_sha or not m_tr or m_sha.group(1) != h.hexdigest():
        return None
    return int(m_tr.group(1))


def oracle_sample(w, inp, layers, heads):
    """Host copies (uint16 bits) of layers x KV heads of the workload."""
    from oracle import bf16_bits
    G = w.group
    h0, h1 = heads
    q = bf16_bits(inp["q"][layers[0]:layers[-1] + 1, :, h0 * G:h1 * G])
    ks = [bf16_bits(inp["k"][l][:, h0:h1]) for l in layers]
    vs = [bf16_bits(inp["v"][l][:, h0:h1]) for l in layers]
    lens = inp["lens"].cpu().numpy()
    mask = [inp["anchor_mask"][l] for l in layers]
    return q, ks, vs, lens, mask


def host_cpu() -> dict:
    """The host's CPU model and logical core count (for the CPU baseline)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"model": model, "nproc": os.cpu_count()}


def time_oracle(w, sample, reps=1, threads=None):
    """Seconds per pass of the oracle's decode step over `sample`, and the
    threads it used (all host cores unless `threads` is given)."""
    import oracle
    o = oracle.load()
    q, ks, vs, lens, mask = sample
    full = o.num_threads()
    if threads:
        o.set_num_threads(threads)
    try:
        used = o.num_threads()
        t0 = time.perf_counter()
        for _ in range(reps):
            o.decode_step(q, ks, vs, lens, w.kappa, w.radius, mask)
        return (time.perf_counter() - t0) / reps, used
    finally:
        if threads:
            o.set_num_threads(full)


# --------------------------------------------------------------------------- arms
def run_reference(args, rank, world):
    """The oracle on the host cores, on a bounded sample of the workload."""
    import torch
    from long_context_decoding_anchor_b200 import synth
    if rank != 0:
        return
    w = synth.WORKLOADS[args.workload]
    layers = list(range(args.ref_layers))
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = synth.make_inputs(w, device=dev, layers=layers)
    sample = oracle_sample(w, inp, layers, (0, w.n_kv_heads))
    del inp
    for _ in range(args.warmup):
        time_oracle(w, sample)
    times = []
    threads = 1
    for _ in range(args.steps):
        t, threads = time_oracle(w, sample)
        times.append(t)
    ms = statistics.mean(times) * 1e3
    value = ms * 1e3 / len(layers)
    n_anchor = sum(w.anchor_mask()[:len(layers)])
    cores = min(threads, w.rows)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": f"{w.name}: {w.describe()}", "sample_layers": layers,
                   "kv_heads": w.n_kv_heads},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "host": host_cpu(),
                         "sample": f"layers {layers[0]}-{layers[-1]} ({n_anchor} anchor + "
                                   f"{len(layers) - n_anchor} refined) x all {w.n_kv_heads} KV "
                                   f"heads of the 128K workload, per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def measure_context_parallel(args, rank, world, dev):
    """The context-parallel step (cp.decode_step_cp) on the 512K workload,
    its context split over the job's ranks (strong scaling: total work fixed).
    Eager schedule timed with CUDA events (max over ranks); with one rank also
    replayed from a CUDA graph, beside the single-GPU step's graph."""
    import math

    import torch
    import long_context_decoding_anchor_b200 as prism
    from long_context_decoding_anchor_b200 import cp, synth
    from long_context_decoding_anchor_b200.runner import DecodeStepGraph

    w = synth.WORKLOADS[5]
    inp = synth.make_inputs(w, device=dev)
    cfg = prism.Config.from_workload(w)
    R, N = world, w.n_layers
    shard_len = math.ceil(w.max_len / R)
    sh = prism.CpShard(R, rank, shard_len)
    if R == 1:
        ks, vs = inp["k"], inp["v"]
    else:
        ks = [cp.shard_rows(k, sh) for k in inp["k"]]
        vs = [cp.shard_rows(v, sh) for v in inp["v"]]
        inp["k"] = inp["v"] = None
        torch.cuda.empty_cache()
    me = cp.CudaShard(cfg, sh, inp["q"], ks, vs, inp["lens"])
    gather = cp.local_gather if R == 1 else cp.dist_gather()
    # the attention half trails on its own stream, with its own exchange group
    attn_gather = cp.local_gather if R == 1 else cp.dist_gather(torch.distributed.new_group())
    side = torch.cuda.Stream(device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        return cp.decode_step_cp(cfg, [me], gather, attn_stream=side, attn_gather=attn_gather)

    n0 = prism.lib().prism_launch_count()
    _, sel = step()
    launches = int(prism.lib().prism_launch_count() - n0)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    st, detail = prism.prism_check_device_status(me.ws)
    if st != 0:
        raise RuntimeError(f"context-parallel step: device status {st} {detail}")
    barrier_if_distributed()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    ms_eager = max_over_ranks(a.elapsed_time(b) / args.steps, dev)
    res = {
        "workload": f"{w.name}: {w.describe()}", "ranks": R, "shard_len": shard_len,
        "scaling": "strong", "launches_per_step": launches,
        "eager_us_per_layer": ms_eager * 1e3 / N,
        "exchange_bytes_per_layer_per_rank": {
            "selection": w.rows * w.kappa * 8,
            "attention_partials": w.batch * w.n_q_heads * (w.head_dim + 2) * 4},
        "how": "per layer: shard-local selection (+ scores), all_gather, exact merge; "
               "shard-local split-softmax partials, all_gather, combine (the attention half "
               "on a second stream behind the merge)",
    }
    if R == 1:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(args.steps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize(dev)
        res["graph_us_per_layer"] = a.elapsed_time(b) / args.steps * 1e3 / N
        single = DecodeStepGraph(cfg, inp["q"], inp["k"], inp["v"], inp["lens"])
        for _ in range(3):
            single.replay()
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(args.steps):
            single.replay()
        b.record(stream)
        torch.cuda.synchronize(dev)
        res["single_gpu_graph_us_per_layer"] = a.elapsed_time(b) / args.steps * 1e3 / N
        _, idx_s = prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"],
                                           want_idx=True)
        res["selections_equal_single_gpu"] = all(torch.equal(sel[l], idx_s[l]) for l in range(N))
        # algorithmic HBM bytes of the step (as for the headline step: anchor K, measured
        # proposal K rows, gathered K/V rows) over the graph-replayed time
        mask = w.anchor_mask()
        lens_h = inp["lens"].cpu().tolist()
        props = []
        for l in range(N):
            if not mask[l]:
                _, _, _, cc = prism.prism_index_refine(cfg, inp["q"][l], inp["k"][l], inp["lens"],
                                                       idx_s[l - 1].contiguous(), cand_cap=1)
                props.append(int(cc.sum()))
        kappa_eff = sum(min(w.kappa, int(L)) for L in lens_h) * w.n_kv_heads
        step_bytes = (sum(mask) * anchor_bytes(w, lens_h) + sum(props) * w.head_dim * 2
                      + N * kappa_eff * w.head_dim * 4)
        peak, peak_kind = peaks()
        for key in ("graph_us_per_layer", "single_gpu_graph_us_per_layer"):
            gbs = step_bytes / (res[key] * N * 1e-6) / 1e9
            res[key.replace("us_per_layer", "step_hbm")] = {"gbs": gbs, "frac": gbs / peak}
        res["step_algorithmic_bytes"] = step_bytes
        res["peak"] = {"gbs": peak, "kind": peak_kind}
        del g, single
    return res


def run_prism(args, rank, world, dev):
    import torch
    import long_context_decoding_anchor_b200 as prism
    from long_context_decoding_anchor_b200 import build as prism_build, synth
    from long_context_decoding_anchor_b200.runner import DecodeStepGraph

    if not os.path.exists(prism.LIB_PATH):
        prism_build.build()
    prism.lib()
    w = synth.WORKLOADS[args.workload]
    if args.layers:
        w = w.replace(n_layers=args.layers)
    inp = synth.make_inputs(w, device=dev)
    if args.profile:
        pool_run = args.mode in ("pool", "pool-int2")
        q2_run = args.mode == "pool-int2"
        chain = [1] + [0] * (w.n_layers - 1) if args.mode == "refine-chain" else None
        cfg = (prism.Config.from_workload(w, mode=prism.MODE_POOL, pool_factor=args.pool,
                                          flags=prism.FLAG_INT2_KEYS if q2_run else 0)
               if pool_run else prism.Config.from_workload(
                   w, **({"anchor_mask": chain} if chain else {})))
        ws = prism.workspace(cfg, dev)
        kq = [prism.prism_quantize_keys(cfg, kk, inp["lens"], ws=ws) for kk in inp["k"]] \
            if q2_run else None
        for _ in range(args.steps):
            if q2_run:
                prism.prism_decode_step_kq(cfg, inp["q"], inp["k"], inp["v"], kq, inp["lens"],
                                           ws=ws)
            else:
                prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"], ws=ws)
        torch.cuda.synchronize(dev)
        st, detail = prism.prism_check_device_status(ws)
        if st != 0:
            raise RuntimeError(f"device status {st} {detail}")
        print(f"profile run: {args.steps} eager steps of {w.name} ({w.n_layers} layers, "
              f"{args.mode}, rho {args.pool})")
        return
    cfg = prism.Config.from_workload(w)
    ws = prism.workspace(cfg, dev)
    N = w.n_layers
    lens_h = inp["lens"].cpu().tolist()
    torch.cuda.synchronize(dev)

    # -- eager reference run: selections (for |P| accounting) and status check
    out_e, idx_e = prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"],
                                           want_idx=True, ws=ws)
    st, detail = prism.prism_check_device_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st} {detail}")
    mask = w.anchor_mask()
    prop_sizes = []
    refine_diag = []
    for l in range(N):
        if mask[l]:
            continue
        _, _, _, cc = prism.prism_index_refine(cfg, inp["q"][l], inp["k"][l], inp["lens"],
                                               idx_e[l - 1].contiguous(), cand_cap=1, ws=ws)
        prop_sizes.append(int(cc.sum()))
        # the layer's own exact top-kappa (an anchor selection of this layer), for recall
        try:
            exact = prism.prism_index_anchor(cfg, inp["q"][l], inp["k"][l], inp["lens"], ws=ws)
            rec = selection_recall(idx_e[l], exact)
            refine_diag.append({"layer": l, "proposal_mean_per_row": float(cc.float().mean()),
                                "proposal_max_per_row": int(cc.max()),
                                "recall_mean": statistics.mean(rec), "recall_min": min(rec)})
        except Exception as e:          # a diagnostic: never costs the line
            refine_diag.append({"layer": l, "error": f"{type(e).__name__}: {e}"})
    n_anchor = sum(mask)
    kappa_eff = sum(min(w.kappa, int(L)) for L in lens_h) * w.n_kv_heads
    gather = kappa_eff * w.head_dim * 2 * 2
    a_bytes = anchor_bytes(w, lens_h)
    step_bytes = n_anchor * a_bytes + sum(prop_sizes) * w.head_dim * 2 + N * gather

    # -- the timed step: CUDA-graph replay of the whole decode step
    if args.no_graph:
        runner = None
        launches_per_step = None

        def step():
            prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"], out=out_e,
                                    ws=ws)
        n0 = prism.lib().prism_launch_count()
        step()
        launches_per_step = int(prism.lib().prism_launch_count() - n0)
    else:
        runner = DecodeStepGraph(cfg, inp["q"], inp["k"], inp["v"], inp["lens"], ws=ws)
        launches_per_step = runner.launches
        step = runner.replay
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    barrier_if_distributed()
    clocks = ClockSampler(gpu_id_for(dev))
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / args.steps
    barrier_if_distributed()
    clk = clocks.stop()
    ms = max_over_ranks(ms, dev)
    st, detail = prism.prism_check_device_status(ws)
    if st != 0:
        raise RuntimeError(f"device status after timing {st} {detail}")
    value = whole_job_us_per_layer(ms, N, world)
    peak, peak_kind = peaks()
    step_gbs = step_bytes / (ms * 1e-3) / 1e9

    # -- dominant kernel: anchor scoring alone, CUDA events around each launch
    anchors = [l for l in range(N) if mask[l]]
    S = torch.empty((w.batch, w.n_kv_heads, w.max_len), dtype=torch.float32, device=dev)
    L = prism.lib()
    import ctypes
    cfgp = ctypes.byref(cfg)

    def score_launch(l):
        rc = L.prism_score_anchor(cfgp, ctypes.c_void_p(inp["q"][l].data_ptr()),
                                  ctypes.c_void_p(inp["k"][l].data_ptr()),
                                  ctypes.c_void_p(inp["lens"].data_ptr()),
                                  ctypes.c_void_p(S.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
                                  ws.numel(), ctypes.c_void_p(stream.cuda_stream))
        if rc != 0:
            raise RuntimeError(f"prism_score_anchor: {rc}")
    for i in range(3):
        score_launch(anchors[i % len(anchors)])
    n_k = max(args.steps, 16)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n_k)]
    for i in range(n_k):
        evs[i][0].record(stream)
        score_launch(anchors[i % len(anchors)])
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    t_score = statistics.mean(a.elapsed_time(b) for a, b in evs) * 1e-3
    ach = a_bytes / t_score / 1e9

    # -- refined layers alone (the second roofline target): the same step with
    #    one anchor at layer 0 and every other layer refined, minus the step of
    #    layer 0 alone; bytes = the measured proposals + the gathered K/V rows
    def graph_ms(c, reps):
        r = DecodeStepGraph(c, inp["q"][:c.n_layers], inp["k"][:c.n_layers],
                            inp["v"][:c.n_layers], inp["lens"])
        for _ in range(3):
            r.replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(reps):
            r.replay()
        b.record(stream)
        torch.cuda.synchronize(dev)
        del r
        return a.elapsed_time(b) / reps
    cfg_r = prism.Config.from_workload(w, anchor_mask=[1] + [0] * (N - 1))
    cfg_0 = prism.Config.from_workload(w.replace(n_layers=1))
    t_r = graph_ms(cfg_r, max(5, args.steps // 2))
    t_0 = graph_ms(cfg_0, max(5, args.steps // 2))
    _, idx_r = prism.prism_decode_step(cfg_r, inp["q"], inp["k"], inp["v"], inp["lens"],
                                       want_idx=True, ws=ws)
    props_r = []
    for l in range(1, N):
        _, _, _, cc = prism.prism_index_refine(cfg_r, inp["q"][l], inp["k"][l], inp["lens"],
                                               idx_r[l - 1].contiguous(), cand_cap=1, ws=ws)
        props_r.append(int(cc.sum()))
    refine_us = (t_r - t_0) * 1e3 / (N - 1)
    refine_bytes = statistics.mean(props_r) * w.head_dim * 2 + gather
    score_src = [os.path.join(ROOT, "long_context_decoding_anchor_b200", "csrc", f)
                 for f in ("score.cu", "prism_internal.cuh")]
    traffic = kernel_traffic(score_src, os.path.join(ROOT, "profiles", "anchor_score_128k.md"))

    # -- pool mode (the paper's own proposal: Eq. (9) group maximum, Eq. (4)
    #    pool of rho*kappa tokens, refined layers rescore the anchor's pool)
    pool = None
    if args.pool > 0:
        rho = args.pool
        cfg_p = prism.Config.from_workload(w, mode=prism.MODE_POOL, pool_factor=rho)
        ws_p = prism.workspace(cfg_p, dev)
        rp = DecodeStepGraph(cfg_p, inp["q"], inp["k"], inp["v"], inp["lens"], ws=ws_p)
        for _ in range(max(3, args.warmup)):
            rp.replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(args.steps):
            rp.replay()
        b.record(stream)
        torch.cuda.synchronize(dev)
        ms_p = max_over_ranks(a.elapsed_time(b) / args.steps, dev)
        launches_p = rp.launches
        del rp
        st, detail = prism.prism_check_device_status(ws_p)
        if st != 0:
            raise RuntimeError(f"device status after the pool-mode step {st} {detail}")
        cfgpp = ctypes.byref(cfg_p)

        def score_max_launch(l):
            rc = L.prism_score_anchor(cfgpp, ctypes.c_void_p(inp["q"][l].data_ptr()),
                                      ctypes.c_void_p(inp["k"][l].data_ptr()),
                                      ctypes.c_void_p(inp["lens"].data_ptr()),
                                      ctypes.c_void_p(S.data_ptr()),
                                      ctypes.c_void_p(ws_p.data_ptr()), ws_p.numel(),
                                      ctypes.c_void_p(stream.cuda_stream))
            if rc != 0:
                raise RuntimeError(f"prism_score_anchor (pool mode): {rc}")
        for i in range(3):
            score_max_launch(anchors[i % len(anchors)])
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n_k)]
        for i in range(n_k):
            evs[i][0].record(stream)
            score_max_launch(anchors[i % len(anchors)])
            evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
        t_max = statistics.mean(x.elapsed_time(y) for x, y in evs) * 1e-3
        # MMA work per launch: every key row against the 16 padded head columns
        tc_flops = 2.0 * sum(int(x) for x in lens_h) * w.n_kv_heads * 16 * w.head_dim
        cfg_pr = prism.Config.from_workload(w, mode=prism.MODE_POOL, pool_factor=rho,
                                            anchor_mask=[1] + [0] * (N - 1))
        cfg_p0 = prism.Config.from_workload(w.replace(n_layers=1), mode=prism.MODE_POOL,
                                            pool_factor=rho)
        t_pr = graph_ms(cfg_pr, max(5, args.steps // 2))
        t_p0 = graph_ms(cfg_p0, max(5, args.steps // 2))
        pool_rows = sum(min(rho * w.kappa, int(x)) for x in lens_h) * w.n_kv_heads
        p_refine_bytes = pool_rows * w.head_dim * 2 + gather
        p_refine_us = (t_pr - t_p0) * 1e3 / (N - 1)
        p_step_bytes = n_anchor * a_bytes + (N - n_anchor) * pool_rows * w.head_dim * 2 + N * gather
        max_src = [os.path.join(ROOT, "long_context_decoding_anchor_b200", "csrc", f)
                   for f in ("score_max.cu", "tc_sm100.cuh", "tiles.cuh", "prism_internal.cuh")]
        traffic_max = kernel_traffic(max_src, os.path.join(ROOT, "profiles", "anchor_score_max_128k.md"))
        pool = {
            "rho": rho, "value": whole_job_us_per_layer(ms_p, N, world), "unit": UNIT,
            "ms_per_step": ms_p, "launches_per_step": launches_p,
            "step_hbm": {"algorithmic_bytes": p_step_bytes,
                         "gbs": p_step_bytes / (ms_p * 1e-3) / 1e9,
                         "frac": p_step_bytes / (ms_p * 1e-3) / 1e9 / peak},
            "anchor_kernel": {"kernel": "k_anchor_score_max (tcgen05)", "bound": "hbm",
                              "achieved": a_bytes / t_max / 1e9, "peak": peak, "unit": "GB/s",
                              "frac": a_bytes / t_max / 1e9 / peak,
                              "us_per_launch": t_max * 1e6, "bytes_per_launch": a_bytes,
                              "traffic": traffic_max,
                              "tensor_tflops": tc_flops / t_max / 1e12},
            "refine_attn": {"bytes_per_layer": p_refine_bytes, "us_per_layer": p_refine_us,
                            "gbs": p_refine_bytes / (p_refine_us * 1e-6) / 1e9,
                            "frac": p_refine_bytes / (p_refine_us * 1e-6) / 1e9 / peak},
            "how": "pool mode (Eq. (9) group maximum, rho*kappa pool) on the same workload "
                   "and inputs, graph-timed like the headline step",
        }

    # -- pool mode on 2-bit proposal keys (Eq. (7)-(9)): the anchor scans and
    #    the pool rescoring read the 2-bit cache, attention the bf16 keys
    pool_q2 = None
    if args.pool > 0 and not args.skip_q2:
        rho = args.pool
        cfg_q = prism.Config.from_workload(w, mode=prism.MODE_POOL, pool_factor=rho,
                                           flags=prism.FLAG_INT2_KEYS)
        ws_q = prism.workspace(cfg_q, dev)
        kq = [prism.prism_quantize_keys(cfg_q, kk, inp["lens"], ws=ws_q) for kk in inp["k"]]
        # the append-time quantizer, timed per layer (not part of a decode step)
        qa, qb_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        qa.record(stream)
        for kk, kqq in zip(inp["k"], kq):
            prism.prism_quantize_keys(cfg_q, kk, inp["lens"], kq=kqq, ws=ws_q, stream=stream)
        qb_.record(stream)
        torch.cuda.synchronize(dev)
        t_quant = qa.elapsed_time(qb_) * 1e3 / N
        rq = DecodeStepGraph(cfg_q, inp["q"], inp["k"], inp["v"], inp["lens"], ws=ws_q,
                             kq_layers=kq)
        for _ in range(max(3, args.warmup)):
            rq.replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(args.steps):
            rq.replay()
        b.record(stream)
        torch.cuda.synchronize(dev)
        ms_q = max_over_ranks(a.elapsed_time(b) / args.steps, dev)
        launches_q = rq.launches
        del rq
        st, detail = prism.prism_check_device_status(ws_q)
        if st != 0:
            raise RuntimeError(f"device status after the 2-bit pool step {st} {detail}")
        cfgqp = ctypes.byref(cfg_q)

        def score_q2_launch(l):
            rc = L.prism_score_anchor(cfgqp, ctypes.c_void_p(inp["q"][l].data_ptr()),
                                      ctypes.c_void_p(kq[l].data_ptr()),
                                      ctypes.c_void_p(inp["lens"].data_ptr()),
                                      ctypes.c_void_p(S.data_ptr()),
                                      ctypes.c_void_p(ws_q.data_ptr()), ws_q.numel(),
                                      ctypes.c_void_p(stream.cuda_stream))
            if rc != 0:
                raise RuntimeError(f"prism_score_anchor (2-bit keys): {rc}")
        for i in range(3):
            score_q2_launch(anchors[i % len(anchors)])
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n_k)]
        for i in range(n_k):
            evs[i][0].record(stream)
            score_q2_launch(anchors[i % len(anchors)])
            evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
        t_q2 = statistics.mean(x.elapsed_time(y) for x, y in evs) * 1e-3
        q2_bytes = sum(int(x) for x in lens_h) * w.n_kv_heads * (w.head_dim // 2)
        pool_rows_q = sum(min(rho * w.kappa, int(x)) for x in lens_h) * w.n_kv_heads
        q2_step_bytes = (n_anchor * q2_bytes + (N - n_anchor) * pool_rows_q * (w.head_dim // 2)
                         + N * gather)
        pool_q2 = {
            "rho": rho, "value": whole_job_us_per_layer(ms_q, N, world), "unit": UNIT,
            "ms_per_step": ms_q, "launches_per_step": launches_q,
            "step_hbm": {"algorithmic_bytes": q2_step_bytes,
                         "gbs": q2_step_bytes / (ms_q * 1e-3) / 1e9,
                         "frac": q2_step_bytes / (ms_q * 1e-3) / 1e9 / peak},
            "anchor_kernel": {"kernel": "k_anchor_score_q2 (mma.sync on 2-bit codes)",
                              "bound": "hbm", "achieved": q2_bytes / t_q2 / 1e9, "peak": peak,
                              "unit": "GB/s", "frac": q2_bytes / t_q2 / 1e9 / peak,
                              "us_per_launch": t_q2 * 1e6, "bytes_per_launch": q2_bytes},
            "quantize_us_per_layer": t_quant,
            "how": "pool mode on the 2-bit cache (64 B a key: codes + fp32 alpha/beta per 32), "
                   "same inputs; the quantizer runs when keys are appended, timed apart",
        }
        del kq

    # -- per-kernel breakdown: device durations (CUPTI) of every kernel of one
    #    replay of the timed step, and of one serial call of each public stage
    refines = [l for l in range(N) if not mask[l]]
    idx_tmp = torch.empty((w.batch, w.n_kv_heads, w.kappa), dtype=torch.int32, device=dev)
    out_tmp = torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device=dev)

    def stages_once():
        la, lr = anchors[0], refines[0]
        prism.prism_index_anchor(cfg, inp["q"][la], inp["k"][la], inp["lens"], idx_out=idx_tmp,
                                 ws=ws, stream=stream)
        prism.prism_index_refine(cfg, inp["q"][lr], inp["k"][lr], inp["lens"],
                                 idx_e[lr - 1].contiguous(), idx_out=idx_tmp, ws=ws,
                                 stream=stream)
        prism.prism_sparse_decode(cfg, inp["q"][lr], inp["k"][lr], inp["v"][lr], inp["lens"],
                                  idx_e[lr].contiguous(), out=out_tmp, ws=ws, stream=stream)
    br = {"how": "device time of each kernel (CUPTI activity records): 'step' over one replay "
                 "of the timed graph (kernels overlap across streams, each counted in full), "
                 "'stages' over one serial call each of prism_index_anchor, prism_index_refine "
                 "and prism_sparse_decode; anchor_score_kernel_us from CUDA events around "
                 "single launches",
          "anchor_score_kernel_us": t_score * 1e6}
    try:
        stages_once()
        br["stages"] = kernel_table(stages_once, dev)["kernels"]
        if runner is not None:
            br["step"] = kernel_table(runner.replay, dev)
    except Exception as e:              # a diagnostic: never costs the line
        br["error"] = f"{type(e).__name__}: {e}"

    # -- the same step as eager launches (no graph), inputs resident
    eager = None
    if not args.no_graph:
        for _ in range(3):
            prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"], out=out_e,
                                    ws=ws, stream=stream)
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            prism.prism_decode_step(cfg, inp["q"], inp["k"], inp["v"], inp["lens"], out=out_e,
                                    ws=ws, stream=stream)
        b.record(stream)
        torch.cuda.synchronize(dev)
        ms_eager = max_over_ranks(a.elapsed_time(b) / args.steps, dev)
        eager = {"value": whole_job_us_per_layer(ms_eager, N, world), "unit": UNIT,
                 "ms_per_step": ms_eager,
                 "how": "prism_decode_step launched eagerly each step (host launch cost included)"}

    # -- end to end through the public call, host buffers, copies in the timed region
    e2e = None
    if not args.skip_e2e:
        q_h = inp["q"].cpu().pin_memory()
        lens_hp = inp["lens"].cpu().pin_memory()
        out_h = torch.empty(out_e.shape, dtype=out_e.dtype).pin_memory()
        q_d = torch.empty_like(inp["q"])
        out_d = torch.empty_like(out_e)

        def e2e_step():
            q_d.copy_(q_h, non_blocking=True)
            inp["lens"].copy_(lens_hp, non_blocking=True)
            prism.prism_decode_step(cfg, q_d, inp["k"], inp["v"], inp["lens"], out=out_d, ws=ws,
                                    stream=stream)
            out_h.copy_(out_d, non_blocking=True)
        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        ms_e2e = max_over_ranks(a.elapsed_time(b) / args.steps, dev)
        e2e = {"value": whole_job_us_per_layer(ms_e2e, N, world), "unit": UNIT,
               "h2d_bytes_per_step": q_h.numel() * 2 + lens_hp.numel() * 4,
               "d2h_bytes_per_step": out_h.numel() * 2,
               "path": "prism_decode_step (eager, public C ABI) with pinned host q/len in "
                       "and out back, KV cache resident"}

    # -- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only),
    #    repeated to about 10 s of CPU time
    cpu = None
    if not args.skip_cpu and rank == 0 and world == 1:
        layers = list(range(min(args.cpu_layers, N)))
        sample = oracle_sample(w, inp, layers, (0, w.n_kv_heads))
        t1, threads = time_oracle(w, sample)
        reps = max(1, min(30, int(10.0 / max(t1, 1e-3))))
        t_cpu, threads = time_oracle(w, sample, reps=reps) if reps > 1 else (t1, threads)
        na = sum(mask[:len(layers)])
        cpu = {"value": t_cpu * 1e6 / len(layers), "unit": UNIT,
               "cores": min(threads, w.rows), "kind": "oracle",
               "sample": f"layers 0-{layers[-1]} ({na} anchor + {len(layers) - na} refined) x all "
                         f"{w.n_kv_heads} KV heads of the 128K workload, mean of {reps} passes "
                         f"({t_cpu * reps:.1f} s)"}
        # the same on one thread, on the first anchor group only (about 1-2 s)
        g_layers = layers[:min(len(layers), w.anchor_every)]
        g_sample = oracle_sample(w, inp, g_layers, (0, w.n_kv_heads))
        t_1, _ = time_oracle(w, g_sample, threads=1)
        cpu["host"] = host_cpu()
        cpu["single_thread"] = {"value": t_1 * 1e6 / len(g_layers), "unit": UNIT, "cores": 1,
                                "sample": f"layers 0-{g_layers[-1]} x all {w.n_kv_heads} KV "
                                          f"heads, one pass ({t_1:.1f} s)"}

    # -- the pages' other workloads at one GPU (replicas per rank, like the headline)
    per_config = None
    if args.configs.strip():
        per_config = {}
        for wid in [int(x) for x in args.configs.split(",") if x.strip()]:
            try:
                per_config[f"c{wid}"] = measure_workload(args, prism, synth, wid, dev, peak,
                                                         max(5, args.steps // 2), world)
            except Exception as e:      # reported in the line; the headline stands
                per_config[f"c{wid}"] = {"error": f"{type(e).__name__}: {e}"}
        per_config["c3"] = {"headline": True, "value": value, "unit": UNIT}

    # -- context parallel (512K workload split over the job's ranks)
    cpar = None
    if not args.skip_cp:
        del runner
        runner = None
        try:
            cpar = measure_context_parallel(args, rank, world, dev)
        except Exception as e:          # reported in the line; the headline stands
            cpar = {"error": f"{type(e).__name__}: {e}"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{w.name}: {w.describe()}", "global_batch": w.batch * world,
                       "seq_len": w.max_len, "parallelism": f"replicas x{world}",
                       "graph": not args.no_graph,
                       "l2": "no flush: each step reads ~%.1f GB of distinct K/V, > 126 MB L2"
                             % (step_bytes / 1e9)},
            "layers_per_s": 1e6 / value,
            "roofline": {"kernel": "k_anchor_score", "bound": "hbm", "achieved": ach,
                         "peak": peak, "unit": "GB/s", "frac": ach / peak, "traffic": traffic,
                         "bytes_per_launch": a_bytes, "us_per_launch": t_score * 1e6,
                         "peak_kind": peak_kind,
                         "share_of_step": n_anchor * t_score * 1e3 / ms,
                         "why": "largest HBM consumer of the step (anchor K: "
                                f"{n_anchor * a_bytes / step_bytes:.0%} of its bytes)"},
            "gpu_launches": launches_per_step * args.steps,
            "launches_per_step": launches_per_step,
            "clocks": clk,
            "eager": eager,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "breakdown_us": br,
            "pool_mode": pool,
            "pool_mode_int2": pool_q2,
            "context_parallel": cpar,
            "refine_diagnostics": {
                "how": "per refined layer of the timed step: recall of the layer's selection "
                       "against its own exact top-kappa (an anchor selection of the same "
                       "layer), and the proposal |P| per (batch, KV head) row",
                "recall_mean": (statistics.mean(d["recall_mean"] for d in refine_diag
                                                if "recall_mean" in d)
                                if any("recall_mean" in d for d in refine_diag) else None),
                "recall_min": (min(d["recall_min"] for d in refine_diag if "recall_min" in d)
                               if any("recall_min" in d for d in refine_diag) else None),
                "errors": [d for d in refine_diag if "error" in d]},
            "per_config": per_config,
            "refine_attn": {"bytes_per_layer": refine_bytes, "us_per_layer": refine_us,
                            "gbs": refine_bytes / (refine_us * 1e-6) / 1e9,
                            "frac": refine_bytes / (refine_us * 1e-6) / 1e9 / peak,
                            "how": "one anchor then 31 refined layers, graph-timed, minus the "
                                   "anchor layer alone, per refined layer; bytes = measured "
                                   "proposal K rows + gathered K/V rows"},
            "step_hbm": {"algorithmic_bytes": step_bytes, "gbs": step_gbs,
                         "frac": step_gbs / peak, "peak": peak, "peak_kind": peak_kind,
                         "proposal_mean_per_row": (statistics.mean(prop_sizes) / w.rows
                                                   if prop_sizes else 0)},
        }
        print(json.dumps(line), flush=True)
    if runner is not None:
        del runner


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    import torch
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=dev)
    try:
        run_prism(args, rank, world, dev)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
