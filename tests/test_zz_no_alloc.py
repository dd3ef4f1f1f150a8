"""prism_sparse_decode_noalloc (no caller workspace, fixed library scratch)
against prism_sparse_decode on the same inputs, two calls in a row, through
the C ABI.  Collected last, so it also runs after every other test."""
import numpy as np
import pytest
import torch

import long_context_decoding_anchor_b200 as prism
from long_context_decoding_anchor_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    prism.lib()


@pytest.mark.parametrize("w", [
    synth.WORKLOADS[2].replace(max_len=6000, n_layers=1),
    synth.WORKLOADS[4].replace(batch=3, max_len=3001, n_layers=1, ragged=(700, 3001)),
])
def test_noalloc_matches_workspace_call_twice(w):
    inp = synth.make_inputs(w, device="cuda", layers=[0])
    cfg = prism.Config.from_workload(w)
    q, k, v, lens = inp["q"][0], inp["k"][0], inp["v"][0], inp["lens"]
    ws = prism.workspace(cfg)
    idx = prism.prism_index_anchor(cfg, q, k, lens, ws=ws)
    ref = prism.prism_sparse_decode(cfg, q, k, v, lens, idx, ws=ws)
    for _ in range(2):
        got = prism.prism_sparse_decode_noalloc(cfg, q, k, v, lens, idx)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)


def test_noalloc_rejects_sizes_above_its_limit():
    w = synth.WORKLOADS[4].replace(batch=129, max_len=512, n_layers=1, ragged=None, kappa=64)
    cfg = prism.Config.from_workload(w)          # 129 * 8 rows > 1024
    z = lambda *s, dt=torch.bfloat16: torch.zeros(*s, dtype=dt, device="cuda")
    q, k = z(w.batch, w.n_q_heads, w.head_dim), z(w.batch, w.n_kv_heads, w.max_len, w.head_dim)
    lens = torch.full((w.batch,), 64, dtype=torch.int32, device="cuda")
    idx = torch.zeros((w.batch, w.n_kv_heads, 64), dtype=torch.int32, device="cuda")
    with pytest.raises(prism.PrismError) as e:
        prism.prism_sparse_decode_noalloc(cfg, q, k, k, lens, idx)
    assert e.value.status == 3                   # PRISM_ERR_WORKSPACE, nothing launched


def test_noalloc_rejects_partials_above_its_float_limit():
    # 16 * 8 rows (within the row limit) x 32 splits x 4 heads x 128 = 2^21
    # partial floats, twice the fixed array's 2^20
    w = synth.WORKLOADS[2].replace(batch=16, max_len=2048, n_layers=1)
    cfg = prism.Config.from_workload(w)
    z = lambda *s, dt=torch.bfloat16: torch.zeros(*s, dtype=dt, device="cuda")
    q, k = z(w.batch, w.n_q_heads, w.head_dim), z(w.batch, w.n_kv_heads, w.max_len, w.head_dim)
    lens = torch.full((w.batch,), w.max_len, dtype=torch.int32, device="cuda")
    idx = torch.zeros((w.batch, w.n_kv_heads, w.kappa), dtype=torch.int32, device="cuda")
    with pytest.raises(prism.PrismError) as e:
        prism.prism_sparse_decode_noalloc(cfg, q, k, k, lens, idx)
    assert e.value.status == 3                   # PRISM_ERR_WORKSPACE, nothing launched


def test_noalloc_at_its_float_limit_matches_workspace_call():
    # 8 * 8 rows x 32 splits x 4 heads x 128 = exactly 2^20 partial floats
    w = synth.WORKLOADS[2].replace(batch=8, max_len=4096, n_layers=1, n_clusters=16)
    inp = synth.make_inputs(w, device="cuda", layers=[0])
    cfg = prism.Config.from_workload(w)
    q, k, v, lens = inp["q"][0], inp["k"][0], inp["v"][0], inp["lens"]
    ws = prism.workspace(cfg)
    idx = prism.prism_index_anchor(cfg, q, k, lens, ws=ws)
    ref = prism.prism_sparse_decode(cfg, q, k, v, lens, idx, ws=ws)
    for _ in range(2):
        got = prism.prism_sparse_decode_noalloc(cfg, q, k, v, lens, idx)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
