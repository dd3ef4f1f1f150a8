"""Edge cases of the CUDA path (GPU only): ties (including -0.0 vs +0.0),
empty and short sequences, kappa >= len, radius 0 and radius >= len,
unsorted / duplicated / padded source selections, and the device status word
(bad lengths and indices are clamped or skipped by the kernels' own bounds
checks and reported; the bounded-wait hook reports a timeout)."""
import numpy as np
import pytest
import torch

import long_context_decoding_anchor_b200 as prism
from gpu_checks import check_anchor, check_attention, check_refine
from oracle import bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    prism.lib()


def _cfg(B, Hq, Hkv, d, L, kappa, radius=2, **kw):
    return prism.Config.make(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, max_len=L,
                             kappa=kappa, radius=radius, **kw)


def _rand(shape, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn(shape, generator=g, device="cuda").to(torch.bfloat16)


def _run_stages(oracle, cfg, q, k, v, lens, q2=None, k2=None, idx_prev=None):
    S = torch.empty((cfg.batch, cfg.n_kv_heads, cfg.max_len), dtype=torch.float32, device="cuda")
    ws = prism.workspace(cfg)
    idx = prism.prism_index_anchor(cfg, q, k, lens, scores_out=S, ws=ws)
    check_anchor(oracle, cfg, q, k, lens, idx, S)
    out = prism.prism_sparse_decode(cfg, q, k, v, lens, idx, ws=ws)
    check_attention(oracle, cfg, q, k, v, lens, idx, out)
    prev = idx if idx_prev is None else idx_prev
    q2 = q if q2 is None else q2
    k2 = k if k2 is None else k2
    idx2, cp, cs, cc = prism.prism_index_refine(cfg, q2, k2, lens, prev, cand_cap=cfg.max_len,
                                                ws=ws)
    check_refine(oracle, cfg, q2, k2, lens, prev, idx2, cp, cs, cc)
    st, detail = prism.prism_check_device_status(ws)
    assert st == 0, detail
    return idx, idx2, out


def test_all_equal_scores_pick_lowest_positions(oracle):
    cfg = _cfg(1, 4, 1, 128, 5000, 300)
    q = _rand((1, 4, 128), 1)
    row = _rand((1, 1, 1, 128), 2)
    k = row.expand(1, 1, 5000, 128).contiguous()
    v = _rand((1, 1, 5000, 128), 3)
    lens = torch.tensor([5000], dtype=torch.int32, device="cuda")
    idx, _, _ = _run_stages(oracle, cfg, q, k, v, lens)
    assert torch.equal(idx[0, 0].cpu(), torch.arange(300, dtype=torch.int32))


def test_signed_zero_scores_tie(oracle):
    """Keys of +0.0 and -0.0 give scores +0.0 and -0.0; they must tie."""
    L, d = 4096, 64
    cfg = _cfg(1, 1, 1, d, L, 40)
    q = torch.ones((1, 1, d), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 1, L, d), dtype=torch.bfloat16, device="cuda")
    k[0, 0, 1::2] = -0.0                        # odd rows: -0.0 keys -> -0.0 scores
    k[0, 0, 3000:3010] = 1.0                    # ten clearly positive scores
    v = _rand((1, 1, L, d), 4)
    lens = torch.tensor([L], dtype=torch.int32, device="cuda")
    S = torch.empty((1, 1, L), dtype=torch.float32, device="cuda")
    idx = prism.prism_index_anchor(cfg, q, k, lens, scores_out=S)
    s = S[0, 0].cpu()
    assert torch.signbit(s[1]) and not torch.signbit(s[0]), "setup: -0.0 and +0.0 scores"
    expect = sorted(list(range(3000, 3010)) + list(range(30)))
    assert idx[0, 0].tolist() == expect
    check_anchor(oracle, cfg, q, k, lens, idx, S)


def test_threshold_ties_cut_by_position(oracle):
    """Scores on few levels: the kappa-th score is shared by many tokens."""
    L, d = 20000, 128
    cfg = _cfg(2, 8, 2, d, L, 1000, radius=3)
    q = _rand((2, 8, d), 5)
    base = _rand((3, d), 6)
    choice = torch.randint(0, 3, (2, 2, L), generator=torch.Generator(device="cuda").manual_seed(7),
                           device="cuda")
    k = base[choice].contiguous()
    v = _rand((2, 2, L, d), 8)
    lens = torch.tensor([L, 12345], dtype=torch.int32, device="cuda")
    _run_stages(oracle, cfg, q, k, v, lens)


def test_empty_and_short_sequences(oracle):
    L, d = 700, 64
    cfg = _cfg(4, 4, 2, d, L, 16, radius=1)
    q = _rand((4, 4, d), 9)
    k = _rand((4, 2, L, d), 10)
    v = _rand((4, 2, L, d), 11)
    lens = torch.tensor([0, 1, 5, 700], dtype=torch.int32, device="cuda")
    idx, idx2, out = _run_stages(oracle, cfg, q, k, v, lens)
    assert torch.all(idx[0] == -1) and torch.all(out[0] == 0)
    assert idx[1, :, 0].tolist() == [0, 0] and torch.all(idx[1, :, 1:] == -1)
    assert torch.equal(idx[2, :, :5].cpu(), torch.arange(5, dtype=torch.int32).expand(2, 5))
    # decode step over the same ragged batch
    cfgs = _cfg(4, 4, 2, d, L, 16, radius=1, n_layers=3, anchor_mask=[1, 0, 0])
    o, i = prism.prism_decode_step(cfgs, q.expand(3, -1, -1, -1).contiguous(), [k] * 3, [v] * 3,
                                   lens, want_idx=True)
    assert torch.all(i[:, 0] == -1) and torch.all(o[:, 0] == 0)


def test_kappa_at_least_len(oracle):
    L, d = 300, 128
    for kappa in (300, 301, 1000):
        cfg = _cfg(1, 2, 1, d, L, kappa, radius=0)
        q, k, v = _rand((1, 2, d), 12), _rand((1, 1, L, d), 13), _rand((1, 1, L, d), 14)
        lens = torch.tensor([L], dtype=torch.int32, device="cuda")
        idx, idx2, _ = _run_stages(oracle, cfg, q, k, v, lens)
        assert torch.equal(idx[0, 0, :L].cpu(), torch.arange(L, dtype=torch.int32))
        assert torch.all(idx[0, 0, L:] == -1)
        assert torch.equal(idx2, idx)


def test_radius_extremes(oracle):
    L, d = 3000, 64
    q, k, v = _rand((1, 8, d), 15), _rand((1, 2, L, d), 16), _rand((1, 2, L, d), 17)
    q2, k2 = _rand((1, 8, d), 18), _rand((1, 2, L, d), 19)
    lens = torch.tensor([L], dtype=torch.int32, device="cuda")
    for r in (0, 1, 40, L, 10 * L):
        cfg = _cfg(1, 8, 2, d, L, 128, radius=r)
        idx, idx2, _ = _run_stages(oracle, cfg, q, k, v, lens, q2=q2, k2=k2)
        if r == 0:
            assert torch.equal(idx2, idx)
        if r >= L:
            exact = prism.prism_index_anchor(cfg, q2, k2, lens)
            assert torch.equal(idx2, exact)


def test_unsorted_duplicate_padded_source(oracle):
    L, d = 4000, 128
    cfg = _cfg(1, 4, 2, d, L, 64, radius=2)
    q, k, v = _rand((1, 4, d), 20), _rand((1, 2, L, d), 21), _rand((1, 2, L, d), 22)
    lens = torch.tensor([L], dtype=torch.int32, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(23)
    prev = torch.randint(0, L, (1, 2, 64), generator=g, device="cuda", dtype=torch.int32)
    prev[0, 0, 10:20] = prev[0, 0, 0]           # duplicates
    prev[0, 1, 50:] = -1                        # padding
    prev[0, 0, 31] = 0
    prev[0, 0, 32] = L - 1                      # both ends of the context
    _run_stages(oracle, cfg, q, k, v, lens, idx_prev=prev)


def test_bad_length_is_clamped_and_reported():
    L, d = 512, 64
    cfg = _cfg(1, 2, 1, d, L, 32)
    q, k = _rand((1, 2, d), 24), _rand((1, 1, L, d), 25)
    ws = prism.workspace(cfg)
    lens = torch.tensor([L + 100], dtype=torch.int32, device="cuda")
    prism.prism_index_anchor(cfg, q, k, lens, ws=ws)
    st, detail = prism.prism_check_device_status(ws)
    assert st == 6 and detail[0] == 2, (st, detail)        # PRISM_ERR_DEVICE, bad length
    st, _ = prism.prism_check_device_status(ws)
    assert st == 0                                          # read-and-clear


def test_bad_index_is_skipped_and_reported(oracle):
    L, d = 256, 128
    cfg = _cfg(1, 4, 1, d, L, 8)
    q, k, v = _rand((1, 4, d), 26), _rand((1, 1, L, d), 27), _rand((1, 1, L, d), 28)
    lens = torch.tensor([200], dtype=torch.int32, device="cuda")
    ws = prism.workspace(cfg)
    idx = torch.tensor([[[3, 7, 9, 210, -1, -1, -1, -1]]], dtype=torch.int32, device="cuda")
    out = prism.prism_sparse_decode(cfg, q, k, v, lens, idx, ws=ws)
    st, detail = prism.prism_check_device_status(ws)
    assert st == 6 and detail[0] == 3 and detail[2] == 210, (st, detail)
    good = torch.tensor([[[3, 7, 9, -1, -1, -1, -1, -1]]], dtype=torch.int32, device="cuda")
    check_attention(oracle, cfg, q, k, v, lens, good, out)


def test_bounded_wait_reports_timeout():
    cfg = _cfg(1, 1, 1, 64, 64, 1)
    ws = prism.workspace(cfg)
    prism.prism_debug_wait_timeout(ws, 2_000_000)        # 2 ms
    st, detail = prism.prism_check_device_status(ws)
    assert st == 5 and detail[0] == 1, (st, detail)     # PRISM_ERR_TIMEOUT
    # the context is still usable afterwards
    x = torch.ones(4, device="cuda") * 2
    assert float(x.sum()) == 8.0
