"""ctypes wrapper around the oracle (``prism_ref.c``).

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
CPU-baseline leg of the benchmark may import this module.  It never imports the
CUDA library's package, and the CUDA library never imports it.

All arrays are numpy; bf16 tensors travel as their raw uint16 bit patterns.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

_i32 = ctypes.c_int
_dbl = ctypes.c_double
_vp = ctypes.c_void_p

MODE_REFINE, MODE_STATIC_REUSE, MODE_DENSE_ANCHOR, MODE_POOL = 0, 1, 2, 3
QGROUP = 32          # group size g of the 2-bit proposal keys (Eq. (7))
CHAIN_PREV, CHAIN_ANCHOR = 0, 1


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected bf16 bit patterns as uint16, got {a.dtype}")
    return a


class Oracle:
    """One loaded oracle library (the proper one, or a planted variant)."""

    def __init__(self, path: str):
        self.path = path
        lib = ctypes.CDLL(path)
        lib.prism_ref_score.argtypes = [_i32, _i32, _vp, _vp, _i32, _vp, _dbl, _vp]
        lib.prism_ref_score.restype = None
        lib.prism_ref_score_max.argtypes = [_i32, _i32, _vp, _vp, _i32, _vp, _dbl, _vp]
        lib.prism_ref_score_max.restype = None
        lib.prism_ref_quantize_row.argtypes = [_i32, _i32, _vp, _vp, _vp, _vp]
        lib.prism_ref_quantize_row.restype = None
        lib.prism_ref_score_max_q2.argtypes = [_i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _vp,
                                               _dbl, _vp]
        lib.prism_ref_score_max_q2.restype = None
        lib.prism_ref_topk.argtypes = [_i32, _vp, _vp, _i32, _vp]
        lib.prism_ref_topk.restype = _i32
        lib.prism_ref_expand.argtypes = [_i32, _i32, _vp, _i32, _vp]
        lib.prism_ref_expand.restype = _i32
        lib.prism_ref_attention.argtypes = [_i32, _i32, _vp, _vp, _vp, _i32, _vp, _dbl, _vp, _vp]
        lib.prism_ref_attention.restype = None
        lib.prism_ref_decode_step.argtypes = [
            _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _i32, _i32, _dbl, _i32, _i32,
            _vp, _vp, _vp, _vp, _vp, _vp, _vp]
        lib.prism_ref_decode_step.restype = _i32
        lib.prism_ref_num_threads.restype = _i32
        lib.prism_ref_set_num_threads.argtypes = [_i32]
        lib.prism_ref_set_num_threads.restype = None
        lib.prism_ref_plant.restype = _i32
        self.lib = lib

    @property
    def plant(self) -> int:
        return self.lib.prism_ref_plant()

    def num_threads(self) -> int:
        return self.lib.prism_ref_num_threads()

    def set_num_threads(self, n: int) -> None:
        """Threads of the row-parallel loops from now on (timing only)."""
        self.lib.prism_ref_set_num_threads(int(n))

    # -- single (batch, KV head) row ----------------------------------------
    def score(self, q_group, k_rows, pos=None, scale=None, n=None, agg="sum"):
        """Scores of positions ``pos`` (or 0..n-1) for one KV head: Eq. (1)
        with the group sum (``agg="sum"``) or Eq. (9)'s group maximum
        (``agg="max"``)."""
        if agg not in ("sum", "max"):
            raise ValueError(f"unknown aggregation {agg!r}")
        q_group = _u16(q_group)
        k_rows = _u16(k_rows)
        G, d = q_group.shape
        if pos is not None:
            pos = np.ascontiguousarray(pos, dtype=np.int32)
            n = pos.shape[0]
            if n and (pos.min() < 0 or pos.max() >= k_rows.shape[0]):
                raise ValueError("position outside the key cache")
        elif n is None:
            n = k_rows.shape[0]
        if scale is None:
            scale = 1.0 / np.sqrt(d)
        out = np.empty(n, dtype=np.float64)
        fn = self.lib.prism_ref_score if agg == "sum" else self.lib.prism_ref_score_max
        fn(d, G, _ptr(q_group), _ptr(k_rows), n, _ptr(pos) if pos is not None else None,
           float(scale), _ptr(out))
        return out

    def quantize(self, k_rows, g=QGROUP):
        """Eq. (7)-(8) on key rows [n][d] (uint16 bf16 bits): codes [n][d]
        uint8 (one per element), alpha and beta [n][d/g] float32."""
        k_rows = _u16(k_rows)
        n, d = k_rows.shape
        codes = np.empty((n, d), np.uint8)
        alpha = np.empty((n, d // g), np.float32)
        beta = np.empty((n, d // g), np.float32)
        for i in range(n):
            self.lib.prism_ref_quantize_row(d, g, _ptr(k_rows[i]), _ptr(codes[i]), _ptr(alpha[i]),
                                            _ptr(beta[i]))
        return codes, alpha, beta

    def score_q2(self, q_group, codes, alpha, beta, pos=None, scale=None, g=QGROUP):
        """Eq. (9) group maximum on dequantized 2-bit keys (fp64)."""
        q_group = _u16(q_group)
        codes = np.ascontiguousarray(codes, np.uint8)
        alpha = np.ascontiguousarray(alpha, np.float32)
        beta = np.ascontiguousarray(beta, np.float32)
        G, d = q_group.shape
        n = codes.shape[0] if pos is None else len(pos)
        if pos is not None:
            pos = np.ascontiguousarray(pos, dtype=np.int32)
        if scale is None:
            scale = 1.0 / np.sqrt(d)
        out = np.empty(n, np.float64)
        self.lib.prism_ref_score_max_q2(d, g, G, _ptr(q_group), _ptr(codes), _ptr(alpha),
                                        _ptr(beta), n, _ptr(pos) if pos is not None else None,
                                        float(scale), _ptr(out))
        return out

    def topk(self, s, kappa, pos=None):
        """Eqs. (2)/(6): top-kappa positions, ascending, -1 padded; and kappa_eff."""
        s = np.ascontiguousarray(s, dtype=np.float64)
        n = s.shape[0]
        if pos is not None:
            pos = np.ascontiguousarray(pos, dtype=np.int32)
            assert pos.shape[0] == n
        out = np.empty(kappa, dtype=np.int32)
        keff = self.lib.prism_ref_topk(n, _ptr(s), _ptr(pos) if pos is not None else None,
                                       int(kappa), _ptr(out))
        return out, keff

    def expand(self, L, idx_prev, r):
        """Positional proposal set around ``idx_prev`` (ascending positions)."""
        idx_prev = np.ascontiguousarray(idx_prev, dtype=np.int32)
        out = np.empty(max(int(L), 1), dtype=np.int32)
        n = self.lib.prism_ref_expand(int(L), idx_prev.shape[0], _ptr(idx_prev), int(r), _ptr(out))
        return out[:n].copy()

    def attention(self, q_group, k_rows, v_rows, idx, scale=None):
        """SparseAttn over ``idx`` for one GQA group: (out [G][d], weight sums [G])."""
        q_group, k_rows, v_rows = _u16(q_group), _u16(k_rows), _u16(v_rows)
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        G, d = q_group.shape
        if idx.size and idx.max() >= min(k_rows.shape[0], v_rows.shape[0]):
            raise ValueError("index outside the cache")
        if scale is None:
            scale = 1.0 / np.sqrt(d)
        out = np.empty((G, d), dtype=np.float64)
        wsum = np.empty(G, dtype=np.float64)
        self.lib.prism_ref_attention(d, G, _ptr(q_group), _ptr(k_rows), _ptr(v_rows),
                                     idx.shape[0], _ptr(idx), float(scale), _ptr(out), _ptr(wsum))
        return out, wsum

    # -- whole decode step ----------------------------------------------------
    def decode_step(self, q, k_layers, v_layers, lens, kappa, radius, anchor_mask,
                    mode=MODE_REFINE, chain=CHAIN_PREV, scale=None, rho=1, want_pool=False,
                    qbits=0):
        """Algorithm 1 over all layers.

        q: [N][B][Hq][d] uint16; k_layers/v_layers: N arrays [B][Hkv][Lmax][d]
        uint16; lens: [B].  Returns (out [N][B][Hq][d] fp64,
        idx [N][B][Hkv][kappa] int32), plus, with ``want_pool`` (MODE_POOL),
        the pool in effect at each layer [N][B][Hkv][rho*kappa] int32.
        """
        q = _u16(q)
        N, B, Hq, d = q.shape
        ks = [_u16(k) for k in k_layers]
        vs = [_u16(v) for v in v_layers]
        assert len(ks) == N and len(vs) == N
        _, Hkv, Lmax, d2 = ks[0].shape
        assert d2 == d
        for t in ks + vs:
            assert t.shape == (B, Hkv, Lmax, d)
        lens = np.ascontiguousarray(lens, dtype=np.int32)
        # layer kinds: 1 anchor (F), 0 refined (R), 2 shared (S)
        mask = np.ascontiguousarray(np.asarray(anchor_mask, dtype=np.uint8))
        assert mask.shape[0] == N
        if scale is None:
            scale = 1.0 / np.sqrt(d)
        kp = (ctypes.c_void_p * N)(*[_ptr(t) for t in ks])
        vp = (ctypes.c_void_p * N)(*[_ptr(t) for t in vs])
        out = np.empty((N, B, Hq, d), dtype=np.float64)
        idx = np.empty((N, B, Hkv, kappa), dtype=np.int32)
        pool = None
        if want_pool:
            if mode != MODE_POOL:
                raise ValueError("pools exist only in MODE_POOL")
            pool = np.empty((N, B, Hkv, int(rho) * int(kappa)), dtype=np.int32)
        rc = self.lib.prism_ref_decode_step(B, Hq, Hkv, d, Lmax, int(kappa), int(radius), N,
                                            _ptr(mask), int(mode), int(chain), float(scale),
                                            int(rho), int(qbits), _ptr(q), ctypes.cast(kp, _vp),
                                            ctypes.cast(vp, _vp), _ptr(lens), _ptr(out),
                                            _ptr(idx), _ptr(pool) if pool is not None else None)
        if rc != 0:
            raise ValueError("oracle rejected the decode-step arguments")
        return (out, idx, pool) if want_pool else (out, idx)


_cache: dict[tuple[int, str | None], Oracle] = {}


def load(plant: int = 0, out_dir: str | None = None) -> Oracle:
    """Build (if needed) and load the oracle, or one of its planted variants."""
    key = (plant, out_dir)
    if key not in _cache:
        _cache[key] = Oracle(_build.build(plant=plant, out_dir=out_dir))
    return _cache[key]


def bf16_bits(t) -> np.ndarray:
    """uint16 bit patterns of a bf16 torch tensor (copied to the host)."""
    import torch
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


PLANTS = {
    1: "score drops one query head of the GQA group",
    2: "TopK tie-break prefers the higher position",
    3: "TopK keeps kappa-1 positions",
    4: "proposal window one position short on the left",
    5: "attention logits miss the 1/sqrt(d) scale",
    6: "attention sums K rows instead of V rows",
    7: "softmax weights not normalised",
    8: "score reads the key cache transposed",
    9: "bf16 widening uses the wrong bit position",
    10: "refined layers always start from the anchor's selection",
    11: "refined layers rescore with the previous layer's keys",
    12: "the group maximum of Eq. (9) is replaced by the group sum",
    13: "the anchor's pool holds kappa tokens instead of rho*kappa",
    14: "pool-mode refined layers rescore the previous selection, not the pool",
    15: "the anchor attends to the pool's first kappa positions, not its best kappa",
    16: "shared layers keep the anchor's selection, not the previous layer's",
    17: "the 2-bit scale divides by 2^b instead of 2^b - 1",
    18: "the 2-bit codes truncate instead of rounding",
    19: "the dequantized key drops the zero-point beta",
}

__all__ = ["Oracle", "load", "bf16_bits", "PLANTS", "MODE_REFINE", "MODE_STATIC_REUSE",
           "MODE_DENSE_ANCHOR", "MODE_POOL", "CHAIN_PREV", "CHAIN_ANCHOR"]
