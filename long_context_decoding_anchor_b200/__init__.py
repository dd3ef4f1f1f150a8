"""Prism Attention decode hot path for B200 (sm_100a): Python binding.

A thin ctypes layer over the C ABI of ``libprism.so`` (declared in
``include/prism.h``).  It only marshals arguments: torch tensors provide
device memory and streams, every step of the computation runs in the CUDA
kernels of the library.  There is no fallback: if the library is missing or
cannot be loaded, every call raises.

Functions carry the C names:
  prism_workspace_size, prism_index_anchor, prism_index_pool,
  prism_index_refine, prism_sparse_decode, prism_decode_step,
  prism_check_device_status, prism_debug_wait_timeout
plus ``Config`` (the prism_config_t struct) and ``workspace()``; and the
context-parallel calls of ``include/prism_cp.h`` (prism_cp_workspace_size,
prism_cp_index_local, prism_cp_merge, prism_cp_attn_local, prism_cp_combine,
with ``CpShard`` and ``cp_workspace()``), which ``cp.py`` strings together.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libprism.so")

MODE_REFINE, MODE_STATIC_REUSE, MODE_DENSE_ANCHOR, MODE_POOL = 0, 1, 2, 3
CHAIN_PREV, CHAIN_ANCHOR = 0, 1
LAYER_REFINED, LAYER_ANCHOR, LAYER_SHARED = 0, 1, 2
FLAG_SERIAL = 1
FLAG_INT2_KEYS = 2
STATUS = {0: "PRISM_OK", 1: "PRISM_ERR_INVALID_ARG", 2: "PRISM_ERR_UNSUPPORTED",
          3: "PRISM_ERR_WORKSPACE", 4: "PRISM_ERR_CUDA", 5: "PRISM_ERR_TIMEOUT",
          6: "PRISM_ERR_DEVICE"}
EXPORTS = ("prism_workspace_size", "prism_index_anchor", "prism_index_refine",
           "prism_sparse_decode", "prism_decode_step", "prism_check_device_status",
           "prism_debug_wait_timeout", "prism_score_anchor", "prism_status_string",
           "prism_version", "prism_launch_count", "prism_sparse_decode_noalloc",
           "prism_index_pool", "prism_quantize_keys", "prism_decode_step_kq",
           "prism_cp_workspace_size", "prism_cp_index_local", "prism_cp_merge",
           "prism_cp_attn_local", "prism_cp_combine")


class PrismError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({_status_text(status)})")


class Config(ctypes.Structure):
    """prism_config_t."""
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("max_len", ctypes.c_int32), ("kappa", ctypes.c_int32),
                ("radius", ctypes.c_int32), ("n_layers", ctypes.c_int32),
                ("anchor_mask", ctypes.POINTER(ctypes.c_uint8)),
                ("mode", ctypes.c_int32), ("chain", ctypes.c_int32),
                ("scale", ctypes.c_float), ("flags", ctypes.c_int32),
                ("pool_factor", ctypes.c_int32)]

    @classmethod
    def make(cls, batch, n_q_heads, n_kv_heads, head_dim, max_len, kappa, radius=0,
             n_layers=1, anchor_mask: Optional[Sequence[int]] = None, mode=MODE_REFINE,
             chain=CHAIN_PREV, scale=0.0, flags=0, pool_factor=1) -> "Config":
        c = cls(batch, n_q_heads, n_kv_heads, head_dim, max_len, kappa, radius, n_layers,
                None, mode, chain, scale, flags, pool_factor)
        if anchor_mask is not None:
            # layer kinds: 1 anchor (F), 0 refined (R), 2 shared (S)
            arr = (ctypes.c_uint8 * len(anchor_mask))(*[int(x) for x in anchor_mask])
            c._mask_keepalive = arr
            c.anchor_mask = ctypes.cast(arr, ctypes.POINTER(ctypes.c_uint8))
        return c

    @classmethod
    def from_workload(cls, w, **kw) -> "Config":
        args = dict(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                    head_dim=w.head_dim, max_len=w.max_len, kappa=w.kappa, radius=w.radius,
                    n_layers=w.n_layers, anchor_mask=w.anchor_mask())
        args.update(kw)
        return cls.make(**args)

    @property
    def rows(self) -> int:
        return self.batch * self.n_kv_heads

    @property
    def src_kappa(self) -> int:
        """Entries of a refined layer's source: the pool (rho * kappa) in pool
        mode, a selection (kappa) otherwise."""
        return self.pool_factor * self.kappa if self.mode == MODE_POOL else self.kappa


class CpShard(ctypes.Structure):
    """prism_cp_shard_t: rank `rank` of `n_ranks` holds the positions
    [rank * shard_len, (rank + 1) * shard_len) of every sequence."""
    _fields_ = [("n_ranks", ctypes.c_int32), ("rank", ctypes.c_int32),
                ("shard_len", ctypes.c_int32)]

    @property
    def lo(self) -> int:
        return self.rank * self.shard_len


_lib = None


def lib() -> ctypes.CDLL:
    """Load libprism.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m long_context_decoding_anchor_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32, u64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_uint64
        cfgp = ctypes.POINTER(Config)
        L.prism_workspace_size.argtypes = [cfgp, ctypes.POINTER(sz)]
        L.prism_index_anchor.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.prism_index_pool.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.prism_index_pool.restype = ctypes.c_int
        L.prism_score_anchor.argtypes = [cfgp, vp, vp, vp, vp, vp, sz, vp]
        L.prism_score_anchor.restype = ctypes.c_int
        L.prism_launch_count.restype = ctypes.c_uint64
        L.prism_launch_count.argtypes = []
        L.prism_index_refine.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, sz, vp]
        L.prism_sparse_decode.argtypes = [cfgp, vp, vp, vp, vp, vp, i32, vp, vp, sz, vp]
        L.prism_decode_step.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.prism_decode_step_kq.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.prism_decode_step_kq.restype = ctypes.c_int
        L.prism_quantize_keys.argtypes = [cfgp, vp, vp, i32, vp, vp, sz, vp]
        L.prism_quantize_keys.restype = ctypes.c_int
        L.prism_sparse_decode_noalloc.argtypes = [cfgp, vp, vp, vp, vp, vp, i32, vp, vp]
        L.prism_sparse_decode_noalloc.restype = ctypes.c_int
        L.prism_check_device_status.argtypes = [vp, sz, vp, ctypes.POINTER(ctypes.c_uint32)]
        L.prism_debug_wait_timeout.argtypes = [vp, sz, u64, vp]
        L.prism_status_string.argtypes = [ctypes.c_int]
        L.prism_status_string.restype = ctypes.c_char_p
        L.prism_version.restype = i32
        shp = ctypes.POINTER(CpShard)
        L.prism_cp_workspace_size.argtypes = [cfgp, shp, ctypes.POINTER(sz)]
        L.prism_cp_index_local.argtypes = [cfgp, shp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.prism_cp_merge.argtypes = [cfgp, shp, i32, vp, vp, vp, vp, vp, sz, vp]
        L.prism_cp_attn_local.argtypes = [cfgp, shp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.prism_cp_combine.argtypes = [cfgp, i32, vp, vp, vp]
        for name in EXPORTS[-5:]:
            getattr(L, name).restype = ctypes.c_int
        for name in EXPORTS[:8]:
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _status_text(st: int) -> str:
    try:
        return lib().prism_status_string(st).decode()
    except Exception:
        return "?"


def _check(st: int, where: str):
    if st != 0:
        raise PrismError(st, where)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


def _need_keys(cfg: Config, k, name="k"):
    """bf16 keys [B][Hkv][Lmax][d], or with FLAG_INT2_KEYS the 2-bit cache
    uint8 [B][Hkv][Lmax][d/2] (prism_quantize_keys)."""
    B, Hkv, d, L = cfg.batch, cfg.n_kv_heads, cfg.head_dim, cfg.max_len
    if cfg.flags & FLAG_INT2_KEYS:
        _need(k, name, torch.uint8, (B, Hkv, L, d // 2))
    else:
        _need(k, name, torch.bfloat16, (B, Hkv, L, d))


def prism_workspace_size(cfg: Config) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().prism_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "prism_workspace_size")
    return n.value


def workspace(cfg: Config, device=None) -> torch.Tensor:
    """A zero-filled workspace buffer for ``cfg`` (uint8; torch allocations are
    512-byte aligned).  Zero-filled so that the status word starts clear."""
    return torch.zeros(prism_workspace_size(cfg), dtype=torch.uint8,
                       device=device or torch.device("cuda"))


def prism_index_anchor(cfg: Config, q, k, lens, idx_out=None, scores_out=None, ws=None,
                       stream=None):
    B, Hq, Hkv, d, L = cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.max_len
    _need(q, "q", torch.bfloat16, (B, Hq, d))
    _need_keys(cfg, k)
    _need(lens, "lens", torch.int32, (B,))
    if idx_out is None:
        idx_out = torch.empty((B, Hkv, cfg.kappa), dtype=torch.int32, device=q.device)
    _need(idx_out, "idx_out", torch.int32, (B, Hkv, cfg.kappa))
    if scores_out is not None:
        _need(scores_out, "scores_out", torch.float32, (B, Hkv, L))
    ws = workspace(cfg, q.device) if ws is None else ws
    _check(lib().prism_index_anchor(ctypes.byref(cfg), _p(q), _p(k), _p(lens), _p(idx_out),
                                    _p(scores_out), _p(ws), ws.numel(), _stream(stream)),
           "prism_index_anchor")
    return idx_out


def prism_index_pool(cfg: Config, q, k, lens, pool_out=None, idx_out=None, scores_out=None,
                     ws=None, stream=None):
    """Pool mode proposal layer: returns (pool [B][Hkv][rho*kappa], idx [B][Hkv][kappa])."""
    B, Hq, Hkv, d, L = cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.max_len
    _need(q, "q", torch.bfloat16, (B, Hq, d))
    _need_keys(cfg, k)
    _need(lens, "lens", torch.int32, (B,))
    n = cfg.pool_factor * cfg.kappa
    if pool_out is None:
        pool_out = torch.empty((B, Hkv, n), dtype=torch.int32, device=q.device)
    if idx_out is None:
        idx_out = torch.empty((B, Hkv, cfg.kappa), dtype=torch.int32, device=q.device)
    _need(pool_out, "pool_out", torch.int32, (B, Hkv, n))
    _need(idx_out, "idx_out", torch.int32, (B, Hkv, cfg.kappa))
    if scores_out is not None:
        _need(scores_out, "scores_out", torch.float32, (B, Hkv, L))
    ws = workspace(cfg, q.device) if ws is None else ws
    _check(lib().prism_index_pool(ctypes.byref(cfg), _p(q), _p(k), _p(lens), _p(pool_out),
                                  _p(idx_out), _p(scores_out), _p(ws), ws.numel(),
                                  _stream(stream)),
           "prism_index_pool")
    return pool_out, idx_out


def prism_score_anchor(cfg: Config, q, k, lens, scores_out=None, ws=None, stream=None):
    """Eq. (1) only: one launch of the anchor scoring kernel."""
    B, Hq, Hkv, d, L = cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.max_len
    _need(q, "q", torch.bfloat16, (B, Hq, d))
    _need_keys(cfg, k)
    _need(lens, "lens", torch.int32, (B,))
    if scores_out is None:
        scores_out = torch.empty((B, Hkv, L), dtype=torch.float32, device=q.device)
    _need(scores_out, "scores_out", torch.float32, (B, Hkv, L))
    ws = workspace(cfg, q.device) if ws is None else ws
    _check(lib().prism_score_anchor(ctypes.byref(cfg), _p(q), _p(k), _p(lens), _p(scores_out),
                                    _p(ws), ws.numel(), _stream(stream)),
           "prism_score_anchor")
    return scores_out


def prism_index_refine(cfg: Config, q, k, lens, idx_prev, idx_out=None, cand_cap=0, ws=None,
                       stream=None):
    """Returns idx_out, or (idx_out, cand_pos, cand_score, cand_count) when cand_cap > 0.
    In pool mode idx_prev is a pool [B][Hkv][rho*kappa]."""
    B, Hq, Hkv, d, L = cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.max_len
    _need(q, "q", torch.bfloat16, (B, Hq, d))
    _need_keys(cfg, k)
    _need(lens, "lens", torch.int32, (B,))
    _need(idx_prev, "idx_prev", torch.int32, (B, Hkv, cfg.src_kappa))
    if idx_out is None:
        idx_out = torch.empty((B, Hkv, cfg.kappa), dtype=torch.int32, device=q.device)
    _need(idx_out, "idx_out", torch.int32, (B, Hkv, cfg.kappa))
    cp = cs = cc = None
    if cand_cap > 0:
        cp = torch.empty((B, Hkv, cand_cap), dtype=torch.int32, device=q.device)
        cs = torch.empty((B, Hkv, cand_cap), dtype=torch.float32, device=q.device)
        cc = torch.empty((B, Hkv), dtype=torch.int32, device=q.device)
    ws = workspace(cfg, q.device) if ws is None else ws
    _check(lib().prism_index_refine(ctypes.byref(cfg), _p(q), _p(k), _p(lens), _p(idx_prev),
                                    _p(idx_out), _p(cp), _p(cs), _p(cc), int(cand_cap), _p(ws),
                                    ws.numel(), _stream(stream)),
           "prism_index_refine")
    return (idx_out, cp, cs, cc) if cand_cap > 0 else idx_out


def prism_sparse_decode(cfg: Config, q, k, v, lens, idx, out=None, ws=None, stream=None):
    B, Hq, Hkv, d, L = cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.max_len
    _need(q, "q", torch.bfloat16, (B, Hq, d))
    _need(k, "k", torch.bfloat16, (B, Hkv, L, d))
    _need(v, "v", torch.bfloat16, (B, Hkv, L, d))
    _need(lens, "lens", torch.int32, (B,))
    if idx.dim() != 3 or tuple(idx.shape[:2]) != (B, Hkv):
        raise ValueError("idx must be [B][Hkv][n_idx]")
    _need(idx, "idx", torch.int32)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, (B, Hq, d))
    ws = workspace(cfg, q.device) if ws is None else ws
    _check(lib().prism_sparse_decode(ctypes.byref(cfg), _p(q), _p(k), _p(v), _p(lens), _p(idx),
                                     int(idx.shape[2]), _p(out), _p(ws), ws.numel(),
                                     _stream(stream)),
           "prism_sparse_decode")
    return out


def prism_sparse_decode_noalloc(cfg: Config, q, k, v, lens, idx, out=None, stream=None):
    """prism_sparse_decode with the library's own fixed scratch (no workspace)."""
    B, Hq, Hkv, d, L = cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.max_len
    _need(q, "q", torch.bfloat16, (B, Hq, d))
    _need(k, "k", torch.bfloat16, (B, Hkv, L, d))
    _need(v, "v", torch.bfloat16, (B, Hkv, L, d))
    _need(lens, "lens", torch.int32, (B,))
    if idx.dim() != 3 or tuple(idx.shape[:2]) != (B, Hkv):
        raise ValueError("idx must be [B][Hkv][n_idx]")
    _need(idx, "idx", torch.int32)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, (B, Hq, d))
    _check(lib().prism_sparse_decode_noalloc(ctypes.byref(cfg), _p(q), _p(k), _p(v), _p(lens),
                                             _p(idx), int(idx.shape[2]), _p(out),
                                             _stream(stream)),
           "prism_sparse_decode_noalloc")
    return out


def prism_decode_step(cfg: Config, q, k_layers, v_layers, lens, out=None, idx_out=None,
                      ws=None, stream=None, want_idx=False):
    N, B, Hq, Hkv, d, L = (cfg.n_layers, cfg.batch, cfg.n_q_heads, cfg.n_kv_heads,
                           cfg.head_dim, cfg.max_len)
    _need(q, "q", torch.bfloat16, (N, B, Hq, d))
    if len(k_layers) != N or len(v_layers) != N:
        raise ValueError("need one K and one V tensor per layer")
    for i, (kk, vv) in enumerate(zip(k_layers, v_layers)):
        _need(kk, f"k[{i}]", torch.bfloat16, (B, Hkv, L, d))
        _need(vv, f"v[{i}]", torch.bfloat16, (B, Hkv, L, d))
    _need(lens, "lens", torch.int32, (B,))
    if out is None:
        out = torch.empty((N, B, Hq, d), dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, (N, B, Hq, d))
    if idx_out is None and want_idx:
        idx_out = torch.empty((N, B, Hkv, cfg.kappa), dtype=torch.int32, device=q.device)
    if idx_out is not None:
        _need(idx_out, "idx_out", torch.int32, (N, B, Hkv, cfg.kappa))
    kp = (ctypes.c_void_p * N)(*[kk.data_ptr() for kk in k_layers])
    vp = (ctypes.c_void_p * N)(*[vv.data_ptr() for vv in v_layers])
    ws = workspace(cfg, q.device) if ws is None else ws
    _check(lib().prism_decode_step(ctypes.byref(cfg), _p(q), ctypes.cast(kp, ctypes.c_void_p),
                                   ctypes.cast(vp, ctypes.c_void_p), _p(lens), _p(out),
                                   _p(idx_out), _p(ws), ws.numel(), _stream(stream)),
           "prism_decode_step")
    return (out, idx_out) if idx_out is not None else out


def prism_quantize_keys(cfg: Config, k, lens, start=0, kq=None, ws=None, stream=None):
    """Eq. (7)-(8): the 2-bit proposal key cache of one layer (uint8
    [B][Hkv][Lmax][d/2]); positions [start, len[b]) are written."""
    B, Hkv, d, L = cfg.batch, cfg.n_kv_heads, cfg.head_dim, cfg.max_len
    _need(k, "k", torch.bfloat16, (B, Hkv, L, d))
    _need(lens, "lens", torch.int32, (B,))
    if kq is None:
        kq = torch.zeros((B, Hkv, L, d // 2), dtype=torch.uint8, device=k.device)
    _need(kq, "kq", torch.uint8, (B, Hkv, L, d // 2))
    ws = workspace(cfg, k.device) if ws is None else ws
    _check(lib().prism_quantize_keys(ctypes.byref(cfg), _p(k), _p(lens), int(start), _p(kq),
                                     _p(ws), ws.numel(), _stream(stream)),
           "prism_quantize_keys")
    return kq


def prism_decode_step_kq(cfg: Config, q, k_layers, v_layers, kq_layers, lens, out=None,
                         idx_out=None, ws=None, stream=None, want_idx=False):
    """prism_decode_step with 2-bit proposal keys (pool mode, FLAG_INT2_KEYS)."""
    N, B, Hq, Hkv, d, L = (cfg.n_layers, cfg.batch, cfg.n_q_heads, cfg.n_kv_heads,
                           cfg.head_dim, cfg.max_len)
    _need(q, "q", torch.bfloat16, (N, B, Hq, d))
    if len(k_layers) != N or len(v_layers) != N or len(kq_layers) != N:
        raise ValueError("need one K, one V and one 2-bit K tensor per layer")
    for i in range(N):
        _need(k_layers[i], f"k[{i}]", torch.bfloat16, (B, Hkv, L, d))
        _need(v_layers[i], f"v[{i}]", torch.bfloat16, (B, Hkv, L, d))
        _need(kq_layers[i], f"kq[{i}]", torch.uint8, (B, Hkv, L, d // 2))
    _need(lens, "lens", torch.int32, (B,))
    if out is None:
        out = torch.empty((N, B, Hq, d), dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, (N, B, Hq, d))
    if idx_out is None and want_idx:
        idx_out = torch.empty((N, B, Hkv, cfg.kappa), dtype=torch.int32, device=q.device)
    if idx_out is not None:
        _need(idx_out, "idx_out", torch.int32, (N, B, Hkv, cfg.kappa))
    arr = lambda ts: (ctypes.c_void_p * N)(*[t.data_ptr() for t in ts])
    kp, vp, kqp = arr(k_layers), arr(v_layers), arr(kq_layers)
    ws = workspace(cfg, q.device) if ws is None else ws
    _check(lib().prism_decode_step_kq(ctypes.byref(cfg), _p(q), ctypes.cast(kp, ctypes.c_void_p),
                                      ctypes.cast(vp, ctypes.c_void_p),
                                      ctypes.cast(kqp, ctypes.c_void_p), _p(lens), _p(out),
                                      _p(idx_out), _p(ws), ws.numel(), _stream(stream)),
           "prism_decode_step_kq")
    return (out, idx_out) if idx_out is not None else out


# -- context parallel (include/prism_cp.h) -----------------------------------------
def prism_cp_workspace_size(cfg: Config, shard: CpShard) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().prism_cp_workspace_size(ctypes.byref(cfg), ctypes.byref(shard), ctypes.byref(n)),
           "prism_cp_workspace_size")
    return n.value


def cp_workspace(cfg: Config, shard: CpShard, device=None) -> torch.Tensor:
    return torch.zeros(prism_cp_workspace_size(cfg, shard), dtype=torch.uint8,
                       device=device or torch.device("cuda"))


def _need_shard_kv(cfg: Config, shard: CpShard, t, name):
    _need(t, name, torch.bfloat16, (cfg.batch, cfg.n_kv_heads, shard.shard_len, cfg.head_dim))


def prism_cp_index_local(cfg: Config, shard: CpShard, q, k, lens, src=None, ws=None,
                         stream=None):
    """This shard's half of a selection: (cand_pos, cand_score) [B][Hkv][kappa],
    plus (pool_pos, pool_score) [B][Hkv][rho*kappa] for a pool-mode anchor
    (src None).  src: the canonical global source selection of a refined layer."""
    B, Hq, Hkv, d = cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    _need(q, "q", torch.bfloat16, (B, Hq, d))
    _need_shard_kv(cfg, shard, k, "k")
    _need(lens, "lens", torch.int32, (B,))
    if src is not None:
        _need(src, "src", torch.int32, (B, Hkv, cfg.src_kappa))
    dev = q.device
    cp = torch.empty((B, Hkv, cfg.kappa), dtype=torch.int32, device=dev)
    cs = torch.empty((B, Hkv, cfg.kappa), dtype=torch.float32, device=dev)
    pp = ps = None
    if cfg.mode == MODE_POOL and src is None:
        pp = torch.empty((B, Hkv, cfg.src_kappa), dtype=torch.int32, device=dev)
        ps = torch.empty((B, Hkv, cfg.src_kappa), dtype=torch.float32, device=dev)
    ws = cp_workspace(cfg, shard, dev) if ws is None else ws
    _check(lib().prism_cp_index_local(ctypes.byref(cfg), ctypes.byref(shard), _p(q), _p(k),
                                      _p(lens), _p(src), _p(cp), _p(cs), _p(pp), _p(ps), _p(ws),
                                      ws.numel(), _stream(stream)),
           "prism_cp_index_local")
    return (cp, cs) if pp is None else (cp, cs, pp, ps)


def prism_cp_merge(cfg: Config, shard: CpShard, cand_pos, cand_score, lens, idx_out=None,
                   ws=None, stream=None):
    """Exact top-n over the gathered lists [R][B][Hkv][n] (n = kappa, or rho*kappa
    for a pool): ascending global positions [B][Hkv][n], -1 padded."""
    R, B, Hkv = shard.n_ranks, cfg.batch, cfg.n_kv_heads
    if cand_pos.dim() != 4:
        raise ValueError("cand_pos must be [R][B][Hkv][n]")
    n = int(cand_pos.shape[3])
    _need(cand_pos, "cand_pos", torch.int32, (R, B, Hkv, n))
    _need(cand_score, "cand_score", torch.float32, (R, B, Hkv, n))
    _need(lens, "lens", torch.int32, (B,))
    if idx_out is None:
        idx_out = torch.empty((B, Hkv, n), dtype=torch.int32, device=cand_pos.device)
    _need(idx_out, "idx_out", torch.int32, (B, Hkv, n))
    ws = cp_workspace(cfg, shard, cand_pos.device) if ws is None else ws
    _check(lib().prism_cp_merge(ctypes.byref(cfg), ctypes.byref(shard), n, _p(cand_pos),
                                _p(cand_score), _p(lens), _p(idx_out), _p(ws), ws.numel(),
                                _stream(stream)),
           "prism_cp_merge")
    return idx_out


def prism_cp_attn_local(cfg: Config, shard: CpShard, q, k, v, lens, idx, part_out=None,
                        ws=None, stream=None):
    """This shard's split-softmax partial fp32 [B][Hq][d + 2] (acc, m, l)."""
    B, Hq, Hkv, d = cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    _need(q, "q", torch.bfloat16, (B, Hq, d))
    _need_shard_kv(cfg, shard, k, "k")
    _need_shard_kv(cfg, shard, v, "v")
    _need(lens, "lens", torch.int32, (B,))
    _need(idx, "idx", torch.int32, (B, Hkv, cfg.kappa))
    if part_out is None:
        part_out = torch.empty((B, Hq, d + 2), dtype=torch.float32, device=q.device)
    _need(part_out, "part_out", torch.float32, (B, Hq, d + 2))
    ws = cp_workspace(cfg, shard, q.device) if ws is None else ws
    _check(lib().prism_cp_attn_local(ctypes.byref(cfg), ctypes.byref(shard), _p(q), _p(k), _p(v),
                                     _p(lens), _p(idx), _p(part_out), _p(ws), ws.numel(),
                                     _stream(stream)),
           "prism_cp_attn_local")
    return part_out


def prism_cp_combine(cfg: Config, part_all, out=None, stream=None):
    """Merge of the gathered partials [R][B][Hq][d + 2] into bf16 [B][Hq][d]."""
    B, Hq, d = cfg.batch, cfg.n_q_heads, cfg.head_dim
    if part_all.dim() != 4:
        raise ValueError("part_all must be [R][B][Hq][d + 2]")
    R = int(part_all.shape[0])
    _need(part_all, "part_all", torch.float32, (R, B, Hq, d + 2))
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=part_all.device)
    _need(out, "out", torch.bfloat16, (B, Hq, d))
    _check(lib().prism_cp_combine(ctypes.byref(cfg), R, _p(part_all), _p(out), _stream(stream)),
           "prism_cp_combine")
    return out


def prism_check_device_status(ws: torch.Tensor, stream=None):
    """Synchronises; returns (status, [code, where, value, 0]) and clears the word."""
    detail = (ctypes.c_uint32 * 4)()
    st = lib().prism_check_device_status(_p(ws), ws.numel(), _stream(stream), detail)
    return st, list(detail)


def prism_debug_wait_timeout(ws: torch.Tensor, limit_ns: int, stream=None):
    _check(lib().prism_debug_wait_timeout(_p(ws), ws.numel(), int(limit_ns), _stream(stream)),
           "prism_debug_wait_timeout")


def raw_status(fn_name: str, *args) -> int:
    """Call a C entry point with raw ctypes arguments; returns the status code
    (used by the argument-validation tests)."""
    return getattr(lib(), fn_name)(*args)


__all__ = ["Config", "PrismError", "lib", "workspace", "prism_workspace_size",
           "prism_index_anchor", "prism_index_pool", "prism_index_refine", "prism_sparse_decode",
           "prism_decode_step", "prism_check_device_status", "prism_debug_wait_timeout",
           "prism_score_anchor", "prism_sparse_decode_noalloc", "raw_status", "MODE_REFINE", "MODE_STATIC_REUSE", "MODE_DENSE_ANCHOR", "MODE_POOL",
           "CHAIN_PREV", "CHAIN_ANCHOR", "LAYER_REFINED", "LAYER_ANCHOR", "LAYER_SHARED", "FLAG_SERIAL",
           "FLAG_INT2_KEYS", "prism_quantize_keys", "prism_decode_step_kq", "EXPORTS", "LIB_PATH",
           "CpShard", "cp_workspace", "prism_cp_workspace_size", "prism_cp_index_local",
           "prism_cp_merge", "prism_cp_attn_local", "prism_cp_combine"]
