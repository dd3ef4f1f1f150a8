"""Small numpy helpers shared by the tests (independent of the oracle and of the
CUDA library)."""
from __future__ import annotations

import itertools
import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name: str):
    with open(os.path.join(GOLDEN, name + ".json")) as f:
        return json.load(f)


def f32_to_bf16_bits(x) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return the bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f64(b) -> np.ndarray:
    u = np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def rand_bf16(rng: np.random.Generator, shape, scale=1.0) -> np.ndarray:
    return f32_to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def lexsort_topk(s, kappa, pos=None) -> np.ndarray:
    """Top-kappa by numpy.lexsort on (-score, position); ascending, -1 padded."""
    s = np.asarray(s, dtype=np.float64)
    n = s.shape[0]
    pos = np.arange(n, dtype=np.int64) if pos is None else np.asarray(pos, dtype=np.int64)
    keff = min(kappa, n)
    order = np.lexsort((pos, -s))[:keff]
    out = np.full(kappa, -1, dtype=np.int64)
    out[:keff] = np.sort(pos[order])
    return out


def subset_topk(s, kappa, pos=None):
    """Brute force over every kappa-subset: the unique subset whose every member
    precedes every non-member in the order (score descending, position
    ascending).  Returns the sorted subset (padded with -1) and how many subsets
    qualified."""
    s = list(map(float, s))
    n = len(s)
    pos = list(range(n)) if pos is None else list(map(int, pos))
    keff = min(kappa, n)

    def before(a, b):
        return s[a] > s[b] or (s[a] == s[b] and pos[a] < pos[b])

    found = []
    for comb in itertools.combinations(range(n), keff):
        inside = set(comb)
        if all(before(a, b) for a in inside for b in range(n) if b not in inside):
            found.append(sorted(pos[a] for a in comb))
    out = None
    if found:
        out = np.full(kappa, -1, dtype=np.int64)
        out[:keff] = found[0]
    return out, len(found)


def brute_expand(L, idx_prev, r):
    cover = set()
    for i in idx_prev:
        i = int(i)
        if i < 0 or i >= L:
            continue
        for p in range(max(0, i - r), min(L - 1, i + r) + 1):
            cover.add(p)
    return np.array(sorted(cover), dtype=np.int64)


def numpy_scores(q_bits, k_bits, scale, pos=None):
    """Eq. (1) by numpy.einsum over the group and the head dimension."""
    q = bf16_bits_to_f64(q_bits)
    k = bf16_bits_to_f64(k_bits)
    if pos is not None:
        k = k[np.asarray(pos, dtype=np.int64)]
    return scale * np.einsum("gd,ld->l", q, k)


def numpy_scores_max(q_bits, k_bits, scale, pos=None):
    """Eq. (9): per-head dot products by numpy.einsum, then numpy's maximum
    over the group."""
    q = bf16_bits_to_f64(q_bits)
    k = bf16_bits_to_f64(k_bits)
    if pos is not None:
        k = k[np.asarray(pos, dtype=np.int64)]
    if k.shape[0] == 0:
        return np.zeros(0)
    return scale * np.einsum("gd,ld->gl", q, k).max(axis=0)


def sdpa_group(q_bits, k_bits, v_bits, idx, scale):
    """Reference attention of one GQA group over a position set, by
    torch.nn.functional.scaled_dot_product_attention in fp64 with a boolean
    mask that admits exactly the selected positions."""
    import torch
    q = torch.from_numpy(bf16_bits_to_f64(q_bits))          # [G][d]
    k = torch.from_numpy(bf16_bits_to_f64(k_bits))          # [L][d]
    v = torch.from_numpy(bf16_bits_to_f64(v_bits))
    L = k.shape[0]
    sel = np.asarray(idx)
    sel = sel[sel >= 0]
    G, d = q.shape
    if sel.size == 0:
        return np.zeros((G, d))
    mask = torch.zeros((1, 1, 1, L), dtype=torch.bool)
    mask[..., torch.from_numpy(sel.astype(np.int64))] = True
    o = torch.nn.functional.scaled_dot_product_attention(
        q.view(1, G, 1, d), k.view(1, 1, L, d).expand(1, G, L, d),
        v.view(1, 1, L, d).expand(1, G, L, d), attn_mask=mask.expand(1, G, 1, L), scale=scale)
    return o.view(G, d).numpy()


def unpack_q2(kq, d):
    """The 2-bit key cache format of include/prism.h read back: kq uint8
    [n][d/2] -> codes [n][d] (uint8), alpha and beta [n][d/32] (float32)."""
    kq = np.ascontiguousarray(kq, dtype=np.uint8)
    n = kq.shape[0]
    ks = d // 16
    codes = np.zeros((n, d), np.uint8)
    for t in range(4):
        for kk in range(ks):
            byte = kq[:, t * ks + kk]
            for i, off in enumerate((2 * t, 2 * t + 1, 2 * t + 8, 2 * t + 9)):
                codes[:, 16 * kk + off] = (byte >> (2 * i)) & 3
    par = kq[:, d // 4:].copy().view(np.float32).reshape(n, d // 32, 2)
    return codes, par[..., 0].copy(), par[..., 1].copy()
