"""C-ABI boundary on the CPU: the library loads, exports every entry point
that include/*.h declare, and rejects invalid arguments on the host
before anything is launched (no GPU needed, no device memory touched)."""
import ctypes
import glob
import os
import re

import pytest

import long_context_decoding_anchor_b200 as prism
from long_context_decoding_anchor_b200 import build as prism_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))


@pytest.fixture(scope="module")
def L():
    prism_build.build()
    return prism.lib()


def declared_symbols():
    text = "".join(open(h).read() for h in HEADERS)
    return sorted(set(re.findall(r"PRISM_API\s+[\w\s\*]+?\b(prism_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for required in ("prism_index_anchor", "prism_index_refine", "prism_sparse_decode",
                     "prism_decode_step", "prism_workspace_size", "prism_cp_index_local",
                     "prism_cp_merge", "prism_cp_attn_local", "prism_cp_combine"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), f"{name} declared in prism.h but not exported"
    assert set(prism.EXPORTS) <= set(declared_symbols())


def test_status_strings(L):
    for code in range(7):
        assert len(L.prism_status_string(code)) > 0
    assert L.prism_version() >= 100


def _cfg(**kw):
    base = dict(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=64, max_len=4096, kappa=256,
                radius=4, n_layers=4, anchor_mask=[1, 0, 0, 0])
    base.update(kw)
    return prism.Config.make(**base)


def test_workspace_size_monotone(L):
    small = prism.prism_workspace_size(_cfg())
    big = prism.prism_workspace_size(_cfg(max_len=8192))
    assert 0 < small < big
    assert prism.prism_workspace_size(_cfg(batch=2)) > small


@pytest.mark.parametrize("bad,status", [
    (dict(head_dim=96), 2), (dict(head_dim=32), 2), (dict(n_q_heads=12, n_kv_heads=8), 1),
    (dict(n_q_heads=24, n_kv_heads=8), 2), (dict(n_q_heads=32, n_kv_heads=2, head_dim=64), 2),
    (dict(kappa=0), 1), (dict(radius=-1), 1), (dict(max_len=0), 1),
    (dict(max_len=(1 << 20) + 1), 2), (dict(batch=0), 1), (dict(mode=4), 1), (dict(chain=2), 1),
    (dict(mode=3, pool_factor=0), 1), (dict(mode=3, pool_factor=-2), 1),
    (dict(mode=3, kappa=1 << 19, pool_factor=4), 2),
    (dict(scale=-1.0), 1), (dict(scale=float("nan")), 1), (dict(batch=70000, n_kv_heads=1,
                                                                  n_q_heads=1), 2),
    (dict(flags=4), 1), (dict(flags=2), 1), (dict(n_layers=-1), 1), (dict(n_layers=5000), 2),
])
def test_invalid_config_rejected(L, bad, status):
    c = _cfg(**bad)
    n = ctypes.c_size_t(0)
    assert L.prism_workspace_size(ctypes.byref(c), ctypes.byref(n)) == status


# Fake device addresses: validation must reject the call before any use.
A16 = ctypes.c_void_p(0x10000)
A4 = ctypes.c_void_p(0x10004)
MIS = ctypes.c_void_p(0x10002)


def test_anchor_argument_validation(L):
    c = _cfg()
    ws_n = prism.prism_workspace_size(c)
    ws = ctypes.c_void_p(0x100000)
    f = L.prism_index_anchor
    cp = ctypes.byref(c)
    assert f(cp, None, A16, A4, A4, None, ws, ws_n, None) == 1          # null q
    assert f(cp, A16, None, A4, A4, None, ws, ws_n, None) == 1          # null k
    assert f(cp, A16, A16, None, A4, None, ws, ws_n, None) == 1         # null len
    assert f(cp, A16, A16, A4, None, None, ws, ws_n, None) == 1         # null idx_out
    assert f(cp, MIS, A16, A4, A4, None, ws, ws_n, None) == 1           # q misaligned
    assert f(cp, A16, MIS, A4, A4, None, ws, ws_n, None) == 1           # k misaligned
    assert f(cp, A16, A16, A4, A4, None, ctypes.c_void_p(0x100010), ws_n, None) == 1  # ws align
    assert f(cp, A16, A16, A4, A4, None, ws, ws_n - 1, None) == 3       # short workspace
    assert f(cp, A16, A16, A4, A4, None, None, ws_n, None) == 1         # null workspace


def test_pool_argument_validation(L):
    c = _cfg(mode=prism.MODE_POOL, pool_factor=4)
    ws_n = prism.prism_workspace_size(c)
    assert ws_n > prism.prism_workspace_size(_cfg())            # room for the pools
    ws = ctypes.c_void_p(0x100000)
    f = L.prism_index_pool
    cp = ctypes.byref(c)
    P = ctypes.c_void_p(0x50000)
    assert f(cp, None, A16, A4, P, A4, None, ws, ws_n, None) == 1          # null q
    assert f(cp, A16, A16, A4, None, A4, None, ws, ws_n, None) == 1        # null pool_out
    assert f(cp, A16, A16, A4, P, None, None, ws, ws_n, None) == 1         # null idx_out
    assert f(cp, A16, A16, A4, P, P, None, ws, ws_n, None) == 1            # pool aliases idx
    assert f(cp, A16, MIS, A4, P, A4, None, ws, ws_n, None) == 1           # k misaligned
    assert f(cp, A16, A16, A4, P, A4, None, ws, ws_n - 1, None) == 3       # short workspace
    other = _cfg()                                                          # not pool mode
    assert f(ctypes.byref(other), A16, A16, A4, P, A4, None, ws, ws_n, None) == 1


def test_refine_argument_validation(L):
    c = _cfg()
    ws_n = prism.prism_workspace_size(c)
    ws = ctypes.c_void_p(0x100000)
    f = L.prism_index_refine
    cp = ctypes.byref(c)
    same = ctypes.c_void_p(0x20000)
    assert f(cp, A16, A16, A4, same, same, None, None, None, 0, ws, ws_n, None) == 1   # alias
    assert f(cp, A16, A16, A4, A4, ctypes.c_void_p(0x30000), A4, None, None, 16, ws, ws_n,
             None) == 1                                                   # partial cand outputs
    assert f(cp, A16, A16, A4, A4, ctypes.c_void_p(0x30000), A4, A4, A4, 0, ws, ws_n,
             None) == 1                                                   # cand_cap 0
    assert f(cp, A16, A16, A4, None, A4, None, None, None, 0, ws, ws_n, None) == 1


def test_sparse_decode_argument_validation(L):
    c = _cfg()
    ws_n = prism.prism_workspace_size(c)
    ws = ctypes.c_void_p(0x100000)
    f = L.prism_sparse_decode
    cp = ctypes.byref(c)
    assert f(cp, A16, A16, A16, A4, A4, 0, A16, ws, ws_n, None) == 1         # n_idx 0
    assert f(cp, A16, A16, A16, A4, A4, 257, A16, ws, ws_n, None) == 1       # n_idx > kappa
    assert f(cp, A16, A16, MIS, A4, A4, 16, A16, ws, ws_n, None) == 1        # v misaligned
    assert f(cp, A16, A16, A16, A4, A4, 16, MIS, ws, ws_n, None) == 1        # out misaligned


def test_decode_step_argument_validation(L):
    ws = ctypes.c_void_p(0x100000)
    c = _cfg(anchor_mask=[0, 1, 0, 0])
    ws_n = prism.prism_workspace_size(c)
    kp = (ctypes.c_void_p * 4)(*[0x40000 + 0x100 * i for i in range(4)])
    f = L.prism_decode_step
    assert f(ctypes.byref(c), A16, kp, kp, A4, A16, None, ws, ws_n, None) == 1  # layer 0 not anchor
    c = _cfg()
    bad = (ctypes.c_void_p * 4)(0x40000, 0x40008, 0x40100, 0x40200)             # k[1] misaligned
    assert f(ctypes.byref(c), A16, bad, kp, A4, A16, None, ws, ws_n, None) == 1
    nul = (ctypes.c_void_p * 4)(0x40000, None, 0x40100, 0x40200)
    assert f(ctypes.byref(c), A16, kp, nul, A4, A16, None, ws, ws_n, None) == 1
    c = _cfg(n_layers=0)
    assert f(ctypes.byref(c), A16, kp, kp, A4, A16, None, ws, ws_n, None) == 1
    c = _cfg(anchor_mask=None)
    assert f(ctypes.byref(c), A16, kp, kp, A4, A16, None, ws, ws_n, None) == 1  # mask required
    c = _cfg(anchor_mask=[2, 0, 0, 0])
    assert f(ctypes.byref(c), A16, kp, kp, A4, A16, None, ws, ws_n, None) == 1  # layer 0 shared
    c = _cfg(anchor_mask=[1, 0, 3, 0])
    assert f(ctypes.byref(c), A16, kp, kp, A4, A16, None, ws, ws_n, None) == 1  # unknown kind


def test_debug_wait_validation(L):
    assert L.prism_debug_wait_timeout(None, 256, 1000, None) == 1
    assert L.prism_debug_wait_timeout(ctypes.c_void_p(0x100000), 256, 0, None) == 1
    assert L.prism_check_device_status(ctypes.c_void_p(0x100010), 256, None, None) == 1


def test_binding_rejects_cpu_tensors():
    import torch
    c = _cfg()
    with pytest.raises(ValueError):
        prism.prism_index_anchor(c, torch.zeros(1, 8, 64, dtype=torch.bfloat16),
                                 torch.zeros(1, 2, 4096, 64, dtype=torch.bfloat16),
                                 torch.zeros(1, dtype=torch.int32))


def test_int2_key_validation(L):
    """The 2-bit key flag belongs to pool mode; the plain step rejects it and
    the kq step needs it."""
    ws = ctypes.c_void_p(0x100000)
    kp = (ctypes.c_void_p * 4)(*[0x40000 + 0x100 * i for i in range(4)])
    c = _cfg(mode=prism.MODE_POOL, pool_factor=4, flags=prism.FLAG_INT2_KEYS)
    ws_n = prism.prism_workspace_size(c)
    assert L.prism_decode_step(ctypes.byref(c), A16, kp, kp, A4, A16, None, ws, ws_n, None) == 1
    plain = _cfg(mode=prism.MODE_POOL, pool_factor=4)
    assert L.prism_decode_step_kq(ctypes.byref(plain), A16, kp, kp, kp, A4, A16, None, ws, ws_n,
                                  None) == 1
    assert L.prism_decode_step_kq(ctypes.byref(c), A16, kp, kp, None, A4, A16, None, ws, ws_n,
                                  None) == 1
    bad = (ctypes.c_void_p * 4)(0x40000, 0x40108, 0x40200, 0x40300)          # kq[1] misaligned
    assert L.prism_decode_step_kq(ctypes.byref(c), A16, kp, kp, bad, A4, A16, None, ws, ws_n,
                                  None) == 1
    q = L.prism_quantize_keys
    assert q(ctypes.byref(c), None, A4, 0, A16, ws, 256, None) == 1
    assert q(ctypes.byref(c), A16, A4, -1, A16, ws, 256, None) == 1          # negative start
    assert q(ctypes.byref(c), A16, A4, 0, MIS, ws, 256, None) == 1           # kq misaligned
    assert q(ctypes.byref(c), A16, A4, 0, A16, None, 256, None) == 1         # no status word


def _shard(n_ranks=2, rank=0, shard_len=2048):
    return prism.CpShard(n_ranks, rank, shard_len)


@pytest.mark.parametrize("sh,cfg_kw,status", [
    (dict(n_ranks=0), {}, 1), (dict(rank=2), {}, 1), (dict(rank=-1), {}, 1),
    (dict(shard_len=0), {}, 1), (dict(shard_len=1000), {}, 1),     # 2 x 1000 < Lmax 4096
    (dict(n_ranks=2049, shard_len=1 << 20), {}, 1),               # positions past 2^31 - 1
    (dict(), dict(mode=3, pool_factor=2, flags=2), 2),              # 2-bit keys
    (dict(), dict(head_dim=96), 2),
])
def test_cp_invalid_shard_rejected(L, sh, cfg_kw, status):
    c, s = _cfg(**cfg_kw), _shard(**sh)
    n = ctypes.c_size_t(0)
    assert L.prism_cp_workspace_size(ctypes.byref(c), ctypes.byref(s), ctypes.byref(n)) == status


def test_cp_workspace_grows_with_ranks_and_shard(L):
    c = _cfg()
    a = prism.prism_cp_workspace_size(c, _shard(2, 0, 2048))
    assert prism.prism_cp_workspace_size(c, _shard(4, 0, 2048)) > a       # merge buffers
    assert prism.prism_cp_workspace_size(c, _shard(2, 0, 4096)) > a       # shard buffers
    assert prism.prism_cp_workspace_size(c, _shard(2, 1, 2048)) == a


def test_cp_argument_validation(L):
    c, s = _cfg(), _shard()
    ws_n = prism.prism_cp_workspace_size(c, s)
    ws = ctypes.c_void_p(0x100000)
    cp_, sp = ctypes.byref(c), ctypes.byref(s)
    f = L.prism_cp_index_local
    assert f(cp_, sp, None, A16, A4, None, A4, A4, None, None, ws, ws_n, None) == 1   # null q
    assert f(cp_, sp, A16, A16, A4, None, None, A4, None, None, ws, ws_n, None) == 1  # null pos
    assert f(cp_, sp, MIS, A16, A4, None, A4, A4, None, None, ws, ws_n, None) == 1    # q align
    assert f(cp_, sp, A16, A16, A4, None, A4, A4, A4, A4, ws, ws_n, None) == 1        # pool bufs
    assert f(cp_, sp, A16, A16, A4, None, A4, A4, None, None, ws, ws_n - 1, None) == 3
    assert f(cp_, sp, A16, A16, A4, None, A4, A4, None, None, None, ws_n, None) == 1
    assert f(cp_, None, A16, A16, A4, None, A4, A4, None, None, ws, ws_n, None) == 1  # no shard
    pc = _cfg(mode=3, pool_factor=2)
    pws = prism.prism_cp_workspace_size(pc, s)
    pcp = ctypes.byref(pc)
    assert f(pcp, sp, A16, A16, A4, None, A4, A4, None, None, ws, pws, None) == 1     # pool anchor
    assert f(pcp, sp, A16, A16, A4, A4, A4, A4, A4, A4, ws, pws, None) == 1           # refined
    m = L.prism_cp_merge
    assert m(cp_, sp, c.kappa + 1, A4, A4, A4, A4, ws, ws_n, None) == 1                # n_out
    assert m(pcp, sp, 3 * pc.kappa, A4, A4, A4, A4, ws, pws, None) == 1
    assert m(cp_, sp, c.kappa, None, A4, A4, A4, ws, ws_n, None) == 1
    assert m(cp_, sp, c.kappa, A4, A4, A4, A4, ws, ws_n - 1, None) == 3
    a = L.prism_cp_attn_local
    assert a(cp_, sp, A16, A16, None, A4, A4, A4, ws, ws_n, None) == 1                 # null v
    assert a(cp_, sp, A16, A16, MIS, A4, A4, A4, ws, ws_n, None) == 1
    assert a(cp_, sp, A16, A16, A16, A4, A4, A4, ws, ws_n - 1, None) == 3
    cb = L.prism_cp_combine
    assert cb(cp_, 0, A4, A16, None) == 1
    assert cb(cp_, 2, None, A16, None) == 1
    assert cb(cp_, 2, A4, MIS, None) == 1


def test_headers_compile_as_c_and_match_the_library(L, tmp_path):
    """include/prism.h and include/prism_cp.h are plain C: a C program built
    with gcc against them links libprism.so, and the struct layouts it sees
    give the same workspace sizes as the Python binding's."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no gcc")
    src = tmp_path / "abi.c"
    src.write_text(r"""
#include <stdio.h>
#include "prism.h"
#include "prism_cp.h"
int main(void) {
    uint8_t mask[4] = {1, 0, 2, 0};
    prism_config_t c = {1, 8, 2, 64, 4096, 256, 4, 4, mask, PRISM_MODE_REFINE,
                        PRISM_CHAIN_PREV, 0.0f, 0, 1};
    prism_cp_shard_t sh = {2, 1, 2048};
    size_t a = 0, b = 0;
    if (prism_workspace_size(&c, &a) != PRISM_OK) return 2;
    if (prism_cp_workspace_size(&c, &sh, &b) != PRISM_OK) return 3;
    printf("%d %zu %zu\n", prism_version(), a, b);
    return 0;
}
""")
    lib_dir = os.path.dirname(prism.LIB_PATH)
    exe = tmp_path / "abi"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), f"-L{lib_dir}", "-l:libprism.so",
                    f"-Wl,-rpath,{lib_dir}"], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    c = _cfg(anchor_mask=[1, 0, 2, 0])
    assert int(out[0]) == L.prism_version()
    assert int(out[1]) == prism.prism_workspace_size(c)
    assert int(out[2]) == prism.prism_cp_workspace_size(c, prism.CpShard(2, 1, 2048))
