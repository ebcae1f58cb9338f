"""The C-ABI library without a GPU: it loads, exports every function include/csa.h
declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import math
import os
import re

import pytest

import sparse_attention_14_b200 as csa
from sparse_attention_14_b200 import build as csa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    csa_build.build()
    return csa.load_library()


def _declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z_0-9]*\s*\*?\s*"
                                r"([a-z][a-z_0-9]*)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert {"csa_compress", "csa_index_topk", "csa_attend", "hca_attend"} <= set(names)
    for n in names:
        assert hasattr(lib, n), "missing export %s" % n
    assert lib.csa_version().decode().startswith("csa_b200")


FAKE = ctypes.c_void_p(0x10000)        # never dereferenced: every call below fails validation
MIS = ctypes.c_void_p(0x10004)         # misaligned


def _err(lib):
    return lib.csa_last_error().decode()


def test_compress_rejects(lib):
    assert lib.csa_compress(FAKE, FAKE, FAKE, 1, 16, 7, 4, 1, 1, None) == -1
    assert "multiple of 8" in _err(lib)
    assert lib.csa_compress(FAKE, FAKE, FAKE, 1, 16, 64, 0, 1, 1, None) == -1
    assert lib.csa_compress(FAKE, FAKE, FAKE, 1, 16, 64, 4, 2, 1, None) == -1
    assert lib.csa_compress(None, FAKE, FAKE, 1, 16, 64, 4, 1, 1, None) == -1
    assert lib.csa_compress(MIS, FAKE, FAKE, 1, 16, 64, 4, 1, 1, None) == -1
    assert "aligned" in _err(lib)
    assert lib.csa_compress(FAKE, FAKE, FAKE, 1, 16, 64, 4, 1, 7, None) == -1
    # empty pool (no window closed) and empty batch are valid no-ops
    assert lib.csa_compress(None, None, None, 1, 3, 64, 4, 1, 1, None) == 0
    assert lib.csa_compress(None, None, None, 0, 64, 64, 4, 1, 1, None) == 0


def test_compress_append_rejects(lib):
    args = lambda **kw: [kw.get("kv", FAKE), kw.get("g", FAKE), kw.get("ks", 4), kw.get("gs", 4),
                         kw.get("state", FAKE), kw.get("pool", FAKE), kw.get("cap", 64),
                         kw.get("B", 2), kw.get("n", 4), kw.get("pos", 8), kw.get("D", 64),
                         kw.get("ratio", 4), kw.get("overlap", 1), kw.get("dtype", 1), None]
    assert lib.csa_compress_append(*args(D=60)) == -1
    assert lib.csa_compress_append(*args(ratio=0)) == -1
    assert lib.csa_compress_append(*args(overlap=2)) == -1
    assert lib.csa_compress_append(*args(pos=-1)) == -1
    assert lib.csa_compress_append(*args(n=-1)) == -1
    assert lib.csa_compress_append(*args(dtype=5)) == -1
    assert lib.csa_compress_append(*args(ks=3)) == -1          # sequences would overlap
    assert lib.csa_compress_append(*args(state=None)) == -1
    assert lib.csa_compress_append(*args(kv=MIS)) == -1
    # entries up to position 11 close 3 entries: a 2-entry pool is too short
    assert lib.csa_compress_append(*args(cap=2)) == -1
    assert "pool_cap" in _err(lib)
    assert lib.csa_compress_append(*args(n=0)) == 0
    assert lib.csa_compress_append(*args(B=0)) == 0
    assert lib.csa_compress_state_bytes(3, 64, 4, 1, 1) == 3 * 2 * 8 * 64 * 2
    assert lib.csa_compress_state_bytes(3, 512, 128, 0, 0) == 3 * 2 * 128 * 512 * 4
    assert lib.csa_compress_state_bytes(3, 60, 4, 1, 1) == 0


def test_rope_rows_rejects(lib):
    args = lambda **kw: [kw.get("x", FAKE), kw.get("out", FAKE), kw.get("rows", 10),
                         kw.get("D", 128), kw.get("R", 64), kw.get("base", 160000.0),
                         kw.get("pos0", 0), kw.get("group", 1), kw.get("period", 10),
                         kw.get("step", 4), kw.get("dtype", 1), None]
    assert lib.csa_rope_rows(*args(D=60)) == -1
    assert lib.csa_rope_rows(*args(R=63)) == -1
    assert lib.csa_rope_rows(*args(R=136)) == -1          # wider than the row
    assert lib.csa_rope_rows(*args(D=1024, R=512)) == -1  # more than 128 pairs
    assert lib.csa_rope_rows(*args(base=0.0)) == -1
    assert lib.csa_rope_rows(*args(group=0)) == -1
    assert lib.csa_rope_rows(*args(period=0)) == -1
    assert lib.csa_rope_rows(*args(pos0=2 ** 31)) == -1
    assert lib.csa_rope_rows(*args(period=2 ** 29, step=8)) == -1
    assert lib.csa_rope_rows(*args(rows=-1)) == -1
    assert lib.csa_rope_rows(*args(x=None)) == -1
    assert lib.csa_rope_rows(*args(out=MIS)) == -1
    assert lib.csa_rope_rows(*args(dtype=3)) == -1
    # out overlapping x without being x
    assert lib.csa_rope_rows(*args(out=ctypes.c_void_p(0x10000 + 256))) == -1
    assert "overlap" in _err(lib)
    assert lib.csa_rope_rows(*args(rows=0)) == 0


def test_index_topk_rejects(lib):
    args = lambda **kw: [kw.get("q", FAKE), kw.get("w", FAKE), kw.get("k", FAKE), kw.get("B", 1),
                         kw.get("S", 8), kw.get("pos", 0), kw.get("P", 2), kw.get("HI", 4),
                         kw.get("dI", 32), kw.get("ratio", 4), kw.get("topk", 16),
                         kw.get("idx", FAKE), None, None, 0, 1, None]
    assert lib.csa_index_topk(*args(topk=0)) == -1
    assert lib.csa_index_topk(*args(topk=4096)) == -1
    assert lib.csa_index_topk(*args(dI=20)) == -1
    assert lib.csa_index_topk(*args(HI=0)) == -1
    assert lib.csa_index_topk(*args(pos=-1)) == -1
    assert lib.csa_index_topk(*args(ratio=0)) == -1
    assert lib.csa_index_topk(*args(idx=None)) == -1
    assert lib.csa_index_topk(*args(q=MIS)) == -1
    assert lib.csa_index_topk(*args(S=0)) == 0


def _attend_args(**kw):
    return [kw.get("q", FAKE), kw.get("kv", FAKE), kw.get("S_kv", 8), kw.get("kv_pos0", 0),
            kw.get("pool", FAKE), kw.get("P", 2), kw.get("idx", FAKE), kw.get("topk", 4),
            kw.get("sink", FAKE), kw.get("out", FAKE), kw.get("B", 1), kw.get("S_q", 8),
            kw.get("q_pos0", 0), kw.get("H", 4), kw.get("D", 64), kw.get("R", 16),
            kw.get("base", 10000.0), kw.get("W", 8), kw.get("ratio", 4), 0.125, None, 0, 1, None]


def test_attend_rejects(lib):
    assert lib.csa_attend(*_attend_args(R=15)) == -1
    assert lib.csa_attend(*_attend_args(R=80)) == -1
    assert lib.csa_attend(*_attend_args(D=60)) == -1
    assert lib.csa_attend(*_attend_args(W=0)) == -1
    assert lib.csa_attend(*_attend_args(q_pos0=-3)) == -1
    assert lib.csa_attend(*_attend_args(base=0.0)) == -1
    assert lib.csa_attend(*_attend_args(idx=None)) == -1
    assert lib.csa_attend(*_attend_args(topk=0)) == -1
    assert lib.csa_attend(*_attend_args(out=MIS)) == -1
    assert lib.csa_attend(*_attend_args(B=0)) == 0
    a = _attend_args(R=15)
    del a[6:8]  # hca_attend has no idx / topk
    assert lib.hca_attend(*a) == -1


def test_binding_raises_without_device_tensors(lib):
    import torch
    x = torch.zeros(1, 8, 64)
    with pytest.raises(ValueError):
        csa.csa_compress(x, x, 4, True)


def _ws_index(B, S_q, q_pos0, P, topk, dtype=None):
    import torch
    return csa.csa_index_topk_workspace_bytes(B, S_q, q_pos0, P, 64, 128, 4, topk,
                                              dtype or torch.bfloat16)


def test_index_workspace_plan(lib):
    """The indexer's workspace query, host logic only: one row of 32-bit score keys per
    query (pitch round_up(P, 4), the total rounded up to 256 bytes) whenever every row has
    at most 16384 visible entries -- prefill calls whose key rows take at most 2 GiB and
    split decode calls -- else candidates (decode) or none (prefill)."""
    import torch
    up = lambda n: (n + 255) // 256 * 256
    # S=8192 prefill, P=2048: 8192 rows of 2048 keys
    assert _ws_index(1, 8192, 0, 2048, 512) == 8192 * 2048 * 4
    # odd P: rows padded to a multiple of 4 keys
    assert _ws_index(2, 603, 0, 150, 64) == up(2 * 603 * 152 * 4)
    # rows longer than 16384 visible entries keep the shared-memory candidates: no workspace
    assert _ws_index(1, 131072, 0, 32768, 512) == 0
    # key rows above 2 GiB (65536 rows of 16384 keys = 4 GiB): candidates, no workspace
    assert _ws_index(1, 65536, 0, 16384, 512) == 0
    # decode, 64 rows at 65536 cached tokens: split over entry ranges, keys of every entry
    assert _ws_index(64, 1, 65535, 16384, 512) == 64 * 16384 * 4
    # decode rows beyond 16384 visible entries: per-range candidates (64-bit keys)
    ws = _ws_index(64, 1, 4 * 20000 - 1, 20000, 512)
    assert ws > 0 and ws % (64 * 512 * 8) == 0
    # the general (fp32) path needs none
    assert _ws_index(1, 8192, 0, 2048, 512, torch.float32) == 0
