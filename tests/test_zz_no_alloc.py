"""csa_attend_noalloc: the attention entry point for callers that cannot allocate device
memory (an operator inside a framework that owns all device memory and passes only
input/output buffers, or a serving loop that must not call cudaMalloc per request).
It keeps its scratch in a fixed array inside the library.  This file is collected last
on purpose: if it fails, a run that stops at the first failure has already run the
other tests.  It must pass alone in a fresh process too."""
import ctypes
import math

import numpy as np
import pytest
import torch

import csa_synth as cs
from csa_synth import LayerSpec
import sparse_attention_14_b200 as csa
from parity_util import TOL, rel_err, to_np

pytestmark = pytest.mark.gpu

SPEC = LayerSpec(name="noalloc_csa_bf16", dtype="bf16", B=2, S_q=640, S_kv=640, q_pos0=0,
                 kv_pos0=0, H=64, D=512, R=64, base=160000.0, W=128, m=4, P=160, kind="csa",
                 H_I=64, d_I=128, topk=48, workload=99)


def _noalloc_fn():
    lib = csa.load_library()
    f = lib.csa_attend_noalloc
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    f.argtypes = [vp, vp, i64, i64, vp, i64, vp, i32, vp, vp, i64, i64, i64, i32, i32, i32,
                  ctypes.c_double, i32, i32, ctypes.c_float, ctypes.c_int, vp]
    f.restype = ctypes.c_int
    return lib, f


def _call_noalloc(f, lib, s, inp, pool, idx, out):
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = f(p(inp["q"]), p(inp["kv"]), s.S_kv, s.kv_pos0, p(pool), s.P, p(idx), s.topk,
           p(inp["sink"]), p(out), s.B, s.S_q, s.q_pos0, s.H, s.D, s.R, s.base, s.W, s.m,
           s.scale, csa.CSA_BF16, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, lib.csa_last_error().decode()


def test_noalloc_matches_workspace_entry_twice():
    s = SPEC
    lib, f = _noalloc_fn()
    inp = cs.make_inputs(s, device="cuda")
    pool = csa.csa_compress(inp["kv"], inp["gate"], s.m, s.overlap)
    idx = csa.csa_index_topk(inp["q_I"], inp["w"], inp["k_I"], s.q_pos0, s.m, s.topk)
    ref = csa.csa_attend(inp["q"], inp["kv"], s.kv_pos0, pool, idx, inp["sink"], s.q_pos0, s.R,
                         s.base, s.W, s.m, s.scale)
    for _ in range(2):
        out = torch.full_like(inp["q"], float("nan"))
        _call_noalloc(f, lib, s, inp, pool, idx, out)
        torch.cuda.synchronize()
        assert rel_err(to_np(out), to_np(ref)) <= TOL["bf16"]
    assert csa.device_status() == 0


def test_noalloc_rejects_too_large_and_other_shapes():
    lib, f = _noalloc_fn()
    s = SPEC
    inp = cs.make_inputs(s, device="cuda")
    pool = torch.zeros((s.B, s.P, s.D), dtype=torch.bfloat16, device="cuda")
    idx = torch.full((s.B, s.S_q, s.topk), -1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(inp["q"])
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # 20000 rows of kv per sequence: beyond the fixed scratch (checked before any launch)
    rc = f(p(inp["q"]), p(inp["kv"]), 20000, 0, p(pool), s.P, p(idx), s.topk, p(inp["sink"]),
           p(out), s.B, 20000, 0, s.H, s.D, s.R, s.base, s.W, s.m, s.scale, csa.CSA_BF16, st)
    assert rc == -2
    assert "scratch" in lib.csa_last_error().decode()
    # head count other than 64: not the shape this entry point handles
    rc = f(p(inp["q"]), p(inp["kv"]), s.S_kv, 0, p(pool), s.P, p(idx), s.topk, p(inp["sink"]),
           p(out), s.B, s.S_q, 0, 32, s.D, s.R, s.base, s.W, s.m, s.scale, csa.CSA_BF16, st)
    assert rc == -2
