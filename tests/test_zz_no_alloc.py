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
from parity_util import TOL, check_topk, kk_rows, oracle_attend, oracle_index, rel_err, to_np

pytestmark = pytest.mark.gpu

SPEC = LayerSpec(name="noalloc_csa_bf16", dtype="bf16", B=2, S_q=640, S_kv=640, q_pos0=0,
                 kv_pos0=0, H=64, D=512, R=64, base=160000.0, W=128, m=4, P=160, kind="csa",
                 H_I=64, d_I=128, topk=48, workload=99)
# run after SPEC: fewer scratch rows than the call before it, so rows a call failed to
# write itself would still hold the larger call's keys and show up as a mismatch
SPEC_SMALL = LayerSpec(name="noalloc_csa_small_bf16", dtype="bf16", B=1, S_q=300, S_kv=300,
                       q_pos0=0, kv_pos0=0, H=64, D=512, R=64, base=160000.0, W=96, m=4, P=75,
                       kind="csa", H_I=64, d_I=128, topk=32, workload=77)


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


def test_noalloc_matches_workspace_entry_and_oracle_twice():
    """Two calls in a row per shape, the larger shape first: each output equals the
    workspace entry point's bit for bit (same kernel, same inputs) and matches the oracle
    within the bf16 tolerance (the oracle attends over the GPU's pool and its validated
    top-k)."""
    lib, f = _noalloc_fn()
    for s in (SPEC, SPEC_SMALL):
        inp = cs.make_inputs(s, device="cuda")
        pool = csa.csa_compress(inp["kv"], inp["gate"], s.m, s.overlap)
        idx = csa.csa_index_topk(inp["q_I"], inp["w"], inp["k_I"], s.q_pos0, s.m, s.topk)
        ref = csa.csa_attend(inp["q"], inp["kv"], s.kv_pos0, pool, idx, inp["sink"], s.q_pos0,
                             s.R, s.base, s.W, s.m, s.scale)
        torch.cuda.synchronize()
        rows = list(range(s.S_q))
        sc, o_idx, _ = oracle_index(s, inp, rows)
        g_idx = idx.cpu().numpy()
        for b in range(s.B):
            check_topk(g_idx[b], o_idx[b], sc[b], kk_rows(s, rows))
        ora = oracle_attend(s, inp, rows, to_np(pool), g_idx)
        for _ in range(2):
            out = torch.full_like(inp["q"], float("nan"))
            _call_noalloc(f, lib, s, inp, pool, idx, out)
            torch.cuda.synchronize()
            assert torch.equal(out, ref), s.name
            assert rel_err(to_np(out), ora) <= TOL["bf16"], s.name
    assert csa.device_status() == 0


def test_noalloc_rejects_too_large_and_other_shapes():
    """Calls the fixed scratch cannot serve are refused on the host before any launch.
    Every buffer really holds the sizes the call declares, so a regression in the size
    guard would run a valid (if unsupported) call instead of touching memory out of
    bounds."""
    lib, f = _noalloc_fn()
    B, S_q, S_kv, P, H, D, topk = 1, 320, 20000, 160, 64, 512, 48
    bf = dict(dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((B, S_q, H, D), **bf)
    kv = torch.zeros((B, S_kv, D), **bf)
    pool = torch.zeros((B, P, D), **bf)
    idx = torch.full((B, S_q, topk), -1, dtype=torch.int32, device="cuda")
    sink = torch.zeros((H,), dtype=torch.float32, device="cuda")
    out = torch.empty_like(q)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    scale = 1.0 / math.sqrt(D)
    # B * (S_kv + P) = 20160 rotated rows: beyond the fixed scratch (S_q * 64 >= S_kv + P,
    # so it is the prefill shape the entry point handles, refused only for its size)
    rc = f(p(q), p(kv), S_kv, 0, p(pool), P, p(idx), topk, p(sink), p(out), B, S_q, 0, H, D, 64,
           160000.0, 128, 4, scale, csa.CSA_BF16, st)
    assert rc == -2
    assert "scratch" in lib.csa_last_error().decode()
    # head count other than 64 (q holds more than the 32 heads declared): not the shape
    # this entry point handles
    rc = f(p(q), p(kv), 600, 0, p(pool), P, p(idx), topk, p(sink), p(out), B, S_q, 0, 32, D, 64,
           160000.0, 128, 4, scale, csa.CSA_BF16, st)
    assert rc == -2
    torch.cuda.synchronize()
