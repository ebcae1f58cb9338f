"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the same seeded
inputs.  Small and mid shapes are checked on every query row (several tiles and a ragged
tail); the five full workloads are checked end to end on sampled rows, in the launch
configuration the benchmark times.  Tolerances are in parity_util."""
from __future__ import annotations

import random

import numpy as np
import pytest
import torch

import csa_synth as cs
import oracle
import sparse_attention_14_b200 as csa
from csa_synth import LayerSpec
from parity_util import (TOL, GpuLayer, check_topk, gpu_cache_update_checked, kk_rows,
                         oracle_attend, oracle_index, oracle_pool, rel_err, to_np)

pytestmark = pytest.mark.gpu

DEV = "cuda"

MID = [
    # fp32, ragged sizes, two sequences
    LayerSpec(name="mid_csa_f32", dtype="f32", B=2, S_q=301, S_kv=301, q_pos0=0, kv_pos0=0, H=8,
              D=64, R=16, base=10000.0, W=32, m=4, P=75, kind="csa", H_I=4, d_I=32, topk=16,
              workload=90),
    # V4-Flash head shape, several key tiles, ragged tail
    LayerSpec(name="mid_csa_bf16", dtype="bf16", B=2, S_q=603, S_kv=603, q_pos0=0, kv_pos0=0,
              H=64, D=512, R=64, base=160000.0, W=128, m=4, P=150, kind="csa", H_I=64, d_I=128,
              topk=64, workload=91),
    LayerSpec(name="mid_hca_bf16", dtype="bf16", B=1, S_q=1000, S_kv=1000, q_pos0=0, kv_pos0=0,
              H=64, D=512, R=64, base=160000.0, W=128, m=128, P=7, kind="hca", workload=92),
    LayerSpec(name="mid_sliding_bf16", dtype="bf16", B=1, S_q=300, S_kv=300, q_pos0=0, kv_pos0=0,
              H=16, D=128, R=32, base=10000.0, W=64, m=4, P=0, kind="sliding", workload=93),
    LayerSpec(name="mid_decode_bf16", dtype="bf16", B=3, S_q=1, S_kv=128, q_pos0=4095,
              kv_pos0=3968, H=64, D=512, R=64, base=160000.0, W=128, m=4, P=1024, kind="csa",
              H_I=64, d_I=128, topk=64, decode=True, workload=94),
    # decode-sized calls whose key tiles are split over two CTAs and merged by the combine
    # kernel: HCA entries, and several queries per sequence over a window of 130 rows
    LayerSpec(name="mid_hca_decode_bf16", dtype="bf16", B=2, S_q=1, S_kv=128, q_pos0=2047,
              kv_pos0=1920, H=64, D=512, R=64, base=160000.0, W=128, m=128, P=16, kind="hca",
              decode=True, workload=87),
    LayerSpec(name="mid_decode_sq3_bf16", dtype="bf16", B=2, S_q=3, S_kv=130, q_pos0=4093,
              kv_pos0=3966, H=64, D=512, R=64, base=160000.0, W=128, m=4, P=1024, kind="csa",
              H_I=64, d_I=128, topk=64, decode=True, workload=86),
    # V4-Flash head shape on the tensor-core path: window-only layer, and a CSA layer
    # whose key count per query is not a multiple of the 128-key tile
    LayerSpec(name="mid_sliding_tc_bf16", dtype="bf16", B=2, S_q=333, S_kv=333, q_pos0=0,
              kv_pos0=0, H=64, D=512, R=64, base=10000.0, W=128, m=4, P=0, kind="sliding",
              workload=97),
    LayerSpec(name="mid_csa_ragged_bf16", dtype="bf16", B=1, S_q=700, S_kv=700, q_pos0=0,
              kv_pos0=0, H=64, D=512, R=64, base=160000.0, W=100, m=4, P=175, kind="csa",
              H_I=64, d_I=128, topk=37, workload=98),
    # a window longer than one 128-key tile, HCA-style entries
    LayerSpec(name="mid_hca_w200_bf16", dtype="bf16", B=2, S_q=600, S_kv=600, q_pos0=0,
              kv_pos0=0, H=64, D=512, R=64, base=160000.0, W=200, m=16, P=37, kind="hca",
              workload=88),
    # indexer buffer cuts (more than 1024 visible entries) and a top-k that is not a
    # power of two
    LayerSpec(name="mid_csa_cut_bf16", dtype="bf16", B=1, S_q=4801, S_kv=4801, q_pos0=0,
              kv_pos0=0, H=64, D=512, R=64, base=160000.0, W=128, m=4, P=1200, kind="csa",
              H_I=64, d_I=128, topk=200, workload=89),
    # decode steps that first run the compressor cache update: three new tokens closing the
    # last CSA entry (main and indexer keys), and one HCA token closing a 128-token window
    # whose state reaches back before the attention window
    LayerSpec(name="mid_decode_step_bf16", dtype="bf16", B=2, S_q=3, S_kv=130, q_pos0=4093,
              kv_pos0=3966, H=64, D=512, R=64, base=160000.0, W=128, m=4, P=1024, kind="csa",
              H_I=64, d_I=128, topk=64, decode=True, cache_update=True, workload=85),
    LayerSpec(name="mid_hca_decode_step_bf16", dtype="bf16", B=2, S_q=1, S_kv=128,
              q_pos0=2047, kv_pos0=1920, H=64, D=512, R=64, base=160000.0, W=128, m=128, P=16,
              kind="hca", decode=True, cache_update=True, workload=84),
    # chunked prefill: queries and raw rows start at position 1024 (a multiple of m and of
    # m'), over a resident pool of the whole sequence so far; tensor-core path (CSA, HCA)
    # and general path
    LayerSpec(name="chunk_csa_bf16", dtype="bf16", B=1, S_q=520, S_kv=520, q_pos0=1024,
              kv_pos0=1024, H=64, D=512, R=64, base=160000.0, W=128, m=4, P=386, kind="csa",
              H_I=64, d_I=128, topk=96, decode=True, workload=83),
    LayerSpec(name="chunk_hca_bf16", dtype="bf16", B=2, S_q=300, S_kv=300, q_pos0=1024,
              kv_pos0=1024, H=64, D=512, R=64, base=160000.0, W=128, m=128, P=10, kind="hca",
              decode=True, workload=82),
    LayerSpec(name="chunk_csa_f32", dtype="f32", B=2, S_q=150, S_kv=150, q_pos0=1024,
              kv_pos0=1024, H=8, D=64, R=16, base=10000.0, W=32, m=4, P=293, kind="csa", H_I=4,
              d_I=32, topk=16, decode=True, workload=81),
    # CSA calls with no compressed entry at all (P = 0): a prefill shorter than m, on the
    # tensor-core and the general path, and a window-only CSA call over three key tiles
    LayerSpec(name="p0_csa_bf16", dtype="bf16", B=2, S_q=3, S_kv=3, q_pos0=0, kv_pos0=0, H=64,
              D=512, R=64, base=160000.0, W=128, m=4, P=0, kind="csa", H_I=64, d_I=128, topk=16,
              workload=80),
    LayerSpec(name="p0_csa_f32", dtype="f32", B=1, S_q=3, S_kv=3, q_pos0=0, kv_pos0=0, H=8,
              D=64, R=16, base=10000.0, W=32, m=4, P=0, kind="csa", H_I=4, d_I=32, topk=16,
              workload=79),
    LayerSpec(name="p0_csa_window_bf16", dtype="bf16", B=1, S_q=300, S_kv=300, q_pos0=0,
              kv_pos0=0, H=64, D=512, R=64, base=160000.0, W=300, m=4, P=0, kind="csa", H_I=64,
              d_I=128, topk=32, decode=True, workload=78),
    # decode-sized calls at an early position: no entry is visible yet, so the query has a
    # single (window) key tile and the second CTA of its split pair has none (an empty
    # partial merged by the first); CSA and HCA
    LayerSpec(name="early_decode_csa_bf16", dtype="bf16", B=3, S_q=1, S_kv=3, q_pos0=2,
              kv_pos0=0, H=64, D=512, R=64, base=160000.0, W=128, m=4, P=100, kind="csa",
              H_I=64, d_I=128, topk=64, decode=True, workload=77),
    LayerSpec(name="early_decode_hca_bf16", dtype="bf16", B=2, S_q=1, S_kv=100, q_pos0=99,
              kv_pos0=0, H=64, D=512, R=64, base=160000.0, W=128, m=128, P=4, kind="hca",
              decode=True, workload=76),
    # odd shapes: general path
    LayerSpec(name="odd_csa_bf16", dtype="bf16", B=1, S_q=77, S_kv=77, q_pos0=0, kv_pos0=0, H=5,
              D=40, R=8, base=10000.0, W=9, m=3, P=25, kind="csa", H_I=3, d_I=24, topk=7,
              workload=95),
    # k > n_vis everywhere, window longer than the sequence
    LayerSpec(name="sat_csa_f32", dtype="f32", B=1, S_q=50, S_kv=50, q_pos0=0, kv_pos0=0, H=4,
              D=32, R=8, base=10000.0, W=64, m=4, P=12, kind="csa", H_I=2, d_I=16, topk=32,
              workload=96),
]


def _inputs(spec):
    return cs.make_inputs(spec, device=DEV)


def _pool_input(spec, inp, ora_pool):
    """Pool both sides attend over in the stage-wise check: the oracle's pool rounded to
    the layer dtype (decode: the resident cache itself)."""
    if spec.decode:
        return inp["pool"]
    if ora_pool is None:
        return None
    return torch.from_numpy(ora_pool).to(device=DEV, dtype=spec.torch_dtype)


@pytest.mark.parametrize("spec", MID, ids=[s.name for s in MID])
def test_compress_parity(spec):
    if spec.decode or spec.kind == "sliding":
        pytest.skip("no compressor in this layer")
    inp = _inputs(spec)
    gpu = GpuLayer(spec, inp).compress()
    torch.cuda.synchronize()
    ref = oracle_pool(spec, inp)
    assert gpu.shape == ref.shape
    assert rel_err(to_np(gpu), ref) <= TOL[spec.dtype]


@pytest.mark.parametrize("spec", [s for s in MID if s.kind == "csa"],
                         ids=[s.name for s in MID if s.kind == "csa"])
def test_index_topk_parity(spec):
    inp = _inputs(spec)
    idx, scores = GpuLayer(spec, inp).index(want_scores=True)
    torch.cuda.synchronize()
    rows = list(range(spec.S_q))
    sc, o_idx, o_sel = oracle_index(spec, inp, rows)
    g_idx = idx.cpu().numpy()
    g_sc = scores.cpu().numpy().astype(np.float64)
    for b in range(spec.B):
        check_topk(g_idx[b], o_idx[b], sc[b], kk_rows(spec, rows))
        # the kept entries come in ascending entry order, and each carries its own score
        for r in range(len(rows)):
            kk = kk_rows(spec, rows)[r]
            assert (np.diff(g_idx[b, r, :kk]) > 0).all(), "row %d not in ascending order" % r
        valid = g_idx[b] >= 0
        if spec.P == 0:
            assert not valid.any()
            continue
        ref = np.where(valid, np.take_along_axis(sc[b], np.maximum(g_idx[b], 0), axis=1), 0.0)
        assert rel_err(np.where(valid, g_sc[b], 0.0), ref) <= TOL[spec.dtype] * 0.05


@pytest.mark.parametrize("spec", MID, ids=[s.name for s in MID])
def test_attend_stagewise_parity(spec):
    """Both sides attend over identical inputs: the oracle's pool (rounded to the layer
    dtype) and the oracle's top-k."""
    inp = _inputs(spec)
    rows = list(range(spec.S_q))
    ora_pool = oracle_pool(spec, inp)
    pool_in = _pool_input(spec, inp, ora_pool)
    idx_in = None
    o_idx = None
    if spec.kind == "csa":
        _, o_idx, _ = oracle_index(spec, inp, rows)
        idx_in = torch.from_numpy(o_idx).to(DEV)
    out = GpuLayer(spec, inp).attend(pool_in, idx_in)
    torch.cuda.synchronize()
    ref = oracle_attend(spec, inp, rows, None if pool_in is None else to_np(pool_in), o_idx)
    assert rel_err(to_np(out), ref) <= TOL[spec.dtype]


def test_decode_split_sink_minus_inf():
    """The combine kernel adds the sink once: with a sink of -inf on half the heads (the
    plain softmax over the keys) the split decode path still matches the oracle."""
    spec = next(x for x in MID if x.name == "mid_decode_bf16")
    inp = _inputs(spec)
    inp["sink"][::2] = float("-inf")
    rows = list(range(spec.S_q))
    _, o_idx, _ = oracle_index(spec, inp, rows)
    out = GpuLayer(spec, inp).attend(inp["pool"], torch.from_numpy(o_idx).to(DEV))
    torch.cuda.synchronize()
    ref = oracle_attend(spec, inp, rows, to_np(inp["pool"]), o_idx)
    assert np.isfinite(to_np(out)).all()
    assert rel_err(to_np(out), ref) <= TOL[spec.dtype]


SINK_CASES = [("mid_csa_bf16", "all"), ("mid_csa_bf16", "half"), ("mid_hca_bf16", "all"),
              ("mid_hca_bf16", "half"), ("mid_csa_f32", "all"), ("mid_csa_f32", "half"),
              ("chunk_csa_bf16", "half")]


@pytest.mark.parametrize("name,pattern", SINK_CASES, ids=["%s-%s" % c for c in SINK_CASES])
def test_sink_minus_inf(name, pattern):
    """A sink of -inf (the plain softmax over the keys) on every head or on every other
    head.  On the prefill tensor-core path the sink is the initial running maximum, so
    -inf there takes its own branch (no exponent of the sink, the first tile sets the
    maximum); the general path and chunked prefill are covered too.  Stage-wise: both
    sides attend over the oracle's pool (rounded to the layer dtype) and top-k."""
    spec = next(x for x in MID if x.name == name)
    inp = _inputs(spec)
    if pattern == "all":
        inp["sink"][:] = float("-inf")
    else:
        inp["sink"][::2] = float("-inf")
    rows = list(range(spec.S_q))
    ora_pool = oracle_pool(spec, inp)
    pool_in = _pool_input(spec, inp, ora_pool)
    o_idx = idx_in = None
    if spec.kind == "csa":
        _, o_idx, _ = oracle_index(spec, inp, rows)
        idx_in = torch.from_numpy(o_idx).to(DEV)
    out = GpuLayer(spec, inp).attend(pool_in, idx_in)
    torch.cuda.synchronize()
    ref = oracle_attend(spec, inp, rows, None if pool_in is None else to_np(pool_in), o_idx)
    assert np.isfinite(ref).all()
    assert np.isfinite(to_np(out)).all()
    assert rel_err(to_np(out), ref) <= TOL[spec.dtype]


def test_tensor_core_path_selected():
    """The V4-Flash head shape takes the tensor-core attention, which needs a workspace
    (rotated keys for prefill, rotated rope chunks of the used keys for decode-sized
    calls); other shapes take the general path."""
    import sparse_attention_14_b200 as csa
    for spec in MID + cs.WORKLOADS[1] + cs.WORKLOADS[2] + cs.WORKLOADS[3]:
        ws = csa.csa_attend_workspace_bytes(0 if spec.kind == "csa" else 1, spec.B, spec.S_q,
                                            spec.S_kv, spec.P, spec.H, spec.D, spec.topk,
                                            spec.torch_dtype)
        tc = spec.dtype == "bf16" and spec.H == 64 and spec.D == 512 and spec.R <= 64
        assert (ws > 0) == tc, spec.name


@pytest.mark.parametrize("S_q,q_pos0,P,topk", [(1203, 0, 1100, 300), (1, 8191, 2048, 512),
                                               (3, 5000, 1500, 896)])
def test_index_all_ties_take_lowest_entries(S_q, q_pos0, P, topk):
    """q_I = 0 makes every score exactly 0: the kept entries must be the lowest visible
    indices (equal scores rank the lower index first), in ascending order; exact."""
    import sparse_attention_14_b200 as csa
    B, m = 2, 4
    q_I = torch.zeros((B, S_q, 64, 128), dtype=torch.bfloat16, device=DEV)
    w = torch.randn((B, S_q, 64), device=DEV).to(torch.bfloat16)
    k_I = torch.randn((B, P, 128), device=DEV).to(torch.bfloat16)
    idx = csa.csa_index_topk(q_I, w, k_I, q_pos0, m, topk).cpu().numpy()
    for i in range(S_q):
        nv = min(P, (q_pos0 + i + 1) // m)
        kk = min(topk, nv)
        want = list(range(kk)) + [-1] * (topk - kk)
        assert idx[0, i].tolist() == want and idx[1, i].tolist() == want, i


@pytest.mark.parametrize("B,S_q,q_pos0,P,topk", [(1, 1200, 12000, 3001, 512), (2, 600, 40000, 9003, 1024),
                                                 (1, 1201, 4947, 1537, 512)])
def test_index_prefill_key_stream_parity(B, S_q, q_pos0, P, topk):
    """Prefill-sized calls go through the persistent key stream and a selection kernel
    sized by the longest row: rows of up to 4096 and 16384 visible entries (block
    selects), and a row-length ramp up to 1537 entries (one warp per row) with an odd P,
    so the key rows are padded.  Sampled rows against the oracle."""
    g = torch.Generator().manual_seed(S_q * 7 + P)
    q_I = (torch.randn((B, S_q, 64, 128), generator=g) * 0.5).to(torch.bfloat16)
    w = torch.randn((B, S_q, 64), generator=g).to(torch.bfloat16)
    k_I = torch.randn((B, P, 128), generator=g).to(torch.bfloat16)
    idx, scores = csa.csa_index_topk(q_I.to(DEV), w.to(DEV), k_I.to(DEV), q_pos0, 4, topk, want_scores=True)
    assert csa.csa_index_topk_workspace_bytes(B, S_q, q_pos0, P, 64, 128, 4, topk) > 0
    torch.cuda.synchronize()
    rows = sorted(random.Random(P).sample(range(S_q), 12) + [0, S_q - 1])
    tpos = np.asarray(rows, dtype=np.int64) + q_pos0
    sc = oracle.index_scores(to_np(q_I[:, rows]), to_np(w[:, rows]), to_np(k_I), tpos, 4)
    o_idx, _ = oracle.topk(sc, tpos, 4, topk)
    g_idx = idx.cpu().numpy()[:, rows]
    g_sc = scores.cpu().numpy()[:, rows].astype(np.float64)
    kk = [min(topk, oracle.n_visible(int(t), 4, P)) for t in tpos]
    for b in range(B):
        check_topk(g_idx[b], o_idx[b], sc[b], kk)
        for r in range(len(rows)):
            assert (np.diff(g_idx[b, r, :kk[r]]) > 0).all(), "row %d not in ascending order" % rows[r]
        valid = g_idx[b] >= 0
        ref = np.where(valid, np.take_along_axis(sc[b], np.maximum(g_idx[b], 0), axis=1), 0.0)
        assert rel_err(np.where(valid, g_sc[b], 0.0), ref) <= TOL["bf16"] * 0.05


def test_no_kernel_gave_up():
    import sparse_attention_14_b200 as csa
    spec = MID[1]
    _end_to_end(spec, list(range(spec.S_q)))
    assert csa.device_status() == 0


def _end_to_end(spec, rows, inp=None, e2e_rows=128):
    """The whole layer on the GPU, every given row checked.

    Stage-wise gate (every row): once check_topk has validated the GPU's selection, the
    oracle attends over the GPU's own top-k and the GPU's pool, so a near-tie swap inside
    the tie band (a legitimate difference) cannot hide or excuse an attention error.
    End to end (the oracle's own pool and top-k): on up to `e2e_rows` rows whose selection
    equals the oracle's in every sequence of the batch."""
    inp = _inputs(spec) if inp is None else inp
    layer = GpuLayer(spec, inp)
    if spec.cache_update:
        gpu_cache_update_checked(spec, inp)
    pool = None
    if spec.decode:
        pool = inp["pool"]
    elif spec.kind != "sliding":
        pool = layer.compress()
    idx = layer.index(want_scores=False) if spec.kind == "csa" else None
    out = layer.attend(pool, idx)
    torch.cuda.synchronize()
    rows_t = torch.tensor(rows, device=DEV)
    g_out = to_np(out[:, rows_t])
    assert np.isfinite(g_out).all()
    ora_pool = oracle_pool(spec, inp)
    if pool is not None and not spec.decode:
        assert rel_err(to_np(pool), ora_pool) <= TOL[spec.dtype]
    same = np.ones((spec.B, len(rows)), dtype=bool)
    o_idx = g_idx = None
    if spec.kind == "csa":
        sc, o_idx, _ = oracle_index(spec, inp, rows)
        g_idx = idx[:, rows_t].cpu().numpy()
        for b in range(spec.B):
            check_topk(g_idx[b], o_idx[b], sc[b], kk_rows(spec, rows))
            for r in range(len(rows)):
                same[b, r] = set(g_idx[b, r].tolist()) == set(o_idx[b, r].tolist())
    ref_stage = oracle_attend(spec, inp, rows, None if pool is None else to_np(pool), g_idx)
    assert rel_err(g_out, ref_stage) <= TOL[spec.dtype]
    agree = [k for k in range(len(rows)) if same[:, k].all()][:e2e_rows]
    if agree:
        sub = [rows[k] for k in agree]
        ref = oracle_attend(spec, inp, sub, ora_pool, None if o_idx is None else o_idx[:, agree])
        assert rel_err(g_out[:, agree], ref) <= TOL[spec.dtype]
    return inp, out


@pytest.mark.parametrize("spec", MID, ids=[s.name for s in MID])
def test_end_to_end_parity(spec):
    _end_to_end(spec, list(range(spec.S_q)))


@pytest.mark.parametrize("workload", [0, 1, 2, 3, 5])
def test_workload_end_to_end(workload):
    for spec in cs.WORKLOADS[workload]:
        rows = list(range(spec.S_q)) if spec.S_q <= 512 else cs.sample_rows(spec, n_random=96)
        _end_to_end(spec, rows)
        torch.cuda.empty_cache()


@pytest.mark.parametrize("layer", [0, 1, 2, 3])
def test_mixed_stack_layer_end_to_end(layer):
    spec = cs.WORKLOADS[4][layer]
    rows = cs.sample_rows(spec, n_random=48)
    _end_to_end(spec, rows)
    torch.cuda.empty_cache()


# ----------------------------------------------------------------------------- cache update
def _chunks(seed, S, m, L):
    r = random.Random(seed)
    sizes = [1, 1, 1, 2, max(1, m - 1), m, L, L + 1, 3 * L + 2, 40]
    out = []
    while sum(out) < S:
        out.append(min(r.choice(sizes), S - sum(out)))
    return out


APPEND_CASES = [  # name, dtype, B, S, D, ratio, overlap
    ("csa_kv_bf16", torch.bfloat16, 3, 203, 512, 4, 1),
    ("csa_index_keys_bf16", torch.bfloat16, 2, 157, 128, 4, 1),
    ("hca_kv_bf16", torch.bfloat16, 2, 421, 512, 128, 0),
    ("csa_kv_f32", torch.float32, 2, 99, 64, 4, 1),
    ("odd_ratio_f32", torch.float32, 3, 50, 24, 3, 0),
    ("wide_ratio2_bf16", torch.bfloat16, 1, 37, 1024, 2, 1),
]


@pytest.mark.parametrize("name,dt,B,S,D,ratio,overlap", APPEND_CASES,
                         ids=[c[0] for c in APPEND_CASES])
def test_append_stream_parity(name, dt, B, S, D, ratio, overlap):
    """A token stream fed in calls of 1 .. 3L+2 rows, each a strided view of one buffer:
    after every call the entries that closed match the oracle's stateful compressor and
    the rest of the pool is untouched; at the end the whole pool matches the stateless
    oracle and the state holds the last L rows bit for bit."""
    seed = 600 + [c[0] for c in APPEND_CASES].index(name)
    kv, gate = cs.stream_rows(B, S, D, dt, seed, device=DEV)
    L = (1 + overlap) * ratio
    tol = TOL["f32" if dt == torch.float32 else "bf16"]
    state = csa.csa_compress_state(B, D, ratio, overlap, dtype=dt)
    pool = torch.zeros((B, S // ratio + 2, D), dtype=dt, device=DEV)
    ora = oracle.CompressorState(B, D, ratio, overlap)
    kv_h, gate_h = to_np(kv), to_np(gate)
    pos = 0
    for n in _chunks(seed, S, ratio, L):
        csa.csa_compress_append(kv[:, pos:pos + n], gate[:, pos:pos + n], state, pos, ratio,
                                overlap, pool=pool)
        ent = ora.append(kv_h[:, pos:pos + n], gate_h[:, pos:pos + n])
        torch.cuda.synchronize()
        j0 = pos // ratio
        if ent.shape[1]:
            assert rel_err(to_np(pool[:, j0:j0 + ent.shape[1]]), ent) <= tol, (pos, n)
        assert (pool[:, j0 + ent.shape[1]:] == 0).all(), (pos, n)
        pos += n
    assert rel_err(to_np(pool[:, :S // ratio]), oracle.compress(kv_h, gate_h, ratio, overlap)) <= tol
    for p in range(max(0, S - L), S):
        assert torch.equal(state[:, 0, p % L], kv[:, p]) and torch.equal(state[:, 1, p % L], gate[:, p])


@pytest.mark.parametrize("ratio,overlap,S0,S", [(4, 1, 61, 90), (128, 0, 300, 530), (4, 1, 5, 20)])
def test_append_resumes_after_prefill(ratio, overlap, S0, S):
    """Prefill pooled by csa_compress, its tail stored into a state that starts as NaN
    (a state-only call, no pool), then decode one token per call: every entry matches the
    stateless oracle over the whole sequence, so the state's initial contents were never
    read."""
    B, D, dt = 2, 512, torch.bfloat16
    kv, gate = cs.stream_rows(B, S, D, dt, 700 + ratio, device=DEV)
    L = (1 + overlap) * ratio
    pool = torch.zeros((B, S // ratio, D), dtype=dt, device=DEV)
    P0 = S0 // ratio
    if P0:
        pool[:, :P0] = csa.csa_compress(kv[:, :S0].contiguous(), gate[:, :S0].contiguous(), ratio,
                                        overlap)
    state = torch.full((B, 2, L, D), float("nan"), dtype=dt, device=DEV)
    t = max(0, S0 - L)
    csa.csa_compress_append(kv[:, t:S0], gate[:, t:S0], state, t, ratio, overlap)
    for p in range(S0, S):
        csa.csa_compress_append(kv[:, p:p + 1], gate[:, p:p + 1], state, p, ratio, overlap,
                                pool=pool)
    torch.cuda.synchronize()
    ref = oracle.compress(to_np(kv), to_np(gate), ratio, overlap)
    got = to_np(pool)
    assert np.isfinite(got).all()
    assert rel_err(got, ref) <= TOL["bf16"]


# ----------------------------------------------------------------------------- indexer RoPE
ROPE_CASES = [  # name, dtype, shape, group, period, step, pos0, rope_dim, base
    ("q_I_bf16", torch.bfloat16, (2, 37, 5, 128), 5, 37, 1, 4000, 64, 160000.0),
    ("k_I_bf16", torch.bfloat16, (2, 50, 128), 1, 50, 4, 0, 64, 160000.0),
    ("odd_f32", torch.float32, (3, 11, 40), 1, 33, 3, 7, 8, 10000.0),
    ("full_width_far_f32", torch.float32, (4, 16), 2, 2, 5, 2 ** 30, 16, 10000.0),
    # groups of rows at one position (64 heads per query; 21 rows in groups of 4, the last
    # one partial): the kernel that computes the angles once per group and column
    ("q_I_h64_bf16", torch.bfloat16, (2, 37, 64, 128), 64, 37, 1, 4000, 64, 160000.0),
    ("ragged_groups_bf16", torch.bfloat16, (3, 7, 128), 4, 5, 3, 11, 64, 10000.0),
]


@pytest.mark.parametrize("name,dt,shape,group,period,step,pos0,R,base", ROPE_CASES,
                         ids=[c[0] for c in ROPE_CASES])
def test_rope_rows_parity(name, dt, shape, group, period, step, pos0, R, base):
    """csa_rope_rows against the oracle's rotation row by row, out of place and in place;
    the channels before the rotated ones are copied bit for bit."""
    x = cs.normal_rows(shape, dt, 800 + [c[0] for c in ROPE_CASES].index(name), device=DEV)
    D = shape[-1]
    rows = x.numel() // D
    out = csa.csa_rope_rows(x, pos0, group, period, step, R, base)
    xi = x.clone()
    csa.csa_rope_rows(xi, pos0, group, period, step, R, base, out=xi)
    torch.cuda.synchronize()
    pos = pos0 + ((np.arange(rows) // group) % period) * step
    ref = oracle.rope(to_np(x).reshape(rows, D), pos, R, base)
    tol = TOL["f32" if dt == torch.float32 else "bf16"]
    assert rel_err(to_np(out).reshape(rows, D), ref) <= tol
    assert torch.equal(out, xi)
    assert torch.equal(out[..., :D - R], x[..., :D - R])


def _pooled_index_keys(spec, dt):
    """Per-token index keys and their gates (seeded), pooled like the main compressor."""
    kI_tok, gI_tok = cs.stream_rows(spec.B, spec.S_kv, spec.d_I, dt, 900 + spec.workload, device=DEV)
    return kI_tok, gI_tok, csa.csa_compress(kI_tok, gI_tok, spec.m, spec.overlap)


def test_indexer_key_pooling_and_rope_end_to_end_f32():
    """The indexer's key path in full (fp32, so top-k sets are compared directly):
    per-token index keys pooled by the gated compressor, queries and pooled keys rotated,
    then scored and selected, against the oracle's compressor, indexer RoPE and top-k."""
    spec = next(x for x in MID if x.name == "mid_csa_f32")
    inp = _inputs(spec)
    R = 16
    kI_tok, gI_tok, k_I = _pooled_index_keys(spec, torch.float32)
    q_rot = csa.csa_rope_rows(inp["q_I"], spec.q_pos0, spec.H_I, spec.S_q, 1, R, spec.base)
    k_rot = csa.csa_rope_rows(k_I, 0, 1, spec.P, spec.m, R, spec.base)
    idx = csa.csa_index_topk(q_rot, inp["w"], k_rot, spec.q_pos0, spec.m, spec.topk)
    torch.cuda.synchronize()
    rows = list(range(spec.S_q))
    tpos = np.asarray(rows, dtype=np.int64) + spec.q_pos0
    o_kI = oracle.compress(to_np(kI_tok), to_np(gI_tok), spec.m, spec.overlap)
    assert rel_err(to_np(k_I), o_kI) <= TOL["f32"]
    sc = oracle.index_scores_rope(to_np(inp["q_I"]), to_np(inp["w"]), o_kI, tpos, spec.m, R,
                                  spec.base)
    o_idx, _ = oracle.topk(sc, tpos, spec.m, spec.topk)
    g_idx = idx.cpu().numpy()
    n_diff = 0
    for b in range(spec.B):
        n_diff += check_topk(g_idx[b], o_idx[b], sc[b], kk_rows(spec, rows))
    assert n_diff <= 0.02 * spec.B * spec.S_q


def test_indexer_key_pooling_and_rope_stagewise_bf16():
    """The same chain at the V4-Flash indexer shape (d_I = 128, rope 64, bf16), stage by
    stage so that bf16 rounding between stages cannot move a top-k boundary: pooled keys
    and both rotations against the oracle, then the indexer on the rotated tensors against
    the oracle indexer on the same tensors."""
    spec = next(x for x in MID if x.name == "mid_csa_bf16")
    inp = _inputs(spec)
    R = 64
    kI_tok, gI_tok, k_I = _pooled_index_keys(spec, torch.bfloat16)
    q_rot = csa.csa_rope_rows(inp["q_I"], spec.q_pos0, spec.H_I, spec.S_q, 1, R, spec.base)
    k_rot = csa.csa_rope_rows(k_I, 0, 1, spec.P, spec.m, R, spec.base)
    idx = csa.csa_index_topk(q_rot, inp["w"], k_rot, spec.q_pos0, spec.m, spec.topk)
    torch.cuda.synchronize()
    rows = list(range(spec.S_q))
    tpos = np.asarray(rows, dtype=np.int64) + spec.q_pos0
    assert rel_err(to_np(k_I), oracle.compress(to_np(kI_tok), to_np(gI_tok), spec.m,
                                               spec.overlap)) <= TOL["bf16"]
    q_ref = oracle.rope(to_np(inp["q_I"]), np.broadcast_to(tpos[None, :, None], q_rot.shape[:3]),
                        R, spec.base)
    k_ref = oracle.rope(to_np(k_I), np.broadcast_to((np.arange(spec.P) * spec.m)[None, :],
                                                    k_rot.shape[:2]), R, spec.base)
    assert rel_err(to_np(q_rot), q_ref) <= TOL["bf16"]
    assert rel_err(to_np(k_rot), k_ref) <= TOL["bf16"]
    sc = oracle.index_scores(to_np(q_rot), to_np(inp["w"]), to_np(k_rot), tpos, spec.m)
    o_idx, _ = oracle.topk(sc, tpos, spec.m, spec.topk)
    g_idx = idx.cpu().numpy()
    for b in range(spec.B):
        check_topk(g_idx[b], o_idx[b], sc[b], kk_rows(spec, rows))


def test_workload6_index_key_path_sampled():
    """Workload 6 at full size, in the benchmark's call sequence, checked stage by stage:
    every pooled index key and every rotated key against the oracle, then the rotated
    queries and the top-k on sampled query rows (the oracle indexer on the same rotated
    tensors).  The attention after it is the one workload 1 checks."""
    spec = cs.WORKLOADS[6][0]
    inp = _inputs(spec)
    R = spec.index_rope
    k_I = csa.csa_compress(inp["kI_tok"], inp["gI_tok"], spec.m, spec.overlap)
    q_rot = csa.csa_rope_rows(inp["q_I"], spec.q_pos0, spec.H_I, spec.S_q, 1, R, spec.base)
    k_rot = csa.csa_rope_rows(k_I, 0, 1, spec.P, spec.m, R, spec.base)
    idx = csa.csa_index_topk(q_rot, inp["w"], k_rot, spec.q_pos0, spec.m, spec.topk)
    torch.cuda.synchronize()
    assert rel_err(to_np(k_I), oracle.compress(to_np(inp["kI_tok"]), to_np(inp["gI_tok"]),
                                               spec.m, spec.overlap)) <= TOL["bf16"]
    k_ref = oracle.rope(to_np(k_I), np.broadcast_to((np.arange(spec.P) * spec.m)[None, :],
                                                    k_rot.shape[:2]), R, spec.base)
    assert rel_err(to_np(k_rot), k_ref) <= TOL["bf16"]
    rows = cs.sample_rows(spec, n_random=64)
    rows_t = torch.tensor(rows, device=DEV)
    tpos = np.asarray(rows, dtype=np.int64) + spec.q_pos0
    q_s = q_rot[:, rows_t]
    q_ref = oracle.rope(to_np(inp["q_I"][:, rows_t]),
                        np.broadcast_to(tpos[None, :, None], q_s.shape[:3]), R, spec.base)
    assert rel_err(to_np(q_s), q_ref) <= TOL["bf16"]
    sc = oracle.index_scores(to_np(q_s), to_np(inp["w"][:, rows_t]), to_np(k_rot), tpos, spec.m)
    o_idx, _ = oracle.topk(sc, tpos, spec.m, spec.topk)
    g_idx = idx[:, rows_t].cpu().numpy()
    for b in range(spec.B):
        check_topk(g_idx[b], o_idx[b], sc[b], kk_rows(spec, rows))


# ----------------------------------------------------------------------------- error path
@pytest.mark.parametrize("name", ["mid_csa_bf16", "mid_decode_bf16"])
def test_bounded_wait_gives_up_and_reports(name):
    """The tensor-core attention's error path, without any fault or hang: with the test
    hook on, its loader publishes nothing, every bounded wait on it runs out after a short
    bound, the kernel frees its tensor memory and returns, and csa_device_status() reports
    bit 0.  The context stays usable: with the hook off the same call matches the oracle
    and reports nothing."""
    spec = next(x for x in MID if x.name == name)
    inp = _inputs(spec)
    rows = list(range(spec.S_q))
    ora_pool = oracle_pool(spec, inp)
    pool_in = _pool_input(spec, inp, ora_pool)
    _, o_idx, _ = oracle_index(spec, inp, rows)
    idx_in = torch.from_numpy(o_idx).to(DEV)
    assert csa.device_status() == 0
    try:
        csa.debug_withhold_attention_loads(True)
        GpuLayer(spec, inp).attend(pool_in, idx_in)
        torch.cuda.synchronize()
        assert csa.device_status() & 1
    finally:
        csa.debug_withhold_attention_loads(False)
    out = GpuLayer(spec, inp).attend(pool_in, idx_in)
    torch.cuda.synchronize()
    assert csa.device_status() == 0
    ref = oracle_attend(spec, inp, rows, to_np(pool_in), o_idx)
    assert rel_err(to_np(out), ref) <= TOL[spec.dtype]
