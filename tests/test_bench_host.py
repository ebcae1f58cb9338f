"""Host logic of bench.py, on the CPU: the per-stage algorithmic work counts that the
roofline divides by, the oracle row sampler and the workload part of the JSON config.

The key counts behind the attention FLOPs are checked against an independent count:
the window rows by brute force over every raw kv row, the entries from the oracle's own
top-k selection (CSA) or visibility count (HCA) on seeded inputs.
"""
from __future__ import annotations

import dataclasses
import json
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import csa_synth as cs  # noqa: E402
import oracle  # noqa: E402


def _brute_window_rows(spec, t):
    # every raw kv row that is causal (position <= t) and inside the window (t - pos < W)
    n = 0
    for r in range(spec.S_kv):
        p = spec.kv_pos0 + r
        if p <= t and t - p < spec.W:
            n += 1
    return n


def _oracle_key_counts(spec):
    """Per (batch, query) number of keys attention reads, from the oracle's selection."""
    inp = cs.make_inputs(spec, "cpu")
    tpos = np.arange(spec.S_q, dtype=np.int64) + spec.q_pos0
    win = np.array([_brute_window_rows(spec, int(t)) for t in tpos])
    if spec.kind == "csa":
        scores = oracle.index_scores(inp["q_I"], inp["w"], inp["k_I"], tpos, spec.m)
        idx, _ = oracle.topk(scores, tpos, spec.m, spec.topk)
        ent = (idx >= 0).sum(axis=-1)                      # [B, n]
        vis = (~np.isnan(scores)).sum(axis=-1)             # [B, n] visible entries
    elif spec.kind == "hca":
        vis = np.array([[oracle.n_visible(int(t), spec.m, spec.P) for t in tpos]] * spec.B)
        ent = vis
    else:
        vis = ent = np.zeros((spec.B, spec.S_q), dtype=np.int64)
    return win[None, :] + ent, vis


def _tiny(kind, **kw):
    base = dict(name="tiny_" + kind, dtype="f32", B=2, S_q=96, S_kv=96, q_pos0=0, kv_pos0=0,
                H=4, D=32, R=8, base=10000.0, W=16, m=4 if kind == "csa" else 16, P=0,
                kind=kind, workload=0)
    if kind == "csa":
        base.update(H_I=2, d_I=16, topk=8)
    base.update(kw)
    if base["P"] == 0 and kind != "sliding":
        base["P"] = (base["kv_pos0"] + base["S_kv"]) // base["m"]
    return cs.LayerSpec(**base)


SPECS = [
    cs.TINY_CSA,
    _tiny("csa"),
    _tiny("hca"),
    _tiny("sliding"),
    # decode-style: three queries at the end of a long context, a resident pool
    _tiny("csa", S_q=3, S_kv=18, q_pos0=1021, kv_pos0=1006, P=256, decode=True),
    _tiny("hca", S_q=1, S_kv=16, q_pos0=2047, kv_pos0=2032, P=128, decode=True),
]


@pytest.mark.parametrize("spec", SPECS, ids=[s.name + ("_dec" if s.decode else "") for s in SPECS])
def test_attend_and_index_flops_match_oracle_selection(spec):
    keys, vis = _oracle_key_counts(spec)
    w = bench.algorithmic_work(spec)
    assert w["attend_flops"] == 4 * spec.H * spec.D * int(keys.sum())
    if spec.kind == "csa":
        assert w["index_flops"] == 2 * spec.H_I * spec.d_I * int(vis.sum())
    else:
        assert w["index_flops"] == 0
        assert "index_bytes" not in w


@pytest.mark.parametrize("spec", SPECS, ids=[s.name + ("_dec" if s.decode else "") for s in SPECS])
def test_byte_counts(spec):
    e = 4 if spec.dtype == "f32" else 2
    w = bench.algorithmic_work(spec)
    # compressor: reads kv and gate, writes the pool; absent in decode and sliding-only
    if spec.decode or spec.kind == "sliding":
        assert "compress_bytes" not in w
    else:
        assert w["compress_bytes"] == spec.B * (2 * spec.S_kv + spec.P) * spec.D * e
    # attention reads q and writes out once, and each distinct kv/pool row at least once
    qo = 2 * spec.B * spec.S_q * spec.H * spec.D * e
    assert qo < w["attend_bytes"] <= qo + spec.B * (spec.S_kv + spec.P) * spec.D * e
    if spec.kind == "csa":
        keys, _ = _oracle_key_counts(spec)
        inp = cs.make_inputs(spec, "cpu")
        tpos = np.arange(spec.S_q, dtype=np.int64) + spec.q_pos0
        idx, _ = oracle.topk(oracle.index_scores(inp["q_I"], inp["w"], inp["k_I"], tpos, spec.m),
                             tpos, spec.m, spec.topk)
        distinct = max(len(set(idx[b][idx[b] >= 0].tolist())) for b in range(spec.B))
        ent_rows = (w["attend_bytes"] // (spec.B * e) - 2 * spec.S_q * spec.H * spec.D) // spec.D \
            - min(spec.S_kv, spec.S_q + spec.W - 1)
        # the model's entry-row count bounds what the oracle actually selected
        assert distinct <= ent_rows <= spec.P


def test_full_size_counts_closed_form():
    # CSA prefill S=8192: every query reads min(t+1, 128) window rows and min(512, (t+1)//4)
    # entries; summing those closed forms by arithmetic series must match the model
    s = cs.CSA_PREFILL
    S, W, k, m = s.S_q, s.W, s.topk, s.m
    win = sum(range(1, W + 1)) + (S - W) * W
    t_full = k * m - 1                     # first t with (t+1)//4 >= 512
    ent = sum((t + 1) // m for t in range(t_full)) + (S - t_full) * k
    assert bench.algorithmic_work(s)["attend_flops"] == 4 * s.H * s.D * (win + ent)
    # CSA decode: one query, 128 window rows and 512 entries per batch element
    d = cs.CSA_DECODE
    assert bench.algorithmic_work(d)["attend_flops"] == 4 * d.B * d.H * d.D * (128 + 512)
    assert bench.algorithmic_work(d)["index_flops"] == 2 * d.B * d.H_I * d.d_I * d.P


@pytest.mark.parametrize("S,n", [(1, 1), (1, 8), (3, 8), (100, 7), (8192, 64), (131072, 16)])
def test_oracle_rows_sampler(S, n):
    spec = dataclasses.replace(cs.TINY_CSA, S_q=S)
    rows = bench.oracle_rows(spec, n)
    assert rows == sorted(set(rows))
    assert len(rows) == min(n, S)
    assert all(0 <= r < S for r in rows)
    if S >= 2 * n:
        # spread over the whole sequence: the sample reaches both the short-context head
        # and the long-context tail of the causal mix
        assert rows[0] < S // n and rows[-1] >= S - S // n


@pytest.mark.parametrize("w", sorted(cs.WORKLOADS))
def test_workload_config_is_plain_json(w):
    specs = cs.WORKLOADS[w]
    cfg = bench.workload_config(w, specs)
    assert json.loads(json.dumps(cfg)) == cfg
    assert cfg["workload"] == bench.workload_name(w, specs)
    assert cfg["layers"] == [s.kind for s in specs]
    assert len(cfg["m"]) == len(cfg["P"]) == len(specs)
    # no model keys: the config names a workload, not a checkpoint
    assert "model" not in cfg


def test_index_key_path_work_and_oracle_sample():
    """Workload 6 (prefill with the indexer's key path): the extra stages' bytes, the stage
    order, and the sampled oracle run that pools the index keys and rotates both sides."""
    s = cs.WORKLOADS[6][0]
    w = bench.algorithmic_work(s)
    assert w["compress_I_bytes"] == (2 * 8192 + 2048) * 128 * 2
    assert w["rope_I_bytes"] == 2 * (8192 * 64 + 2048) * 128 * 2
    base = bench.algorithmic_work(cs.CSA_PREFILL)
    assert {k: v for k, v in w.items() if k not in ("compress_I_bytes", "rope_I_bytes")} == base
    assert bench.LayerRunner.stages(type("R", (), {"spec": s})()) == \
        ["compress", "compress_I", "rope_I", "index", "attend"]
    small = dataclasses.replace(s, S_q=96, S_kv=96, P=24, topk=8, H=4, D=64, R=16, H_I=4, d_I=32,
                                index_rope=16, workload=72)
    assert bench.oracle_sample_run(small, [0, 50, 95]) > 0
