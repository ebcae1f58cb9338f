"""Helpers for GPU-vs-oracle parity: run a layer through the C ABI, run the oracle on the
same seeded inputs (or a sampled subset of query rows), and compare.

Tolerances (written here, used by every parity test):
  * floating outputs: max|gpu - ref| / max|ref| <= 1e-4 (fp32 layers) or 2e-2 (bf16
    layers, fp32 accumulation);
  * top-k: the kept sets have the same size min(k, n_vis) and every entry in their
    symmetric difference has an oracle score within 1e-3 relative of the oracle's k-th
    kept score (so exact ties pass and nothing else may differ).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import sparse_attention_14_b200 as csa

TOL = {"f32": 1e-4, "bf16": 2e-2}
TIE_BAND = 1e-3


def rel_err(gpu, ref) -> float:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.max(np.abs(ref))
    if den == 0:
        return float(np.max(np.abs(gpu)))
    return float(np.max(np.abs(gpu - ref)) / den)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64) if t.dtype == torch.bfloat16 \
        else t.detach().cpu().numpy()


def check_topk(gpu_idx, ora_idx, ora_scores_full, kk_per_row):
    """gpu_idx, ora_idx [n,k] int; ora_scores_full [n,P] fp64 oracle scores;
    kk_per_row [n].  Returns the number of rows whose sets differ (inside the tie band).
    Raises AssertionError for any difference outside the band."""
    n_diff = 0
    for r in range(gpu_idx.shape[0]):
        kk = int(kk_per_row[r])
        g = gpu_idx[r]
        o = ora_idx[r]
        assert (g[kk:] == -1).all(), "row %d: slots past min(k, n_vis) must be -1" % r
        assert (g[:kk] >= 0).all(), "row %d: missing entries" % r
        gs, os_ = set(g[:kk].tolist()), set(o[:kk].tolist())
        assert len(gs) == kk, "row %d: duplicate entries" % r
        if gs == os_:
            continue
        n_diff += 1
        kth = ora_scores_full[r, o[kk - 1]]
        for j in gs ^ os_:
            s = ora_scores_full[r, j]
            assert abs(s - kth) <= TIE_BAND * abs(kth), \
                "row %d: entry %d (score %.9g) differs outside the tie band of %.9g" % (r, j, s, kth)
    return n_diff


class GpuLayer:
    """Runs one layer of a LayerSpec through the library on CUDA tensors."""

    def __init__(self, spec, inp):
        self.spec = spec
        self.inp = inp

    def compress(self):
        s, i = self.spec, self.inp
        return csa.csa_compress(i["kv"], i["gate"], s.m, s.overlap)

    def index(self, want_scores=True):
        s, i = self.spec, self.inp
        return csa.csa_index_topk(i["q_I"], i["w"], i["k_I"], s.q_pos0, s.m, s.topk,
                                  want_scores=want_scores)

    def attend(self, pool, idx):
        s, i = self.spec, self.inp
        if s.kind == "csa":
            return csa.csa_attend(i["q"], i["kv"], s.kv_pos0, pool, idx, i["sink"], s.q_pos0, s.R,
                                  s.base, s.W, s.m, s.scale)
        return csa.hca_attend(i["q"], i["kv"], s.kv_pos0, pool if s.kind == "hca" else None,
                              i["sink"], s.q_pos0, s.R, s.base, s.W, s.m, s.scale)


def oracle_pool(spec, inp):
    if spec.decode:
        return to_np(inp["pool"])
    if spec.kind == "sliding":
        return None
    return oracle.compress(to_np(inp["kv"]), to_np(inp["gate"]), spec.m, spec.overlap)


def oracle_index(spec, inp, rows):
    tpos = np.asarray(rows, dtype=np.int64) + spec.q_pos0
    q_I = to_np(inp["q_I"][:, rows])
    w = to_np(inp["w"][:, rows])
    sc = oracle.index_scores(q_I, w, to_np(inp["k_I"]), tpos, spec.m)
    idx, sel = oracle.topk(sc, tpos, spec.m, spec.topk)
    return sc, idx, sel


def oracle_attend(spec, inp, rows, pool, idx):
    tpos = np.asarray(rows, dtype=np.int64) + spec.q_pos0
    mode = "csa" if spec.kind == "csa" else "hca"
    return oracle.attend(to_np(inp["q"][:, rows]), tpos, to_np(inp["kv"]), spec.kv_pos0, pool,
                         spec.m, idx, to_np(inp["sink"]), spec.R, spec.base, spec.W, spec.scale,
                         mode)


def kk_rows(spec, rows):
    return [min(spec.topk, oracle.n_visible(r + spec.q_pos0, spec.m, spec.P)) for r in rows]
