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

import csa_synth as cs
import oracle
import sparse_attention_14_b200 as csa

TOL = {"f32": 1e-4, "bf16": 2e-2}
TIE_BAND = 1e-3


def rel_err(gpu, ref) -> float:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    if ref.size == 0:
        return 0.0
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

    def append(self):
        """Decode-time cache update: the new tokens into the main compressor state (closed
        entries into the pool) and their index keys into the indexer's (into k_I)."""
        s, i = self.spec, self.inp
        csa.csa_compress_append(cs.kv_new(s, i), i["gate_new"], i["state"], s.q_pos0, s.m,
                                s.overlap, pool=i["pool"])
        if s.kind == "csa":
            csa.csa_compress_append(i["kI_new"], i["gI_new"], i["state_I"], s.q_pos0, s.m,
                                    s.overlap, pool=i["k_I"])

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


def oracle_cache_update(spec, inp):
    """The oracle's stateful compressors, rebuilt from the step's input states, fed the
    new tokens: [(cache key, first entry j0, entries [B, n, D]), ...] for the main
    compressor ("pool") and, for CSA, the indexer's key compressor ("k_I")."""
    comps = [("state", cs.kv_new(spec, inp), "gate_new", "pool")]
    if spec.kind == "csa":
        comps.append(("state_I", inp["kI_new"], "gI_new", "k_I"))
    out = []
    for st_key, new, g_key, cache in comps:
        kh, gh, s0 = cs.ring_history(inp[st_key], spec.q_pos0, spec.m, spec.overlap)
        st = oracle.CompressorState.resume(to_np(kh), to_np(gh), s0, spec.m, spec.overlap)
        out.append((cache, spec.q_pos0 // spec.m, st.append(to_np(new), to_np(inp[g_key]))))
    return out


def gpu_cache_update_checked(spec, inp):
    """Run the step's cache update on the GPU (csa_compress_append on the main and the
    indexer state) and check it: the closed entries against the oracle, every other cache
    row near them unchanged, the new rows stored in their state slots bit for bit."""
    expected = oracle_cache_update(spec, inp)
    L = spec.ring
    keep = {}
    for cache, j0, ent in expected:
        lo, hi = max(0, j0 - 3), min(inp[cache].shape[1], j0 + ent.shape[1] + 3)
        keep[cache] = (lo, hi, inp[cache][:, lo:hi].clone())
    GpuLayer(spec, inp).append()
    torch.cuda.synchronize()
    for cache, j0, ent in expected:
        n = ent.shape[1]
        assert n == (spec.q_pos0 + spec.S_q) // spec.m - spec.q_pos0 // spec.m
        if n:
            assert rel_err(to_np(inp[cache][:, j0:j0 + n]), ent) <= TOL[spec.dtype], cache
        lo, hi, before = keep[cache]
        after = inp[cache][:, lo:hi]
        for r in range(hi - lo):
            if not (j0 <= lo + r < j0 + n):
                assert torch.equal(after[:, r], before[:, r]), (cache, lo + r)
    news = [("state", cs.kv_new(spec, inp), inp["gate_new"])]
    if spec.kind == "csa":
        news.append(("state_I", inp["kI_new"], inp["gI_new"]))
    for st_key, kv_rows, g_rows in news:
        for i in range(max(0, spec.S_q - L), spec.S_q):
            slot = (spec.q_pos0 + i) % L
            assert torch.equal(inp[st_key][:, 0, slot], kv_rows[:, i]), (st_key, i)
            assert torch.equal(inp[st_key][:, 1, slot], g_rows[:, i]), (st_key, i)


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
