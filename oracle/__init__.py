"""fp64 CPU oracle for the DeepSeek-V4 hybrid compressed attention layer.

TEST INFRASTRUCTURE ONLY: the CPU tests, the smoke check and the benchmark's CPU
baseline call it; the product path never does.  The arithmetic lives in plain C
(csa_oracle.c, compiled with gcc into liboracle.so); this module only converts arrays to
float64 and calls it.  It shares no code with the CUDA library.

Function map (each C function's comment cites the page passage it follows):
  compress      -> orc_compress       gated pooling, CSA/HCA windows
  CompressorState.append -> orc_compress_step   stateful (decode) compressor
  n_visible     -> orc_n_visible      causal visibility of compressed entries
  index_scores  -> orc_index_scores   Lightning Indexer score
  index_scores_rope -> orc_rope_rows + orc_index_scores   the same with indexer RoPE
  topk          -> orc_topk           top-k with -1 marker
  attend        -> orc_attend         sink MQA over window + entries, RoPE, de-rotation
  attend_keys   -> orc_attend_keys    the same for one query over explicit keys
  rope          -> orc_rope_rows      interleaved-pair partial RoPE
  grouped_out_proj -> numpy matmuls   grouped low-rank output projection (after attention)
  kv_gate_proj  -> numpy matmuls      kv_proj + kv_norm and gate_proj (before the compressor)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_lp = ctypes.POINTER(ctypes.c_int64)
_ip = ctypes.POINTER(ctypes.c_int32)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile csa_oracle.c with gcc (-O2, OpenMP, IEEE semantics: no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path: str):
    lib = ctypes.CDLL(path)
    lib.orc_rope_rows.argtypes = [_dp, _dp, _i64, _i64, _i64, ctypes.c_double]
    lib.orc_compress.argtypes = [_dp, _dp, _dp, _i64, _i64, _i64, _i64, ctypes.c_int]
    lib.orc_compress_step.argtypes = [_dp, _dp, _dp, _dp, _lp, _lp, _dp, _dp, _i64, _i64, _i64,
                                      _i64, ctypes.c_int, _dp, _i64, _lp]
    lib.orc_n_visible.argtypes = [_i64, _i64, _i64]
    lib.orc_n_visible.restype = _i64
    lib.orc_index_scores.argtypes = [_dp, _dp, _dp, _lp, _i64, _i64, _i64, _i64, _i64, _i64, _dp]
    lib.orc_topk.argtypes = [_dp, _lp, _i64, _i64, _i64, _i64, _i64, _ip, _dp]
    lib.orc_attend_keys.argtypes = [_dp, ctypes.c_double, _dp, _dp, _i64, _dp, _i64, _i64, _i64,
                                    ctypes.c_double, ctypes.c_double, _dp]
    lib.orc_attend.argtypes = [_dp, _lp, _i64, _dp, _i64, _i64, _dp, _i64, _i64, _ip, _i64,
                               ctypes.c_int, _dp, _i64, _i64, _i64, _i64, ctypes.c_double, _i64,
                               ctypes.c_double, _dp]
    return lib


class using:
    """Run oracle calls against another build of csa_oracle.c (the mutation tests build
    deliberately broken copies to show that the pins catch them)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        _load()
        self._saved = _lib
        _lib = _bind(self.path)
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self._saved
        return False


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = _bind(_LIB)
            _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor -> numpy without importing torch here
        x = x.detach().float().cpu().numpy() if str(x.dtype) == "torch.bfloat16" else x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError("oracle %s failed with code %d" % (what, rc))


def rope(x, pos, R: int, base: float) -> np.ndarray:
    """Rotate rows x[..., D] at positions pos[...] (one per row)."""
    a = _f64(x).copy()
    D = a.shape[-1]
    rows = a.reshape(-1, D)
    p = np.ascontiguousarray(np.broadcast_to(np.asarray(pos, dtype=np.float64),
                                             a.shape[:-1]).reshape(-1))
    _check(_load().orc_rope_rows(_ptr(rows, _dp), _ptr(p, _dp), rows.shape[0], D, R, base), "rope")
    return rows.reshape(a.shape)


def compress(kv, gate, m: int, overlap: int) -> np.ndarray:
    """kv, gate [B,S,D] -> pool [B, S//m, D]."""
    kv, gate = _f64(kv), _f64(gate)
    B, S, D = kv.shape
    pool = np.zeros((B, S // m, D), dtype=np.float64)
    _check(_load().orc_compress(_ptr(kv, _dp), _ptr(gate, _dp), _ptr(pool, _dp), B, S, D, m,
                                int(overlap)), "compress")
    return pool


class CompressorState:
    """Stateful compressor of B sequences for decode (orc_compress_step): a buffer of the
    open window, the last closed block (overlap) and a token counter, all fp64."""

    def __init__(self, B: int, D: int, m: int, overlap: int):
        self.B, self.D, self.m, self.overlap = B, D, m, int(bool(overlap))
        self.buf_kv = np.zeros((B, m, D))
        self.buf_gate = np.zeros((B, m, D))
        self.ovl_kv = np.zeros((B, m, D))
        self.ovl_gate = np.zeros((B, m, D))
        self.counter = np.zeros(B, dtype=np.int64)
        self.n_ovl = np.zeros(B, dtype=np.int64)

    @classmethod
    def resume(cls, kv_hist, gate_hist, s0: int, m: int, overlap: int) -> "CompressorState":
        """The state after the rows of positions [s0, s0+n) (kv_hist, gate_hist [B,n,D]),
        rebuilt by replaying them from s0, a window start (s0 % m == 0) from which the
        buffer and, with overlap, the last closed block are covered.  Entries that close
        during the replay are dropped (the first one lacks its own overlap block)."""
        if s0 % m:
            raise ValueError("CompressorState.resume: s0 must be a multiple of m")
        kv = _f64(kv_hist)
        st = cls(kv.shape[0], kv.shape[2], m, overlap)
        st.counter[:] = s0
        st.append(kv, gate_hist)
        return st

    def append(self, kv_new, gate_new) -> np.ndarray:
        """kv_new, gate_new [B,n,D] (the next n tokens) -> the entries whose windows close
        among them, [B, n_closed, D] in closing order (n_closed may be 0)."""
        kv, gate = _f64(kv_new), _f64(gate_new)
        B, n, D = kv.shape
        if B != self.B or D != self.D or gate.shape != kv.shape:
            raise ValueError("CompressorState.append: shape mismatch")
        max_out = n // self.m + 1
        out = np.zeros((B, max_out, D))
        n_out = np.zeros(B, dtype=np.int64)
        _check(_load().orc_compress_step(_ptr(self.buf_kv, _dp), _ptr(self.buf_gate, _dp),
                                         _ptr(self.ovl_kv, _dp), _ptr(self.ovl_gate, _dp),
                                         _ptr(self.counter, _lp), _ptr(self.n_ovl, _lp),
                                         _ptr(kv, _dp), _ptr(gate, _dp), n, B, D, self.m,
                                         self.overlap, _ptr(out, _dp), max_out,
                                         _ptr(n_out, _lp)), "compress_step")
        if B and not np.all(n_out == n_out[0]):
            raise ValueError("CompressorState.append: sequences closed different counts")
        return out[:, : int(n_out[0]) if B else 0]


def n_visible(t: int, m: int, P: int) -> int:
    return int(_load().orc_n_visible(t, m, P))


def index_scores(q_I, w, k_I, tpos, m: int) -> np.ndarray:
    """q_I [B,n,H_I,d_I], w [B,n,H_I], k_I [B,P,d_I], tpos [n] -> scores [B,n,P] (NaN = not visible)."""
    q_I, w, k_I = _f64(q_I), _f64(w), _f64(k_I)
    B, n, HI, dI = q_I.shape
    P = k_I.shape[1]
    tp = np.ascontiguousarray(np.asarray(tpos, dtype=np.int64))
    out = np.zeros((B, n, P), dtype=np.float64)
    _check(_load().orc_index_scores(_ptr(q_I, _dp), _ptr(w, _dp), _ptr(k_I, _dp), _ptr(tp, _lp),
                                    B, n, P, HI, dI, m, _ptr(out, _dp)), "index_scores")
    return out


def index_scores_rope(q_I, w, k_I, tpos, m: int, R: int, base: float) -> np.ndarray:
    """The Lightning Indexer score with the indexer's own rotary embedding: every head of
    q_I[t] is rotated at t and every pooled key k_I[j] at j*m (interleaved pairs on the
    last R channels, orc_rope_rows), then scored as index_scores does."""
    q = _f64(q_I)
    k = _f64(k_I)
    B, n, HI, dI = q.shape
    P = k.shape[1]
    tp = np.asarray(tpos, dtype=np.float64)
    q_rot = rope(q, np.broadcast_to(tp[None, :, None], (B, n, HI)), R, base)
    k_rot = rope(k, np.broadcast_to((np.arange(P, dtype=np.float64) * m)[None, :], (B, P)), R, base)
    return index_scores(q_rot, w, k_rot, tpos, m)


def topk(scores, tpos, m: int, k: int):
    """scores [B,n,P] -> (idx int32 [B,n,k] with -1 padding, selected scores [B,n,k])."""
    sc = _f64(scores)
    B, n, P = sc.shape
    tp = np.ascontiguousarray(np.asarray(tpos, dtype=np.int64))
    idx = np.zeros((B, n, k), dtype=np.int32)
    sel = np.zeros((B, n, k), dtype=np.float64)
    _check(_load().orc_topk(_ptr(sc, _dp), _ptr(tp, _lp), B, n, P, m, k, _ptr(idx, _ip),
                            _ptr(sel, _dp)), "topk")
    return idx, sel


def attend_keys(q, tq: float, keys, kpos, sink, R: int, base: float, scale: float) -> np.ndarray:
    """One query q [H,D] at tq over explicit un-rotated keys [n,D] at kpos [n]."""
    q, keys, sink = _f64(q), _f64(keys), _f64(sink)
    H, D = q.shape
    kp = np.ascontiguousarray(np.asarray(kpos, dtype=np.float64))
    out = np.zeros((H, D), dtype=np.float64)
    _check(_load().orc_attend_keys(_ptr(q, _dp), float(tq), _ptr(keys, _dp), _ptr(kp, _dp),
                                   keys.shape[0], _ptr(sink, _dp), H, D, R, base, scale,
                                   _ptr(out, _dp)), "attend_keys")
    return out


def attend(q, tpos, kv, kv_pos0: int, pool, m: int, idx, sink, R: int, base: float, W: int,
           scale: float, mode: str) -> np.ndarray:
    """q [B,n,H,D] at positions tpos [n]; kv [B,S_kv,D] from kv_pos0; pool [B,P,D] or None;
    idx [B,n,k] int32 (mode "csa") or None (mode "hca" / "sliding"); sink [H]."""
    q, kv, sink = _f64(q), _f64(kv), _f64(sink)
    B, n, H, D = q.shape
    S_kv = kv.shape[1]
    if pool is None:
        pool = np.zeros((B, 0, D), dtype=np.float64)
    pool = _f64(pool)
    P = pool.shape[1]
    tp = np.ascontiguousarray(np.asarray(tpos, dtype=np.int64))
    if mode == "csa":
        idx_a = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
        k = idx_a.shape[-1]
        mode_i = 0
    else:
        idx_a = np.zeros((1,), dtype=np.int32)
        k = 0
        mode_i = 1
    out = np.zeros((B, n, H, D), dtype=np.float64)
    _check(_load().orc_attend(_ptr(q, _dp), _ptr(tp, _lp), n, _ptr(kv, _dp), S_kv, kv_pos0,
                              _ptr(pool, _dp), P, m, _ptr(idx_a, _ip), k, mode_i,
                              _ptr(sink, _dp), B, H, D, R, base, W, scale, _ptr(out, _dp)),
           "attend")
    return out


def grouped_out_proj(o, w_a, w_b, return_groups: bool = False):
    """Grouped low-rank output projection after the attention (HF docs model_doc/
    deepseek_v4, section 2.3 "Grouped Output Projection": o_groups head groups ->
    o_lora_rank per group -> hidden_size, computed by DeepseekV4GroupedLinear (o_a_proj)
    and then o_b_proj; HF PR #45616: the grouped linear's forward is a per-group batched
    matmul, and the output's rope slice is un-rotated before this projection).

    o    [B,S,H,D]          de-rotated attention output
    w_a  [G, r, (H/G)*D]    o_a_proj: group g projects heads [g*H/G, (g+1)*H/G), flattened
                            head-major, to r features
    w_b  [hidden, G*r]      o_b_proj over the G groups' features, group-major
    -> y [B,S,hidden] (and z [B,S,G,r] when return_groups).
    Plain fp64 matmuls per group, in the order the definition states."""
    o, w_a, w_b = _f64(o), _f64(w_a), _f64(w_b)
    B, S, H, D = o.shape
    G, r, per = w_a.shape
    if H % G or per != (H // G) * D or w_b.shape[1] != G * r:
        raise ValueError("grouped_out_proj: shapes do not match")
    x = o.reshape(B, S, G, per)
    z = np.zeros((B, S, G, r))
    for g in range(G):
        z[:, :, g] = x[:, :, g] @ w_a[g].T
    y = z.reshape(B, S, G * r) @ w_b.T
    return (y, z) if return_groups else y


def kv_gate_proj(x, w_kv, w_gate, kv_norm_w, eps: float):
    """The compressor's input projections (TransformerLens deepseek_v4 bridge: the
    compressor's kv_proj, gate_proj and kv_norm submodules, an RMSNormalizationBridge).
    Reading taken (the pages name the modules, not their order): per token the K=V row is
    kv_proj of the token, RMS-normalised over its D channels and scaled by the norm's
    weight; the gate logits are gate_proj of the token.

    x [..., hidden]; w_kv, w_gate [D, hidden]; kv_norm_w [D]
    -> kv [..., D] = u / sqrt(mean(u^2) + eps) * kv_norm_w with u = x . w_kv^T,
       gate [..., D] = x . w_gate^T.
    Plain fp64 matmuls and the norm in the order the definition states."""
    x, w_kv, w_gate, g = _f64(x), _f64(w_kv), _f64(w_gate), _f64(kv_norm_w)
    if w_kv.shape != w_gate.shape or w_kv.shape[1] != x.shape[-1] or g.shape != (w_kv.shape[0],):
        raise ValueError("kv_gate_proj: shapes do not match")
    u = x @ w_kv.T
    kv = u / np.sqrt((u * u).mean(axis=-1, keepdims=True) + eps) * g
    gate = x @ w_gate.T
    return kv, gate
