"""Seeded synthetic inputs and layer shapes for the DeepSeek-V4 hybrid attention layer.

This module is shared by the CUDA path's tests/bench and by the CPU oracle's tests.
It holds sizes and random-number recipes only: no step of the method's arithmetic
(pooling, scoring, selection, RoPE, softmax) lives here.

Workload shapes follow the V4-Flash layer described on the pages:
  * window 128, CSA ratio m=4 (overlapping windows), HCA ratio m'=128
    (optimum-intel issue #1748, "What V4-Flash adds vs V3");
  * head_dim 512 (HF transformers PR #45616, "Config inherits DeepseekV3Config");
  * a single shared K=V head and a per-head sink (HF docs model_doc/deepseek_v4,
    "Hybrid attention (section 2.3)").

Value recipe (the same for every workload): q, kv, gate logits, q_I, k_I ~ N(0,1);
indexer head weights w ~ N(0,1)/sqrt(H_I); sink logits ~ N(0,1) in fp32; every kv row
(and every directly generated pool row) RMS-normalised, x / sqrt(mean(x^2) + 1e-6),
in fp64 before rounding to the storage dtype.

Decode step with the cache update (workload 5): the main compressor's state is the ring of
the last (1+overlap)*m raw rows before the new token, in the layout csa_compress_append
documents (row of position p in slot p mod L); its kv rows are the window rows of those
positions (the same tokens), its gates N(0,1).  The indexer's per-token keys and gates
(state_I, kI_new, gI_new) and the new token's gate are N(0,1).  The new token's kv row is
the last row of the window.

Seeds: tensor seed = 1000*workload + 100*layer + tensor_id, tensor ids in the order
q, kv, gate, q_I, k_I, w, sink, pool, gate_new, state, state_I, kI_new, gI_new, kI_tok,
gI_tok.

Prefill with the indexer's key path (workload 6): instead of pooled k_I, per-token index
keys kI_tok (RMS-normalised N(0,1) rows, as the indexer's kv_norm leaves them) and their
gate logits gI_tok (N(0,1)), both [B,S,d_I].
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import torch

TENSOR_IDS = {"q": 0, "kv": 1, "gate": 2, "q_I": 3, "k_I": 4, "w": 5, "sink": 6, "pool": 7,
              "gate_new": 8, "state": 9, "state_I": 10, "kI_new": 11, "gI_new": 12,
              "kI_tok": 13, "gI_tok": 14, "x": 15, "proj": 16}
RMS_EPS = 1e-6


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    """Shape of one attention layer call.

    kind: "csa" (compressed sparse: indexer + top-k), "hca" (heavily compressed: every
    visible entry) or "sliding" (window only, no pool).
    Query i sits at absolute position q_pos0 + i; raw kv row r at kv_pos0 + r.
    decode=True means the pool and k_I are a resident cache (no compressor run).
    cache_update=True (decode only) adds the compressor cache update to the step: the S_q
    new tokens (the last S_q window rows, at q_pos0..) go through the main compressor's
    state and, with their per-token index keys, through the indexer's key compressor;
    the entries that close are written into the pool and k_I before they are read.
    pool_index_keys=True (prefill CSA) pools k_I in the step from per-token index keys
    by the same gated compressor; index_rope > 0 rotates that many trailing channels of
    every indexer query head (at t) and pooled key (at j*m) before scoring.
    proj=True (prefill) adds the projections around the layer to the step: the raw K=V
    rows and gate logits come from the token states x [B,S,hidden] by the compressor's
    kv_proj + kv_norm and gate_proj, and the attention output goes through the grouped
    low-rank output projection to y [B,S,hidden].
    """

    name: str
    dtype: str  # "f32" or "bf16"
    B: int
    S_q: int
    S_kv: int
    q_pos0: int
    kv_pos0: int
    H: int
    D: int
    R: int
    base: float
    W: int
    m: int
    P: int
    kind: str
    H_I: int = 0
    d_I: int = 0
    topk: int = 0
    decode: bool = False
    cache_update: bool = False
    pool_index_keys: bool = False
    index_rope: int = 0
    proj: bool = False
    workload: int = 0
    layer: int = 0

    @property
    def overlap(self) -> int:
        return 1 if self.kind == "csa" else 0

    @property
    def ring(self) -> int:
        """Rows a compressor state keeps: (1+overlap)*m."""
        return (1 + self.overlap) * self.m

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def seed(self, tensor: str) -> int:
        return 1000 * self.workload + 100 * self.layer + TENSOR_IDS[tensor]


def prefill(name, dtype, S, H, D, R, base, W, m, kind, H_I=0, d_I=0, topk=0, B=1,
            workload=0, layer=0) -> LayerSpec:
    P = 0 if kind == "sliding" else S // m
    return LayerSpec(name=name, dtype=dtype, B=B, S_q=S, S_kv=S, q_pos0=0, kv_pos0=0,
                     H=H, D=D, R=R, base=base, W=W, m=m, P=P, kind=kind, H_I=H_I,
                     d_I=d_I, topk=topk, workload=workload, layer=layer)


# The five workloads.  Bases: one RoPE base per layer, used for q, window keys, entries
# and the output de-rotation; compressed layers use the slower 160000 base and the
# sliding-only layer the main 10000 base (HF PR #45616, note on compress_rope_parameters:
# compressed layers swap in their own rope_theta; mlx-lm PR #1797: two rotation speeds,
# one per kind of layer).
TINY_CSA = prefill("tiny_csa_f32", "f32", S=256, H=8, D=64, R=16, base=10000.0, W=32,
                   m=4, kind="csa", H_I=4, d_I=32, topk=16, workload=0)
CSA_PREFILL = prefill("csa_prefill_s8192", "bf16", S=8192, H=64, D=512, R=64,
                      base=160000.0, W=128, m=4, kind="csa", H_I=64, d_I=128, topk=512,
                      workload=1)
HCA_PREFILL = prefill("hca_prefill_s65536", "bf16", S=65536, H=64, D=512, R=64,
                      base=160000.0, W=128, m=128, kind="hca", workload=2)
CSA_DECODE = LayerSpec(name="csa_decode_b64_ctx65536", dtype="bf16", B=64, S_q=1, S_kv=128,
                       q_pos0=65535, kv_pos0=65408, H=64, D=512, R=64, base=160000.0,
                       W=128, m=4, P=16384, kind="csa", H_I=64, d_I=128, topk=512,
                       decode=True, workload=3)


CSA_PREFILL_INDEX_KEYS = dataclasses.replace(CSA_PREFILL, name="csa_prefill_s8192_index_keys",
                                             pool_index_keys=True, index_rope=64, workload=6)
CSA_DECODE_STEP = dataclasses.replace(CSA_DECODE, name="csa_decode_step_b64_ctx65536",
                                      cache_update=True, workload=5)


def mixed_stack(S: int = 131072) -> List[LayerSpec]:
    """Four-layer long-context block: CSA, HCA, CSA, sliding-only."""
    return [
        prefill("mixed_l0_csa", "bf16", S=S, H=64, D=512, R=64, base=160000.0, W=128, m=4,
                kind="csa", H_I=64, d_I=128, topk=512, workload=4, layer=0),
        prefill("mixed_l1_hca", "bf16", S=S, H=64, D=512, R=64, base=160000.0, W=128, m=128,
                kind="hca", workload=4, layer=1),
        prefill("mixed_l2_csa", "bf16", S=S, H=64, D=512, R=64, base=160000.0, W=128, m=4,
                kind="csa", H_I=64, d_I=128, topk=512, workload=4, layer=2),
        prefill("mixed_l3_sliding", "bf16", S=S, H=64, D=512, R=64, base=10000.0, W=128,
                m=4, kind="sliding", workload=4, layer=3),
    ]


CSA_PREFILL_PROJ = dataclasses.replace(CSA_PREFILL, name="csa_prefill_s8192_proj", proj=True,
                                       workload=7)

WORKLOADS: Dict[int, List[LayerSpec]] = {
    0: [TINY_CSA],
    1: [CSA_PREFILL],
    2: [HCA_PREFILL],
    3: [CSA_DECODE],
    4: mixed_stack(),
    5: [CSA_DECODE_STEP],
    6: [CSA_PREFILL_INDEX_KEYS],
    7: [CSA_PREFILL_PROJ],
}


def _randn(shape, seed: int, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def _rms_rows(x: torch.Tensor) -> torch.Tensor:
    xd = x.double()
    return xd / torch.sqrt(xd.pow(2).mean(dim=-1, keepdim=True) + RMS_EPS)


def make_inputs(spec: LayerSpec, device="cpu") -> Dict[str, Optional[torch.Tensor]]:
    """Seeded inputs for one layer, in the layer's storage dtype, on `device`.

    q [B,S_q,H,D]; kv [B,S_kv,D]; gate [B,S_kv,D] (prefill) ; pool [B,P,D] (decode);
    q_I [B,S_q,H_I,d_I]; w [B,S_q,H_I]; k_I [B,P,d_I] (CSA only); sink [H] fp32.
    The random stream depends on the device type; callers compare both sides on one copy.
    """
    dt = spec.torch_dtype
    out: Dict[str, Optional[torch.Tensor]] = {}
    out["q"] = _randn((spec.B, spec.S_q, spec.H, spec.D), spec.seed("q"), device).to(dt)
    out["kv"] = _rms_rows(_randn((spec.B, spec.S_kv, spec.D), spec.seed("kv"), device)).to(dt)
    if spec.decode:
        out["gate"] = None
        out["pool"] = _rms_rows(_randn((spec.B, spec.P, spec.D), spec.seed("pool"), device)).to(dt)
    else:
        out["gate"] = _randn((spec.B, spec.S_kv, spec.D), spec.seed("gate"), device).to(dt)
        out["pool"] = None
    if spec.kind == "csa":
        out["q_I"] = _randn((spec.B, spec.S_q, spec.H_I, spec.d_I), spec.seed("q_I"), device).to(dt)
        out["k_I"] = _randn((spec.B, spec.P, spec.d_I), spec.seed("k_I"), device).to(dt)
        out["w"] = (_randn((spec.B, spec.S_q, spec.H_I), spec.seed("w"), device)
                    / math.sqrt(spec.H_I)).to(dt)
    else:
        out["q_I"] = out["k_I"] = out["w"] = None
    out["sink"] = _randn((spec.H,), spec.seed("sink"), device)
    if spec.pool_index_keys:
        assert spec.kind == "csa" and not spec.decode
        out["k_I"] = None
        out["kI_tok"] = _rms_rows(_randn((spec.B, spec.S_kv, spec.d_I), spec.seed("kI_tok"),
                                         device)).to(dt)
        out["gI_tok"] = _randn((spec.B, spec.S_kv, spec.d_I), spec.seed("gI_tok"), device).to(dt)
    if spec.proj:
        assert not spec.decode and spec.kind != "sliding"
        # the step makes the raw K=V rows and gates itself, from x
        out["kv"] = out["gate"] = None
        out["x"] = _randn((spec.B, spec.S_kv, PROJ_HIDDEN), spec.seed("x"), device).to(dt)
        out.update(proj_weights(spec.H, spec.D, PROJ_GROUPS, PROJ_RANK, PROJ_HIDDEN, dt,
                                spec.seed("proj"), device=device))
    if spec.cache_update:
        assert spec.decode and spec.kind != "sliding" and spec.kv_pos0 + spec.S_kv == spec.q_pos0 + spec.S_q
        L = spec.ring
        st = _randn((spec.B, 2, L, spec.D), spec.seed("state"), device)
        st[:, 0] = _rms_rows(st[:, 0]).float()
        for p in range(spec.q_pos0 - L, spec.q_pos0):
            r = p - spec.kv_pos0
            if p >= 0 and 0 <= r < spec.S_kv:
                st[:, 0, p % L] = out["kv"][:, r].float()
        out["state"] = st.to(dt)
        out["gate_new"] = _randn((spec.B, spec.S_q, spec.D), spec.seed("gate_new"), device).to(dt)
        if spec.kind == "csa":
            out["state_I"] = _randn((spec.B, 2, L, spec.d_I), spec.seed("state_I"), device).to(dt)
            out["kI_new"] = _randn((spec.B, spec.S_q, spec.d_I), spec.seed("kI_new"), device).to(dt)
            out["gI_new"] = _randn((spec.B, spec.S_q, spec.d_I), spec.seed("gI_new"), device).to(dt)
    return out


def normal_rows(shape, dtype: torch.dtype, seed: int, device="cpu") -> torch.Tensor:
    """N(0,1) values of any shape (rows to rotate, and the like)."""
    return _randn(tuple(shape), seed, device).to(dtype)


def stream_rows(B: int, S: int, D: int, dtype: torch.dtype, seed: int, device="cpu"):
    """Raw rows of S tokens fed to a compressor: kv RMS-normalised N(0,1), gate N(0,1)
    (seeds `seed` and `seed + 1`)."""
    kv = _rms_rows(_randn((B, S, D), seed, device)).to(dtype)
    gate = _randn((B, S, D), seed + 1, device).to(dtype)
    return kv, gate


def kv_new(spec: LayerSpec, inp) -> torch.Tensor:
    """The new tokens' raw rows in a cache-update step: a view of the window's last S_q rows."""
    return inp["kv"][:, spec.S_kv - spec.S_q:]


def ring_history(state: torch.Tensor, pos0: int, m: int, overlap: int):
    """Rows of positions [s0, pos0) held by a compressor state [B, 2, L, D] (slot p mod L),
    s0 the start of the last closed block (overlap) or of the open window (no overlap):
    (kv rows [B, n, D], gate rows [B, n, D], s0).  Replaying them from s0 into a fresh
    stateful compressor rebuilds its buffer and overlap block."""
    L = state.shape[2]
    s0 = max(0, (pos0 // m - overlap) * m)
    slots = [p % L for p in range(s0, pos0)]
    return state[:, 0, slots], state[:, 1, slots], s0


def sample_rows(spec: LayerSpec, n_random: int = 256, seed: int = 12345) -> List[int]:
    """Query rows (0-based) to check on large shapes: the early rows, rows around the
    window edge, the top-k saturation point, every 128-boundary neighbourhood that is
    cheap, the last 16 rows and a seeded random set."""
    S = spec.S_q
    rows = set()
    m = max(spec.m, 1)
    rows.update(range(0, min(S, 2 * m + 2)))
    for c in (spec.W - 1, spec.W, spec.W + 1):
        if 0 <= c < S:
            rows.add(c)
    if spec.topk:
        for c in (spec.topk * m - 2, spec.topk * m - 1, spec.topk * m):
            if 0 <= c < S:
                rows.add(c)
    for c in range(127, S, max(128, S // 16)):
        rows.update(x for x in (c, c + 1) if x < S)
    rows.update(range(max(0, S - 16), S))
    g = torch.Generator().manual_seed(seed)
    if S > 0:
        rows.update(torch.randint(0, S, (n_random,), generator=g).tolist())
    return sorted(rows)


# Projection sizes around the layer.  The pages name o_groups, o_lora_rank and hidden_size
# but give no values; these are readings at the V4-Flash head shape: 64 heads of 512 in 8
# groups of 8 heads, 1024 low-rank features per group, a 4096-wide hidden state.
PROJ_HIDDEN, PROJ_GROUPS, PROJ_RANK = 4096, 8, 1024


def proj_weights(H: int, D: int, G: int, r: int, hidden: int, dtype: torch.dtype, seed: int,
                 device="cpu"):
    """Seeded weights of the projections, scaled like a linear layer's default init
    (N(0,1) / sqrt(fan_in)): w_a [G, r, (H/G)*D], w_b [hidden, G*r] (output projection);
    w_kv, w_gate [D, hidden] and kv_norm_w [D] ~ 1 + N(0,1)/10 (compressor inputs);
    seeds seed .. seed+4."""
    per = (H // G) * D
    w_a = (_randn((G, r, per), seed, device) / math.sqrt(per)).to(dtype)
    w_b = (_randn((hidden, G * r), seed + 1, device) / math.sqrt(G * r)).to(dtype)
    w_kv = (_randn((D, hidden), seed + 2, device) / math.sqrt(hidden)).to(dtype)
    w_gate = (_randn((D, hidden), seed + 3, device) / math.sqrt(hidden)).to(dtype)
    kv_norm_w = (1.0 + 0.1 * _randn((D,), seed + 4, device)).to(dtype)
    return {"w_a": w_a, "w_b": w_b, "w_kv": w_kv, "w_gate": w_gate, "kv_norm_w": kv_norm_w}
