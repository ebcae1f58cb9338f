"""GPU parity of the projections around the layer (the C ABI against the fp64 oracle on
the same seeded bf16 inputs): the grouped low-rank output projection after the attention
and the compressor's kv/gate input projections with the kv RMSNorm.  Shapes span several
128-row tiles with a ragged tail, several 256-column tiles and every o_a group; the full
V4-Flash-like sizes are checked on sampled rows.  Tolerance: bf16 (2e-2, max-norm
relative), as for every bf16 layer output."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import csa_synth as cs
import oracle
import sparse_attention_14_b200 as csa
from parity_util import TOL, rel_err, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"

OUT_CASES = [  # name, M, H, D, G, r, hidden
    ("small_2groups", 300, 8, 64, 2, 256, 512),
    ("ragged_4groups", 389, 16, 128, 4, 256, 768),
    ("v4_flash_rows", 8192, 64, 512, 8, 1024, 4096),
]


@pytest.mark.parametrize("name,M,H,D,G,r,hidden", OUT_CASES, ids=[c[0] for c in OUT_CASES])
def test_out_proj_parity(name, M, H, D, G, r, hidden):
    seed = 1100 + [c[0] for c in OUT_CASES].index(name) * 10
    w = cs.proj_weights(H, D, G, r, hidden, torch.bfloat16, seed, device=DEV)
    o = cs.normal_rows((M, H, D), torch.bfloat16, seed + 7, device=DEV)
    y = csa.csa_out_proj(o, w["w_a"], w["w_b"])
    torch.cuda.synchronize()
    assert csa.device_status() == 0
    rows = np.arange(M) if M <= 512 else np.unique(np.r_[np.arange(0, 130), np.arange(M - 130, M),
                                                          np.random.default_rng(seed).integers(0, M, 200)])
    rt = torch.from_numpy(rows).to(DEV)
    ref = oracle.grouped_out_proj(to_np(o[rt])[None], to_np(w["w_a"]), to_np(w["w_b"]))[0]
    assert rel_err(to_np(y[rt]), ref) <= TOL["bf16"]


KV_CASES = [  # name, M, hidden, D
    ("small_d256", 200, 256, 256),
    ("ragged_d512", 333, 1024, 512),
    ("v4_flash_rows", 8192, 4096, 512),
]


@pytest.mark.parametrize("name,M,hidden,D", KV_CASES, ids=[c[0] for c in KV_CASES])
def test_kv_gate_proj_parity(name, M, hidden, D):
    seed = 1200 + [c[0] for c in KV_CASES].index(name) * 10
    w = cs.proj_weights(8, D, 1, 256, 256, torch.bfloat16, seed, device=DEV)
    w_kv = (torch.randn((D, hidden), generator=torch.Generator(DEV).manual_seed(seed + 5), device=DEV)
            / hidden ** 0.5).to(torch.bfloat16)
    x = cs.normal_rows((M, hidden), torch.bfloat16, seed + 7, device=DEV)
    w_gate = (torch.randn((D, hidden), generator=torch.Generator(DEV).manual_seed(seed + 6), device=DEV)
              / hidden ** 0.5).to(torch.bfloat16)
    kv, gate = csa.csa_kv_gate_proj(x, w_kv, w_gate, w["kv_norm_w"], 1e-6)
    torch.cuda.synchronize()
    assert csa.device_status() == 0
    rows = np.arange(M) if M <= 512 else np.unique(np.r_[np.arange(0, 130), np.arange(M - 130, M),
                                                          np.random.default_rng(seed).integers(0, M, 200)])
    rt = torch.from_numpy(rows).to(DEV)
    kv_ref, gate_ref = oracle.kv_gate_proj(to_np(x[rt]), to_np(w_kv), to_np(w_gate),
                                           to_np(w["kv_norm_w"]), 1e-6)
    assert rel_err(to_np(gate[rt]), gate_ref) <= TOL["bf16"]
    assert rel_err(to_np(kv[rt]), kv_ref) <= TOL["bf16"]
    # every K=V row comes out RMS-normalised (times the norm weight)
    unit = to_np(kv[rt]) / to_np(w["kv_norm_w"])[None]
    np.testing.assert_allclose(np.sqrt((unit ** 2).mean(axis=-1)), 1.0, rtol=2e-2)


def test_projections_reject_unsupported_shapes():
    o = torch.zeros((4, 8, 64), dtype=torch.bfloat16, device=DEV)
    w_a = torch.zeros((2, 100, 256), dtype=torch.bfloat16, device=DEV)   # r not a multiple of 256
    w_b = torch.zeros((256, 200), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(csa.CsaError):
        csa.csa_out_proj(o, w_a, w_b)
    x = torch.zeros((4, 100), dtype=torch.bfloat16, device=DEV)          # hidden not a multiple of 64
    w = torch.zeros((256, 100), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(csa.CsaError):
        csa.csa_kv_gate_proj(x, w, w, torch.ones(256, dtype=torch.bfloat16, device=DEV))


def test_workload7_layer_with_projections_sampled():
    """The CSA prefill layer with its projections at full size (S = 8192, hidden 4096), in
    the benchmark's call sequence, checked stage by stage on sampled rows: kv/gate against
    the oracle's projections of the same token rows, the pool over the GPU's kv/gate, the
    top-k sets (tie band), the attention over the GPU's pool, rows and validated top-k, and
    the output projection of the GPU's attention output."""
    from parity_util import check_topk, kk_rows
    spec = cs.WORKLOADS[7][0]
    inp = cs.make_inputs(spec, device=DEV)
    kv, gate = csa.csa_kv_gate_proj(inp["x"], inp["w_kv"], inp["w_gate"], inp["kv_norm_w"], 1e-6)
    pool = csa.csa_compress(kv, gate, spec.m, spec.overlap)
    idx = csa.csa_index_topk(inp["q_I"], inp["w"], inp["k_I"], spec.q_pos0, spec.m, spec.topk)
    out = csa.csa_attend(inp["q"], kv, spec.kv_pos0, pool, idx, inp["sink"], spec.q_pos0, spec.R,
                         spec.base, spec.W, spec.m, spec.scale)
    y = csa.csa_out_proj(out, inp["w_a"], inp["w_b"])
    torch.cuda.synchronize()
    assert csa.device_status() == 0
    rows = cs.sample_rows(spec, n_random=48)
    rt = torch.tensor(rows, device=DEV)
    kv_ref, gate_ref = oracle.kv_gate_proj(to_np(inp["x"][0, rt]), to_np(inp["w_kv"]),
                                           to_np(inp["w_gate"]), to_np(inp["kv_norm_w"]), 1e-6)
    assert rel_err(to_np(kv[0, rt]), kv_ref) <= TOL["bf16"]
    assert rel_err(to_np(gate[0, rt]), gate_ref) <= TOL["bf16"]
    kv_h = to_np(kv)
    assert rel_err(to_np(pool), oracle.compress(kv_h, to_np(gate), spec.m, spec.overlap)) <= TOL["bf16"]
    tpos = np.asarray(rows, dtype=np.int64) + spec.q_pos0
    sc = oracle.index_scores(to_np(inp["q_I"][:, rt]), to_np(inp["w"][:, rt]), to_np(inp["k_I"]), tpos,
                             spec.m)
    o_idx, _ = oracle.topk(sc, tpos, spec.m, spec.topk)
    g_idx = idx[:, rt].cpu().numpy()
    check_topk(g_idx[0], o_idx[0], sc[0], kk_rows(spec, rows))
    ref = oracle.attend(to_np(inp["q"][:, rt]), tpos, kv_h, spec.kv_pos0, to_np(pool), spec.m, g_idx,
                        to_np(inp["sink"]), spec.R, spec.base, spec.W, spec.scale, "csa")
    assert rel_err(to_np(out[:, rt]), ref) <= TOL["bf16"]
    y_ref = oracle.grouped_out_proj(to_np(out[:, rt]), to_np(inp["w_a"]), to_np(inp["w_b"]))
    assert rel_err(to_np(y[:, rt]), y_ref) <= TOL["bf16"]
