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
