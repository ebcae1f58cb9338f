"""The sharded CSA prefill on the GPU: two ranks emulated one after the other on one device
(phase 1 of both, the all-gather done as the concatenation it produces, then phase 2 of
both), through the library's kernels, at the full S = 8192 prefill shape.  Every query
row's top-k and attention output must equal the unsharded call's bit for bit: a row's
work does not depend on which rank computes it."""
from __future__ import annotations

import pytest
import torch

import csa_synth as cs
import sparse_attention_14_b200 as csa
from sparse_attention_14_b200 import shard

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 4])
def test_sharded_prefill_equals_unsharded(world):
    spec = cs.CSA_PREFILL
    inp = cs.make_inputs(spec, device="cuda")
    pool = csa.csa_compress(inp["kv"], inp["gate"], spec.m, spec.overlap)
    idx = csa.csa_index_topk(inp["q_I"], inp["w"], inp["k_I"], 0, spec.m, spec.topk)
    out = csa.csa_attend(inp["q"], inp["kv"], 0, pool, idx, inp["sink"], 0, spec.R, spec.base, spec.W,
                         spec.m, spec.scale)
    be = shard.LibraryBackend()
    loc = [shard.local_entries(be, world, r, inp, spec) for r in range(world)]
    g_pool = torch.cat([p for p, _ in loc], dim=1)[:, :spec.P]
    g_k = torch.cat([k for _, k in loc], dim=1)[:, :spec.P]
    torch.cuda.synchronize()
    assert torch.equal(g_pool, pool)
    assert torch.equal(g_k, inp["k_I"])
    covered = torch.zeros(spec.S_q, dtype=torch.bool)
    for r in range(world):
        res = shard.attend_rows(be, world, r, inp, spec, g_pool, g_k)
        torch.cuda.synchronize()
        for (c0, c1), ix, o in zip(res["chunks"], res["idx"], res["out"]):
            assert torch.equal(ix, idx[:, c0:c1]), (r, c0)
            assert torch.equal(o, out[:, c0:c1]), (r, c0)
            covered[c0:c1] = True
    assert covered.all()
    assert csa.device_status() == 0
