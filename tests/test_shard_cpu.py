"""The sharded CSA prefill (query rows over ranks, one all-gather of the compressed entries
and index keys) on the CPU with the gloo backend, world_size 2: the host logic of
sparse_attention_14_b200.shard with the fp64 oracle standing in for the kernels, against
the oracle's unsharded layer on the same inputs."""
from __future__ import annotations

import datetime
import os
import socket
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _spec():
    from csa_synth import LayerSpec
    return LayerSpec(name="shard_tiny_f32", dtype="f32", B=2, S_q=97, S_kv=97, q_pos0=0, kv_pos0=0,
                     H=4, D=32, R=8, base=10000.0, W=16, m=4, P=24, kind="csa", H_I=2, d_I=16, topk=8,
                     workload=75)


class OracleBackend:
    """The oracle's CPU implementation of each step (test infrastructure) and a gloo
    all-gather, behind the backend interface the sharded runner calls."""

    def __init__(self, world):
        import oracle
        self.o, self.world = oracle, world

    def rows(self, t, a, b):
        return np.ascontiguousarray(t[:, a:b])

    def pad_rows(self, t, n):
        pad = np.zeros((t.shape[0], n - t.shape[1]) + t.shape[2:])
        return np.concatenate([t, pad], axis=1)

    def all_gather(self, t):
        if self.world == 1:
            return t
        parts = [torch.zeros(t.shape, dtype=torch.float64) for _ in range(self.world)]
        dist.all_gather(parts, torch.from_numpy(np.ascontiguousarray(t)))
        return np.concatenate([p.numpy() for p in parts], axis=1)

    def compress(self, kv, gate, m, overlap):
        return self.o.compress(kv, gate, m, overlap)

    def index_topk(self, q_I, w, k_I, q_pos0, m, topk):
        tpos = np.arange(q_I.shape[1], dtype=np.int64) + q_pos0
        sc = self.o.index_scores(q_I, w, k_I, tpos, m)
        return self.o.topk(sc, tpos, m, topk)[0]

    def attend(self, q, kv, kv_pos0, pool, idx, sink, q_pos0, R, base, W, m, scale):
        tpos = np.arange(q.shape[1], dtype=np.int64) + q_pos0
        return self.o.attend(q, tpos, kv, kv_pos0, pool, m, idx, sink, R, base, W, scale, "csa")


def _inputs(spec):
    import csa_synth as cs
    inp = cs.make_inputs(spec, device="cpu")
    return {k: (None if v is None else v.double().numpy()) for k, v in inp.items()}


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        from sparse_attention_14_b200 import shard
        spec = _spec()
        res = shard.prefill_sharded(OracleBackend(world), world, rank, _inputs(spec), spec)
        q.put((rank, res["chunks"], [o for o in res["out"]], [i for i in res["idx"]], res["pool"],
               res["k_I"]))
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_partition_covers_rows_and_entries():
    sys.path.insert(0, ROOT)
    from sparse_attention_14_b200 import shard
    for S, world in [(97, 2), (8192, 4), (5, 4), (131072, 8)]:
        rows = sorted(r for rk in range(world) for c0, c1 in shard.zigzag_chunks(S, world, rk)
                      for r in range(c0, c1))
        assert rows == list(range(S))
    for P, world in [(24, 2), (2048, 8), (3, 4), (0, 2)]:
        got = []
        for rk in range(world):
            j0, j1, pn = shard.entry_range(P, world, rk)
            assert j1 - j0 <= pn
            got += list(range(j0, j1))
        assert got == list(range(P))
    # the raw rows an entry range reads: its windows, plus one block of halo for overlap
    assert shard.entry_rows(5, 9, 4, 1) == (16, 36, 1)
    assert shard.entry_rows(0, 9, 4, 1) == (0, 36, 0)
    assert shard.entry_rows(5, 9, 128, 0) == (640, 1152, 0)
    assert shard.window_rows(100, 200, 128) == (0, 200)
    assert shard.window_rows(300, 400, 128) == (173, 400)


def test_two_ranks_gloo_match_unsharded_oracle():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    import oracle
    spec = _spec()
    inp = _inputs(spec)
    pool = oracle.compress(inp["kv"], inp["gate"], spec.m, spec.overlap)
    tpos = np.arange(spec.S_q, dtype=np.int64)
    sc = oracle.index_scores(inp["q_I"], inp["w"], inp["k_I"], tpos, spec.m)
    idx, _ = oracle.topk(sc, tpos, spec.m, spec.topk)
    out = oracle.attend(inp["q"], tpos, inp["kv"], 0, pool, spec.m, idx, inp["sink"], spec.R, spec.base,
                        spec.W, spec.scale, "csa")
    covered = np.zeros(spec.S_q, dtype=bool)
    for rank, chunks, outs, idxs, g_pool, g_k in res:
        # every rank holds the whole pool and index keys after the all-gather
        np.testing.assert_allclose(g_pool, pool, rtol=1e-12, atol=1e-12)
        np.testing.assert_array_equal(g_k, inp["k_I"])
        for (c0, c1), o, ix in zip(chunks, outs, idxs):
            np.testing.assert_array_equal(ix, idx[:, c0:c1])
            np.testing.assert_allclose(o, out[:, c0:c1], rtol=1e-11, atol=1e-11)
            covered[c0:c1] = True
    assert covered.all()
