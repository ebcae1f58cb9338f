"""CSA prefill of one long sequence sharded over the GPUs of one node (query rows), with
one all-gather of the compressed entries and their index keys.

The layer's work splits by query row: a query needs its own q, q_I, w, the raw K=V rows of
its sliding window and every visible compressed entry with its index key.  Rank r of N:

  * owns the query rows of two chunks of the sequence, chunk r and chunk 2N-1-r of 2N
    equal chunks (a zig-zag split: causal attention makes late rows dearer, the pairing
    evens out the ranks);
  * pools the compressed entries [r*Pn, (r+1)*Pn) of the sequence (Pn = ceil(P/N)) from
    the raw rows their windows cover (for CSA's overlapping windows one block of m rows
    before its first entry is read as a halo), and holds the matching index keys;
  * all-gathers the entries and index keys of every rank (one collective each, padded to
    N*Pn rows), after which every query row it owns sees the whole pool;
  * runs the indexer and the attention on its own chunks, reading the raw rows of each
    chunk plus the window-1 rows before it.

The arithmetic runs in the backend's kernels; this module only slices, calls and
gathers.  `backend` provides compress, index_topk, attend (the library calls, or any
object with the same signatures) and all_gather (a collective over the ranks).
"""
from __future__ import annotations

from typing import List, Tuple


def zigzag_chunks(S: int, world: int, rank: int) -> List[Tuple[int, int]]:
    """Query rows of `rank`: chunks rank and 2*world-1-rank of 2*world near-equal chunks
    of [0, S) (a single chunk when world == 1)."""
    if world == 1:
        return [(0, S)]
    n = 2 * world
    bounds = [S * k // n for k in range(n + 1)]
    out = []
    for c in (rank, n - 1 - rank):
        if bounds[c + 1] > bounds[c]:
            out.append((bounds[c], bounds[c + 1]))
    return out


def entry_range(P: int, world: int, rank: int) -> Tuple[int, int, int]:
    """Entries [j0, j1) that `rank` pools, and the padded per-rank count Pn."""
    pn = (P + world - 1) // world if P else 0
    j0 = min(P, rank * pn)
    j1 = min(P, j0 + pn)
    return j0, j1, pn


def entry_rows(j0: int, j1: int, m: int, overlap: int) -> Tuple[int, int, int]:
    """Raw rows [a, b) whose pooling gives entries j0 .. j1-1, and how many leading
    entries of that pooling to drop (an overlapping window clipped at row a)."""
    if j1 <= j0:
        return 0, 0, 0
    if overlap and j0 > 0:
        return (j0 - 1) * m, j1 * m, 1
    return j0 * m, j1 * m, 0


def window_rows(c0: int, c1: int, window: int) -> Tuple[int, int]:
    """Raw rows [a, b) a chunk of query rows [c0, c1) reads for its sliding windows."""
    return max(0, c0 - window + 1), c1


def local_entries(backend, world: int, rank: int, inp: dict, spec):
    """Phase 1 on `rank`: its compressed entries and their index keys, each padded to Pn
    rows ([B, Pn, D] and [B, Pn, d_I]), ready for the all-gather."""
    m, ov = spec.m, spec.overlap
    j0, j1, pn = entry_range(spec.P, world, rank)
    a, b, drop = entry_rows(j0, j1, m, ov)
    pool_loc = backend.compress(backend.rows(inp["kv"], a, b), backend.rows(inp["gate"], a, b), m, ov)
    pool_loc = backend.rows(pool_loc, drop, drop + (j1 - j0))
    k_loc = backend.rows(inp["k_I"], j0, j1)
    return backend.pad_rows(pool_loc, pn), backend.pad_rows(k_loc, pn)


def attend_rows(backend, world: int, rank: int, inp: dict, spec, pool, k_I) -> dict:
    """Phase 2 on `rank`: indexer and attention for its query chunks over the gathered pool
    and index keys ([B, P, ...]).  Returns {"chunks", "idx", "out"} (one entry per chunk)."""
    res = {"chunks": zigzag_chunks(spec.S_q, world, rank), "out": [], "idx": []}
    for c0, c1 in res["chunks"]:
        wa, wb = window_rows(c0, c1, spec.W)
        idx = backend.index_topk(backend.rows(inp["q_I"], c0, c1), backend.rows(inp["w"], c0, c1), k_I,
                                 c0, spec.m, spec.topk)
        out = backend.attend(backend.rows(inp["q"], c0, c1), backend.rows(inp["kv"], wa, wb), wa, pool, idx,
                             inp["sink"], c0, spec.R, spec.base, spec.W, spec.m, spec.scale)
        res["idx"].append(idx)
        res["out"].append(out)
    return res


def prefill_sharded(backend, world: int, rank: int, inp: dict, spec) -> dict:
    """The CSA prefill layer for the rows `rank` owns: phase 1, one all-gather of the
    entries and one of the index keys, phase 2.  inp holds the sequence's inputs as the
    backend's tensors ([B, S, ...]); a rank reads only the slices it needs.  Returns the
    phase-2 result plus the gathered "pool" and "k_I"."""
    pool_loc, k_loc = local_entries(backend, world, rank, inp, spec)
    pool = backend.rows(backend.all_gather(pool_loc), 0, spec.P)
    k_I = backend.rows(backend.all_gather(k_loc), 0, spec.P)
    res = attend_rows(backend, world, rank, inp, spec, pool, k_I)
    res["pool"], res["k_I"] = pool, k_I
    return res


class LibraryBackend:
    """The library's kernels on this rank's GPU, with NCCL (torch.distributed) for the
    all-gather.  Row slices of [B, S, ...] tensors are made contiguous before a call."""

    def __init__(self, group=None):
        import torch
        import torch.distributed as dist

        import sparse_attention_14_b200 as csa
        self.torch, self.dist, self.csa, self.group = torch, dist, csa, group

    def rows(self, t, a, b):
        return t[:, a:b].contiguous()

    def pad_rows(self, t, n):
        if t.shape[1] == n:
            return t
        pad = self.torch.zeros((t.shape[0], n - t.shape[1]) + tuple(t.shape[2:]), dtype=t.dtype,
                               device=t.device)
        return self.torch.cat([t, pad], dim=1)

    def all_gather(self, t):
        """[B, n, ...] per rank -> [B, world*n, ...], rank-major along the rows."""
        world = self.dist.get_world_size(self.group) if self.dist.is_initialized() else 1
        if world == 1:
            return t
        buf = self.torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        self.dist.all_gather_into_tensor(buf, t.contiguous(), group=self.group)
        return buf.transpose(0, 1).reshape((t.shape[0], world * t.shape[1]) + tuple(t.shape[2:]))

    def compress(self, kv, gate, m, overlap):
        return self.csa.csa_compress(kv, gate, m, overlap)

    def index_topk(self, q_I, w, k_I, q_pos0, m, topk):
        return self.csa.csa_index_topk(q_I, w, k_I, q_pos0, m, topk)

    def attend(self, q, kv, kv_pos0, pool, idx, sink, q_pos0, R, base, W, m, scale):
        return self.csa.csa_attend(q, kv, kv_pos0, pool, idx, sink, q_pos0, R, base, W, m, scale)
