"""Pins for the fp64 oracle: each check compares the oracle with something other than
itself -- a value the pages print (tests/golden/*.json, each with its citation), a closed
form, an invariant the layer must satisfy, a library routine in a special case that
reduces to it, or brute force on tiny inputs.

Each pin is a plain function that raises AssertionError.  test_oracle_pins.py runs them;
test_oracle_mutations.py runs them against deliberately broken builds of the oracle to
show that each plausible mistake fails at least one pin.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rng(seed):
    return np.random.default_rng(seed)


def _rms(x):
    return x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + 1e-6)


# ----------------------------------------------------------------------------- compressor
def pin_compress_uniform_gate_is_mean():
    """Uniform gates make the gated pool the plain mean over each window."""
    r = _rng(1)
    B, S, D, m = 2, 37, 5, 4
    kv = r.standard_normal((B, S, D))
    gate = np.full((B, S, D), 0.7)
    for overlap in (1, 0):
        pool = oracle.compress(kv, gate, m, overlap)
        assert pool.shape == (B, S // m, D)
        for j in range(S // m):
            lo = max(0, (j - 1) * m) if overlap else j * m
            ref = kv[:, lo:(j + 1) * m, :].mean(axis=1)
            np.testing.assert_allclose(pool[:, j], ref, rtol=1e-12, atol=1e-13)


def pin_compress_one_hot_gate_copies_row():
    """A gate logit 60 above the rest of the window selects that token's kv row."""
    r = _rng(2)
    B, S, D, m = 1, 32, 6, 4
    kv = r.standard_normal((B, S, D))
    for overlap in (1, 0):
        P = S // m
        gate = np.zeros((B, S, D))
        pick = []
        for j in range(P):
            lo = max(0, (j - 1) * m) if overlap else j * m
            hi = (j + 1) * m
            s = lo + (j * 7 + 3) % (hi - lo)
            pick.append(s)
        # gates are per token: make each chosen token dominate only the window that picks
        # it by testing one entry at a time
        for j in range(P):
            g = np.zeros((B, S, D))
            g[:, pick[j], :] = 60.0
            pool = oracle.compress(kv, g, m, overlap)
            np.testing.assert_allclose(pool[:, j], kv[:, pick[j]], rtol=0, atol=1e-20 + 1e-12)


def pin_compress_window_extents():
    """Perturbing token s changes exactly the entries whose window holds s:
    CSA (overlap) entries s//m and s//m + 1, HCA entry s//m, nothing past P*m."""
    r = _rng(3)
    B, S, D, m = 1, 30, 3, 4
    kv = r.standard_normal((B, S, D))
    gate = r.standard_normal((B, S, D))
    P = S // m
    for overlap in (1, 0):
        base = oracle.compress(kv, gate, m, overlap)
        for s in range(S):
            kv2 = kv.copy()
            kv2[:, s, :] += 1.0
            changed = set(np.nonzero(np.any(oracle.compress(kv2, gate, m, overlap) != base,
                                            axis=(0, 2)))[0].tolist())
            want = {s // m, s // m + 1} if overlap else {s // m}
            want = {j for j in want if j < P}
            assert changed == want, (overlap, s, changed, want)


def pin_compress_empty_pool():
    """HF PR #45616: the compressor returns an empty pool when no window has closed."""
    kv = np.ones((2, 3, 4))
    assert oracle.compress(kv, kv, 4, 1).shape == (2, 0, 4)
    assert oracle.compress(kv, kv, 128, 0).shape == (2, 0, 4)


def pin_compress_two_token_golden():
    g = _golden("compress_two_tokens.json")
    kv = np.array(g["kv"], dtype=np.float64)
    gate = np.broadcast_to(np.array(g["gate_token_logits"])[None, :, None], kv.shape).copy()
    pool = oracle.compress(kv, gate, g["m"], g["overlap"])
    np.testing.assert_allclose(pool, np.array(g["pool"]), rtol=1e-14, atol=1e-14)


# ----------------------------------------------------------------------------- stateful compressor
def _chunks(rng, S, m):
    """A split of S tokens into calls: single tokens, a window's worth, runs across
    several windows, in a seeded random order."""
    sizes = [1, 1, 2, max(1, m - 1), m, m + 1, 2 * m + 1, 3, 5 * m]
    out = []
    while sum(out) < S:
        out.append(min(int(rng.choice(sizes)), S - sum(out)))
    return out


def pin_stateful_compressor_equals_whole_sequence():
    """HF PR #45616 (compressor state on the cache: buffer, pooled cache; one update per
    call) and HF docs "Cache layers" (buffer / pool / counter, CSA overlap state): pooling
    token by token through the state yields the entries the stateless compressor computes
    over the whole sequence, for any split of the stream into calls, and each call emits
    exactly the entries whose windows close inside it."""
    for m, overlap, D in ((4, 1, 6), (8, 0, 5), (1, 1, 3), (3, 0, 4), (2, 1, 2)):
        rng = _rng(300 + 10 * m + overlap)
        B, S = 2, 61
        kv = rng.standard_normal((B, S, D))
        gate = 3.0 * rng.standard_normal((B, S, D))
        ref = oracle.compress(kv, gate, m, overlap)
        for chunks in ([1] * S, [S], _chunks(rng, S, m), _chunks(rng, S, m)):
            st = oracle.CompressorState(B, D, m, overlap)
            got, start = [], 0
            for c in chunks:
                e = st.append(kv[:, start:start + c], gate[:, start:start + c])
                assert e.shape == (B, (start + c) // m - start // m, D), (m, overlap, start, c)
                got.append(e)
                start += c
            np.testing.assert_allclose(np.concatenate(got, axis=1), ref, rtol=1e-13, atol=1e-13)


def pin_stateful_compressor_closes_at_worked_example():
    """HF docs "Attention mask layout", HCA paragraph (m=8): entry 0 (tokens 0..7) exists
    once token 7 is in, entry 1 (tokens 8..15) once token 15 is in; HF PR #45616: before a
    window closes the compressor returns an empty tensor, not nothing."""
    g = _golden("hca_visibility_m8.json")
    m, T = g["m"], g["tokens"]
    close_at = {t0: int(j) for j, t0 in g["first_visible_query"].items()}
    rng = _rng(7)
    kv, gate = rng.standard_normal((1, T, 3)), rng.standard_normal((1, T, 3))
    st = oracle.CompressorState(1, 3, m, 0)
    for t in range(T):
        e = st.append(kv[:, t:t + 1], gate[:, t:t + 1])
        if t in close_at:
            assert e.shape == (1, 1, 3), t
            j = close_at[t]
            w = np.exp(gate[0, j * m:(j + 1) * m] - gate[0, j * m:(j + 1) * m].max(axis=0))
            np.testing.assert_allclose(e[0, 0], (w * kv[0, j * m:(j + 1) * m]).sum(0) / w.sum(0),
                                       rtol=1e-13)
        else:
            assert e.shape == (1, 0, 3), t


def pin_stateful_compressor_state_holds_open_window():
    """The state after n tokens: the counter is n, the buffer holds the n mod m tokens of
    the open window, and (CSA, overlap) the overlap block is the last closed block."""
    m, D, B = 4, 3, 2
    rng = _rng(11)
    kv, gate = rng.standard_normal((B, 23, D)), rng.standard_normal((B, 23, D))
    st = oracle.CompressorState(B, D, m, 1)
    n = 0
    for c in (3, 1, 6, 2, 11):
        st.append(kv[:, n:n + c], gate[:, n:n + c])
        n += c
        assert list(st.counter) == [n] * B
        r = n % m
        np.testing.assert_array_equal(st.buf_kv[:, :r], kv[:, n - r:n])
        np.testing.assert_array_equal(st.buf_gate[:, :r], gate[:, n - r:n])
        if n >= m:
            c0 = (n // m - 1) * m
            assert list(st.n_ovl) == [m] * B
            np.testing.assert_array_equal(st.ovl_kv, kv[:, c0:c0 + m])
            np.testing.assert_array_equal(st.ovl_gate, gate[:, c0:c0 + m])


# ----------------------------------------------------------------------------- visibility
def pin_visibility_worked_example():
    g = _golden("hca_visibility_m8.json")
    m, T = g["m"], g["tokens"]
    P = T // m
    for j_str, t0 in g["first_visible_query"].items():
        j = int(j_str)
        for t in range(T):
            assert (j < oracle.n_visible(t, m, P)) == (t >= t0), (j, t)


def pin_hca_visibility_by_perturbation():
    """Changing pool entry j moves exactly the HCA outputs of queries t >= (j+1)m-1."""
    g = _golden("hca_visibility_m8.json")
    m, T = g["m"], g["tokens"]
    r = _rng(4)
    H, D = 2, 8
    q = r.standard_normal((1, T, H, D))
    kv = _rms(r.standard_normal((1, T, D)))
    pool = _rms(r.standard_normal((1, T // m, D)))
    sink = r.standard_normal(H)
    tpos = np.arange(T)
    base = oracle.attend(q, tpos, kv, 0, pool, m, None, sink, 4, 10000.0, 8, D ** -0.5, "hca")
    for j_str, t0 in g["first_visible_query"].items():
        p2 = pool.copy()
        p2[:, int(j_str)] += 0.5
        o2 = oracle.attend(q, tpos, kv, 0, p2, m, None, sink, 4, 10000.0, 8, D ** -0.5, "hca")
        moved = np.any(o2 != base, axis=(0, 2, 3))
        assert moved.tolist() == [t >= t0 for t in range(T)], (j_str, moved)


def pin_sliding_window_by_perturbation():
    """Sliding-only layer: row s reaches query t iff t-W < s <= t (the page's demo)."""
    g = _golden("sliding_window_w8.json")
    W, T = g["window"], g["tokens"]
    r = _rng(5)
    H, D = 2, 8
    q = r.standard_normal((1, T, H, D))
    kv = _rms(r.standard_normal((1, T, D)))
    sink = r.standard_normal(H)
    tpos = np.arange(T)
    base = oracle.attend(q, tpos, kv, 0, None, 4, None, sink, 2, 10000.0, W, D ** -0.5, "hca")
    reach = np.zeros((T, T), dtype=bool)
    for s in range(T):
        kv2 = kv.copy()
        kv2[:, s] += 0.5
        o2 = oracle.attend(q, tpos, kv2, 0, None, 4, None, sink, 2, 10000.0, W, D ** -0.5, "hca")
        reach[:, s] = np.any(o2 != base, axis=(0, 2, 3))
    for t_str, (lo, hi) in g["visible_keys_of_query"].items():
        t = int(t_str)
        assert np.nonzero(reach[t])[0].tolist() == list(range(lo, hi + 1)), (t, reach[t])
    for t in range(T):
        assert np.nonzero(reach[t])[0].tolist() == list(range(max(0, t - W + 1), t + 1))


def pin_csa_early_queries_get_marker():
    g = _golden("csa_early_queries_m4.json")
    m, k, T = g["m"], g["topk"], g["tokens"]
    r = _rng(6)
    P = T // m
    tpos = np.arange(T)
    sc = oracle.index_scores(r.standard_normal((1, T, 2, 4)), r.standard_normal((1, T, 2)),
                             r.standard_normal((1, P, 4)), tpos, m)
    idx, _ = oracle.topk(sc, tpos, m, k)
    for t in g["all_minus_one_queries"]:
        assert (idx[0, t] == -1).all()
    t = g["first_query_with_entry"]
    assert idx[0, t, 0] == 0 and idx[0, t, 1] == -1


# ----------------------------------------------------------------------------- indexer
def pin_indexer_unit_keys_golden():
    g = _golden("indexer_unit_keys.json")
    q = np.array(g["q_I_heads"])[None, None]          # [1,1,2,4]
    w = np.array(g["w"])[None, None]                  # [1,1,2]
    kI = np.eye(4)[None]                              # [1,4,4]
    t = g["query_position"]
    sc = oracle.index_scores(q, w, kI, [t], g["m"])
    np.testing.assert_allclose(sc[0, 0], g["scores"], rtol=0, atol=1e-15)
    idx, _ = oracle.topk(sc, [t], g["m"], 2)
    assert idx[0, 0].tolist() == g["top2"]


def pin_indexer_rope_zero_width_is_plain_indexer():
    """No rotated channels: the indexer with RoPE is the plain indexer."""
    rng = _rng(40)
    q, w, k = rng.standard_normal((2, 5, 3, 8)), rng.standard_normal((2, 5, 3)), rng.standard_normal((2, 6, 8))
    tpos = [3, 8, 11, 20, 23]
    np.testing.assert_array_equal(oracle.index_scores_rope(q, w, k, tpos, 4, 0, 10000.0),
                                  oracle.index_scores(q, w, k, tpos, 4))


def pin_indexer_rope_relative_position():
    """RoPE makes the score a function of t - j*m: moving the query by c*m positions and
    the keys by c entries (c new entries in front) leaves every score unchanged."""
    rng = _rng(41)
    m, c, R, base = 4, 5, 8, 160000.0
    q, w = rng.standard_normal((1, 3, 2, 16)), rng.standard_normal((1, 3, 2))
    k = rng.standard_normal((1, 9, 16))
    tpos = np.array([35, 36, 39])
    k2 = np.concatenate([rng.standard_normal((1, c, 16)), k], axis=1)
    s1 = oracle.index_scores_rope(q, w, k, tpos, m, R, base)
    s2 = oracle.index_scores_rope(q, w, k2, tpos + c * m, m, R, base)
    np.testing.assert_allclose(s2[:, :, c:], s1, rtol=1e-12, atol=1e-12)
    # and it is not the plain indexer: the rotation does change the scores
    assert np.nanmax(np.abs(s1 - oracle.index_scores(q, w, k, tpos, m))) > 1e-3


def pin_indexer_rope_two_dim_closed_form():
    """d_I = R = 2, one head, w = 1 (pair 0 turns by the position itself): q at angle a
    rotated by t, key j at angle b_j rotated by j*m, so the score is
    max(0, |q| |k_j| cos(a + t - b_j - j*m))."""
    m, t, a, qn = 3, 14, 0.3, 1.7
    b = np.array([0.2, -1.1, 2.5, 0.9])
    kn = np.array([1.0, 0.5, 2.0, 1.3])
    q = np.array([qn * math.cos(a), qn * math.sin(a)])[None, None, None]
    k = np.stack([kn * np.cos(b), kn * np.sin(b)], axis=-1)[None]
    sc = oracle.index_scores_rope(q, np.ones((1, 1, 1)), k, [t], m, 2, 10000.0)[0, 0]
    want = [max(0.0, qn * kn[j] * math.cos(a + t - b[j] - j * m)) for j in range(4)]
    np.testing.assert_allclose(sc, want, rtol=1e-12, atol=1e-12)


def pin_indexer_single_head_ranking():
    """H_I=1, w=1: the ranking is that of ReLU(q.k) (dot products from numpy matmul)."""
    r = _rng(7)
    P, d, m = 40, 16, 2
    q = r.standard_normal((1, 1, 1, d))
    kI = r.standard_normal((1, P, d))
    t = 2 * P  # everything visible
    sc = oracle.index_scores(q, np.ones((1, 1, 1)), kI, [t], m)
    ref = np.maximum(kI[0] @ q[0, 0, 0], 0.0)
    np.testing.assert_allclose(sc[0, 0], ref, rtol=1e-12, atol=1e-12)


def pin_topk_brute_force():
    """Top-k equals a full sort by (score desc, index asc) done with Python's sorted()."""
    r = _rng(8)
    B, n, P, m, k = 2, 9, 23, 3, 5
    sc = np.round(r.standard_normal((B, n, P)), 1)   # coarse values: plenty of exact ties
    tpos = np.array([0, 1, 2, 5, 8, 11, 30, 68, 100])
    idx, sel = oracle.topk(sc, tpos, m, k)
    for b in range(B):
        for i, t in enumerate(tpos):
            nv = min(P, (t + 1) // m)
            order = sorted(range(nv), key=lambda j: (-sc[b, i, j], j))[:k]
            want = order + [-1] * (k - len(order))
            assert idx[b, i].tolist() == want, (b, i, idx[b, i], want)


def pin_topk_saturates():
    """k >= n_vis selects every visible entry, then -1."""
    r = _rng(9)
    P, m = 10, 4
    tpos = [3, 7, 20, 39, 100]
    sc = r.standard_normal((1, len(tpos), P))
    idx, _ = oracle.topk(sc, tpos, m, 16)
    for i, t in enumerate(tpos):
        nv = min(P, (t + 1) // m)
        assert sorted(idx[0, i, :nv].tolist()) == list(range(nv))
        assert (idx[0, i, nv:] == -1).all()


# ----------------------------------------------------------------------------- RoPE
def pin_rope_pairs_and_angles():
    """Channel pairs (D-R+2i, D-R+2i+1) turn by pos * base^(-2i/R); other channels stay."""
    D, R, base = 10, 4, 100.0
    for pair in range(R // 2):
        x = np.zeros(D)
        x[D - R + 2 * pair] = 1.0
        pos = 3.0
        y = oracle.rope(x[None], [pos], R, base)[0]
        ang = pos * base ** (-2.0 * pair / R)
        want = np.zeros(D)
        want[D - R + 2 * pair] = math.cos(ang)
        want[D - R + 2 * pair + 1] = math.sin(ang)
        np.testing.assert_allclose(y, want, rtol=0, atol=1e-15)
    x = _rng(10).standard_normal((5, D))
    y = oracle.rope(x, [7.0] * 5, R, base)
    np.testing.assert_array_equal(y[:, :D - R], x[:, :D - R])


def pin_rope_orthogonal_and_inverse():
    r = _rng(11)
    D, R = 64, 16
    x = r.standard_normal((20, D))
    pos = r.integers(0, 200000, size=20).astype(np.float64)
    y = oracle.rope(x, pos, R, 10000.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    z = oracle.rope(y, -pos, R, 10000.0)
    np.testing.assert_allclose(z, x, rtol=0, atol=1e-11)


# ----------------------------------------------------------------------------- attention
def pin_single_key_closed_form():
    """One key, any rope: o = v e^l / (e^l + e^s) with l = scale q.v when the key sits at
    the query's position (rotation cancels in l and in the de-rotated output)."""
    r = _rng(12)
    H, D, R = 3, 16, 8
    q = r.standard_normal((H, D))
    v = r.standard_normal((1, D))
    sink = r.standard_normal(H)
    t = 12345.0
    scale = 0.3
    o = oracle.attend_keys(q, t, v, [t], sink, R, 10000.0, scale)
    for h in range(H):
        lg = scale * float(q[h] @ v[0])
        want = v[0] * math.exp(lg) / (math.exp(lg) + math.exp(sink[h]))
        np.testing.assert_allclose(o[h], want, rtol=1e-12, atol=1e-14)


def pin_two_dim_rope_relative_phase():
    """D=R=2, base irrelevant (theta_0 = 1): q=(1,0), key (1,0) at s, query at t:
    l = scale cos(t-s) and the de-rotated value is (cos(s-t), sin(s-t))."""
    scale, t = 0.9, 5.0
    q = np.array([[1.0, 0.0]])
    keys = np.array([[1.0, 0.0], [1.0, 0.0]])
    kpos = [2.0, 4.5]
    sink = np.array([-0.25])
    o = oracle.attend_keys(q, t, keys, kpos, sink, 2, 10000.0, scale)
    ls = [scale * math.cos(t - s) for s in kpos]
    M = max(ls + [sink[0]])
    Z = math.exp(sink[0] - M) + sum(math.exp(l - M) for l in ls)
    want = sum(math.exp(l - M) / Z * np.array([math.cos(s - t), math.sin(s - t)])
               for l, s in zip(ls, kpos))
    np.testing.assert_allclose(o[0], want, rtol=1e-13, atol=1e-15)


def pin_sink_minus_inf_is_causal_sdpa():
    """R=0, no pool, window >= S, sink = -inf: textbook causal MQA; checked against
    torch's scaled_dot_product_attention in float64 on the CPU."""
    r = _rng(13)
    B, S, H, D = 2, 11, 3, 8
    q = r.standard_normal((B, S, H, D))
    kv = r.standard_normal((B, S, D))
    sink = np.full(H, -np.inf)
    o = oracle.attend(q, np.arange(S), kv, 0, None, 4, None, sink, 0, 10000.0, S, D ** -0.5,
                      "hca")
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)                # B,H,S,D
    kt = torch.from_numpy(kv)[:, None].expand(B, H, S, D)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, is_causal=True)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=1e-12, atol=1e-13)


def pin_topk_at_least_pool_is_dense():
    """CSA with k >= P (every visible entry selected) equals HCA's dense attention."""
    r = _rng(14)
    B, S, H, D, R, m, W = 1, 40, 2, 16, 4, 4, 6
    P = S // m
    q = r.standard_normal((B, S, H, D))
    kv = _rms(r.standard_normal((B, S, D)))
    pool = oracle.compress(kv, r.standard_normal((B, S, D)), m, 1)
    sink = r.standard_normal(H)
    tpos = np.arange(S)
    sc = oracle.index_scores(r.standard_normal((B, S, 2, 8)), r.standard_normal((B, S, 2)),
                             r.standard_normal((B, P, 8)), tpos, m)
    idx, _ = oracle.topk(sc, tpos, m, P + 3)
    o_csa = oracle.attend(q, tpos, kv, 0, pool, m, idx, sink, R, 10000.0, W, D ** -0.5, "csa")
    o_hca = oracle.attend(q, tpos, kv, 0, pool, m, None, sink, R, 10000.0, W, D ** -0.5, "hca")
    np.testing.assert_allclose(o_csa, o_hca, rtol=1e-12, atol=1e-14)


def pin_position_shift_invariance():
    """Shifting the query and every key position by 1024 leaves the de-rotated output
    unchanged (explicit keys, and the window-only layer through the layer entry)."""
    r = _rng(15)
    H, D, R, base = 3, 32, 16, 10000.0
    q = r.standard_normal((H, D))
    keys = _rms(r.standard_normal((9, D)))
    kpos = np.array([0, 3, 4, 7, 8, 20, 33, 40, 41], dtype=np.float64)
    sink = r.standard_normal(H)
    a = oracle.attend_keys(q, 41.0, keys, kpos, sink, R, base, D ** -0.5)
    b = oracle.attend_keys(q, 41.0 + 1024, keys, kpos + 1024, sink, R, base, D ** -0.5)
    np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-11)
    S = 20
    qs = r.standard_normal((1, S, H, D))
    kv = _rms(r.standard_normal((1, S, D)))
    o1 = oracle.attend(qs, np.arange(S), kv, 0, None, 4, None, sink, R, base, 8, D ** -0.5, "hca")
    o2 = oracle.attend(qs, np.arange(S) + 1024, kv, 1024, None, 4, None, sink, R, base, 8,
                       D ** -0.5, "hca")
    np.testing.assert_allclose(o1, o2, rtol=1e-9, atol=1e-11)


def pin_entry_position_and_duplicates():
    """A CSA entry is a key rotated at j*m; a window row also covered by an entry counts
    twice (checked against the explicit-key form)."""
    r = _rng(16)
    H, D, R, m, W = 2, 16, 8, 4, 4
    S = 16
    q = r.standard_normal((1, S, H, D))
    kv = _rms(r.standard_normal((1, S, D)))
    pool = _rms(r.standard_normal((1, S // m, D)))
    sink = r.standard_normal(H)
    t = 11
    idx = np.full((1, 1, 3), -1, dtype=np.int32)
    idx[0, 0, :2] = [2, 0]
    o = oracle.attend(q[:, t:t + 1], [t], kv, 0, pool, m, idx, sink, R, 10000.0, W, D ** -0.5,
                      "csa")
    keys = np.concatenate([kv[0, t - W + 1:t + 1], pool[0, [2, 0]]])
    kpos = list(range(t - W + 1, t + 1)) + [2 * m, 0]
    want = oracle.attend_keys(q[0, t], t, keys, kpos, sink, R, 10000.0, D ** -0.5)
    np.testing.assert_allclose(o[0, 0], want, rtol=1e-13, atol=1e-15)
    # duplicate: entry row equal to a window row doubles that row's weight
    keys2 = np.concatenate([keys, keys[-3:-2]])
    kpos2 = kpos + [kpos[-3]]
    dup = oracle.attend_keys(q[0, t], t, keys2, kpos2, sink, R, 10000.0, D ** -0.5)
    assert not np.allclose(dup, want)


# ----------------------------------------------------------------------------- output projection
def _proj_weights(rng, G, r, H, D, hidden):
    return rng.standard_normal((G, r, (H // G) * D)), rng.standard_normal((hidden, G * r))


def pin_grouped_out_proj_one_group_is_two_linears():
    """With one group the projection is o_b_proj(o_a_proj(flattened heads)): checked with
    torch.nn.functional.linear in float64."""
    rng = _rng(50)
    B, S, H, D, r, hidden = 2, 3, 4, 6, 5, 7
    o = rng.standard_normal((B, S, H, D))
    w_a, w_b = _proj_weights(rng, 1, r, H, D, hidden)
    t = torch.from_numpy
    want = torch.nn.functional.linear(torch.nn.functional.linear(t(o).reshape(B, S, H * D),
                                                                 t(w_a[0])), t(w_b)).numpy()
    np.testing.assert_allclose(oracle.grouped_out_proj(o, w_a, w_b), want, rtol=1e-12, atol=1e-12)


def pin_grouped_out_proj_block_diagonal():
    """G groups equal one dense o_a_proj whose weight is block-diagonal in the groups
    (scipy's block_diag), followed by o_b_proj."""
    from scipy.linalg import block_diag
    rng = _rng(51)
    B, S, H, D, G, r, hidden = 1, 4, 8, 3, 4, 2, 5
    o = rng.standard_normal((B, S, H, D))
    w_a, w_b = _proj_weights(rng, G, r, H, D, hidden)
    dense = block_diag(*[w_a[g] for g in range(G)])          # [G*r, H*D]
    want = (o.reshape(B, S, H * D) @ dense.T) @ w_b.T
    np.testing.assert_allclose(oracle.grouped_out_proj(o, w_a, w_b), want, rtol=1e-12, atol=1e-12)


def pin_grouped_out_proj_head_groups():
    """Group g sees exactly heads [g*H/G, (g+1)*H/G): changing one head moves only its
    group's low-rank features."""
    rng = _rng(52)
    B, S, H, D, G, r, hidden = 1, 2, 8, 4, 4, 3, 6
    o = rng.standard_normal((B, S, H, D))
    w_a, w_b = _proj_weights(rng, G, r, H, D, hidden)
    _, z0 = oracle.grouped_out_proj(o, w_a, w_b, return_groups=True)
    for h in range(H):
        o2 = o.copy()
        o2[:, :, h] += 1.0
        _, z1 = oracle.grouped_out_proj(o2, w_a, w_b, return_groups=True)
        moved = np.abs(z1 - z0).max(axis=(0, 1, 3)) > 1e-9
        assert moved.tolist() == [g == h // (H // G) for g in range(G)], h


# ----------------------------------------------------------------------------- input projections
def pin_kv_gate_proj_one_hot_weights_select_channels():
    """One-hot weight rows make both projections pick token channels: gate channel d is
    x[..., perm[d]] (a transposed weight would pick a different channel), and kv is that
    selection divided by its own RMS, times the norm weight (closed form)."""
    rng = _rng(60)
    hidden, D = 9, 5
    x = rng.standard_normal((2, 3, hidden))
    perm = rng.permutation(hidden)[:D]
    w = np.zeros((D, hidden))
    w[np.arange(D), perm] = 1.0
    gam = rng.uniform(0.5, 2.0, D)
    eps = 1e-6
    kv, gate = oracle.kv_gate_proj(x, w, w, gam, eps)
    sel = x[..., perm]
    np.testing.assert_allclose(gate, sel, rtol=0, atol=0)
    want = sel / np.sqrt((sel ** 2).sum(axis=-1, keepdims=True) / D + eps) * gam
    np.testing.assert_allclose(kv, want, rtol=1e-13, atol=1e-13)


def pin_kv_gate_proj_norm_invariants():
    """With a unit norm weight and eps = 0 every K=V row has mean square exactly 1 and is
    unchanged by scaling the token; the gate logits scale with the token; the norm
    weight multiplies channel by channel after the normalisation."""
    rng = _rng(61)
    hidden, D = 16, 8
    x = rng.standard_normal((4, hidden))
    wk, wg = rng.standard_normal((D, hidden)), rng.standard_normal((D, hidden))
    ones = np.ones(D)
    kv, gate = oracle.kv_gate_proj(x, wk, wg, ones, 0.0)
    np.testing.assert_allclose((kv ** 2).mean(axis=-1), 1.0, rtol=1e-13)
    kv3, gate3 = oracle.kv_gate_proj(3.0 * x, wk, wg, ones, 0.0)
    np.testing.assert_allclose(kv3, kv, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gate3, 3.0 * gate, rtol=1e-12, atol=1e-12)
    gam = rng.uniform(0.5, 2.0, D)
    kvg, _ = oracle.kv_gate_proj(x, wk, wg, gam, 0.0)
    np.testing.assert_allclose(kvg, kv * gam, rtol=1e-12, atol=1e-12)


def pin_kv_gate_proj_epsilon():
    """eps enters under the square root with the mean square: for a token whose projection
    is the constant c on every channel, kv = c / sqrt(c^2 + eps) (closed form)."""
    hidden, D = 4, 6
    x = np.array([[1.0, 0.0, 0.0, 0.0]])
    c = 0.01
    w = np.zeros((D, hidden))
    w[:, 0] = c
    kv, gate = oracle.kv_gate_proj(x, w, w, np.ones(D), 1e-4)
    np.testing.assert_allclose(kv, c / math.sqrt(c * c + 1e-4), rtol=1e-13)
    np.testing.assert_allclose(gate, c, rtol=0)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
