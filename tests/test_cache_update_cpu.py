"""Host side of the decode step with the compressor cache update, on the CPU: the seeded
step inputs (state rings in the layout csa_compress_append documents), rebuilding the
oracle's stateful compressor from them, and the bench's work count for the step."""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest
import torch

import bench
import csa_synth as cs
import oracle


def _small_step(kind="csa"):
    if kind == "csa":
        return dataclasses.replace(cs.CSA_DECODE_STEP, B=2, P=1024, q_pos0=4095, kv_pos0=3968,
                                   workload=70)
    return dataclasses.replace(cs.CSA_DECODE_STEP, kind="hca", m=128, P=32, q_pos0=4095,
                               kv_pos0=3968, H_I=0, d_I=0, topk=0, workload=71)


def _f64(t):
    return t.double().numpy()


@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_state_ring_holds_window_rows(kind):
    spec = _small_step(kind)
    inp = cs.make_inputs(spec)
    L = spec.ring
    for p in range(spec.q_pos0 - L, spec.q_pos0):
        r = p - spec.kv_pos0
        if 0 <= r < spec.S_kv:
            assert torch.equal(inp["state"][:, 0, p % L], inp["kv"][:, r]), p
    # the new token is the window's last row
    assert torch.equal(cs.kv_new(spec, inp)[:, 0], inp["kv"][:, -1])
    assert ("state_I" in inp) == (kind == "csa")


@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_resumed_oracle_entry_is_the_closing_window(kind):
    """Rebuilding the oracle's compressor from the ring and appending the new token gives
    the entry pooled directly over the tokens of its window (stateless oracle on those
    rows laid out as a short sequence whose last window is that one)."""
    spec = _small_step(kind)
    inp = cs.make_inputs(spec)
    m, L, t = spec.m, spec.ring, spec.q_pos0
    kh, gh, s0 = cs.ring_history(inp["state"], t, m, spec.overlap)
    st = oracle.CompressorState.resume(_f64(kh), _f64(gh), s0, m, spec.overlap)
    ent = st.append(_f64(cs.kv_new(spec, inp)), _f64(inp["gate_new"]))
    assert ent.shape == (spec.B, 1, spec.D)
    # the window of the entry closing at t: positions [t+1-L, t+1)
    win = list(range(t + 1 - L, t + 1))
    kv = torch.stack([inp["state"][:, 0, p % L] if p < t else inp["kv"][:, -1] for p in win], 1)
    g = torch.stack([inp["state"][:, 1, p % L] if p < t else inp["gate_new"][:, 0] for p in win], 1)
    ref = oracle.compress(_f64(kv), _f64(g), m, spec.overlap)[:, -1]
    np.testing.assert_allclose(ent[:, 0], ref, rtol=1e-13, atol=1e-13)


def test_resume_needs_a_window_start():
    with pytest.raises(ValueError):
        oracle.CompressorState.resume(np.zeros((1, 3, 4)), np.zeros((1, 3, 4)), 5, 4, 1)


def test_step_work_counts():
    s = cs.CSA_DECODE_STEP
    w = bench.algorithmic_work(s)
    # one token: read + store kv and gate (4 rows), 7 earlier rows of the closing window
    # (kv + gate), one entry written; main compressor at D=512 and indexer keys at d_I=128
    assert w["append_bytes"] == s.B * (4 + 14 + 1) * (512 + 128) * 2
    base = bench.algorithmic_work(cs.CSA_DECODE)
    assert {k: v for k, v in w.items() if k != "append_bytes"} == base
    runner_stages = ["append", "index", "attend"]
    assert bench.LayerRunner.stages(type("R", (), {"spec": s})()) == runner_stages


def test_oracle_sample_run_includes_the_update():
    spec = _small_step("csa")
    dt = bench.oracle_sample_run(spec, [0])
    assert dt > 0


def test_append_window_reach_invariants():
    """The facts the cache-update kernel's layout rests on, over many calls: entries that
    close in a call at pos0 are j0 = pos0 // m onwards; each window ends inside the call's
    rows and starts no earlier than pos0 - L + 1 (so a ring of L rows holds every earlier
    row it needs); and from the third closing entry on a window starts at or after pos0
    (so only the first chunk of entries reads the ring)."""
    rng = np.random.default_rng(5)
    for _ in range(20000):
        m = int(rng.integers(1, 160))
        overlap = int(rng.integers(0, 2))
        L = (1 + overlap) * m
        pos0 = int(rng.integers(0, 10 * m + 50))
        n_new = int(rng.integers(1, 4 * L + 3))
        j0 = pos0 // m
        n_close = (pos0 + n_new) // m - j0
        closing = [j for j in range(j0 - 2, (pos0 + n_new) // m + 2)
                   if pos0 <= (j + 1) * m - 1 < pos0 + n_new]
        assert closing == list(range(j0, j0 + n_close))
        for c, j in enumerate(closing):
            lo = max(0, (j - overlap) * m)
            hi = (j + 1) * m
            assert hi <= pos0 + n_new
            assert lo >= pos0 - L + 1
            if c >= 2:
                assert lo >= pos0
