"""Benchmark: DeepSeek-V4 CSA/HCA attention layer on B200 through the C ABI.

One step = the whole hot path over one batch of seeded synthetic input already resident
in HBM: KV Compressor -> Lightning Indexer + top-k -> sparse sink attention (for the CSA
prefill workload: csa_compress, csa_index_topk, csa_attend).  Default workload: the CSA
prefill layer at V4-Flash head shape (B=1, S=8192, H=64, D=512, rope 64, window 128,
m=4, 2048 entries, H_I=64, d_I=128, top-k 512).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 0..6] [--impl reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own independent layer
instance (its own seeded sequence), no data-path collective; value = all ranks' tokens
over the max-over-ranks device time (weak scaling).  --impl reference times the fp64 CPU
oracle on the host cores instead (rank 0 only), on a bounded sample of query rows.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA/HCA layer tokens/s (prefill, decode) on 1 B200; % of HBM / bf16 TC roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- work model
def n_vis(t, m, P):
    return min(P, (t + 1) // m) if t >= 0 else 0


def n_win(spec, t):
    lo = max(t - spec.W + 1, spec.kv_pos0)
    hi = min(t, spec.kv_pos0 + spec.S_kv - 1)
    return max(0, hi - lo + 1)


def algorithmic_work(spec):
    """Per-stage algorithmic work of one layer call (the definitions' counts):
    compress bytes = kv + gate read + pool written; indexer FLOPs = sum_t 2 H_I d_I n_vis(t);
    attention FLOPs = sum_t 4 H D |K_t|; attention HBM bytes = q read + out written +
    each distinct kv/pool row once."""
    e = 4 if spec.dtype == "f32" else 2
    w = {}
    if not spec.decode and spec.kind != "sliding":
        w["compress_bytes"] = spec.B * (2 * spec.S_kv * spec.D + spec.P * spec.D) * e
    keys = 0
    idx_flops = 0
    for i in range(spec.S_q):
        t = spec.q_pos0 + i
        nv = n_vis(t, spec.m, spec.P)
        ne = min(spec.topk, nv) if spec.kind == "csa" else (nv if spec.kind == "hca" else 0)
        keys += n_win(spec, t) + ne
        if spec.kind == "csa":
            idx_flops += 2 * spec.H_I * spec.d_I * nv
    w["attend_flops"] = 4 * spec.B * spec.H * spec.D * keys
    w["index_flops"] = spec.B * idx_flops
    # distinct rows an attention call must read: every window row it touches, and at most
    # min(P, S_q*k) (CSA) / P (HCA) entries
    ent_rows = min(spec.P, spec.S_q * spec.topk) if spec.kind == "csa" else spec.P
    win_rows = min(spec.S_kv, spec.S_q + spec.W - 1)
    w["attend_bytes"] = spec.B * (2 * spec.S_q * spec.H * spec.D + (win_rows + ent_rows) * spec.D) * e
    if spec.kind == "csa":
        w["index_bytes"] = spec.B * (spec.S_q * spec.H_I * (spec.d_I + 1) + spec.P * spec.d_I) * e \
            + spec.B * spec.S_q * spec.topk * 4
    if spec.pool_index_keys:
        w["compress_I_bytes"] = spec.B * (2 * spec.S_kv * spec.d_I + spec.P * spec.d_I) * e
    if spec.index_rope:
        # every indexer query head and every pooled key read and written once
        w["rope_I_bytes"] = 2 * spec.B * (spec.S_q * spec.H_I + spec.P) * spec.d_I * e
    if spec.proj:
        import csa_synth as cs
        M = spec.B * spec.S_q
        w["proj_in_flops"] = 2 * M * cs.PROJ_HIDDEN * 2 * spec.D
        w["proj_out_flops"] = 2 * M * (spec.H * spec.D * cs.PROJ_RANK
                                       + cs.PROJ_GROUPS * cs.PROJ_RANK * cs.PROJ_HIDDEN)
    if spec.cache_update:
        # per compressor (main at D, indexer keys at d_I): the new rows read and stored in the
        # state (kv + gate), the state rows a closing window reaches back to read (kv + gate),
        # each closed entry written
        n_close = (spec.q_pos0 + spec.S_q) // spec.m - spec.q_pos0 // spec.m
        back = spec.q_pos0 - max(0, (spec.q_pos0 // spec.m - spec.overlap) * spec.m) if n_close else 0
        rows = 4 * spec.S_q + 2 * back + n_close
        w["append_bytes"] = spec.B * rows * (spec.D + (spec.d_I if spec.kind == "csa" else 0)) * e
    return w


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", "csa_clocks_%d_%d.csv" % (os.getpid(), gpu_index))

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu),
                                          "--query-gpu=" + self.FIELDS, "--format=csv,noheader",
                                          "-lms", "20"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sms, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 9:
                    continue
                try:
                    sms.append(float(p[1].split()[0]))
                    maxs.append(float(p[2].split()[0]))
                except ValueError:
                    continue
                for n, v in zip(names, p[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sms:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = sorted(sms)[len(sms) // 4:] or sms  # drop idle-edge samples
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(maxs),
                "samples": len(sms), "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- GPU arm
def workload_specs(workload: int):
    import csa_synth as cs
    return cs.WORKLOADS[workload]


def rank_spec(spec, rank):
    """Rank r runs its own independent layer instance: same shape, its own seeded inputs."""
    return dataclasses.replace(spec, workload=spec.workload + 10 * rank) if rank else spec


def max_over_ranks(ms: float, world: int, device) -> float:
    """Device time of the slowest rank (one all-reduce of a scalar; no data-path traffic)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class LayerRunner:
    """Holds one layer's device inputs/outputs and runs it through the C ABI."""

    def __init__(self, spec, device):
        import torch
        import csa_synth as cs
        import sparse_attention_14_b200 as csa
        self.csa, self.torch, self.spec = csa, torch, spec
        self.inp = cs.make_inputs(spec, device=device)
        s = spec
        dt = s.torch_dtype
        self.pool = self.inp["pool"] if s.decode else (
            torch.empty((s.B, s.P, s.D), dtype=dt, device=device) if s.kind != "sliding" else None)
        self.idx = torch.empty((s.B, s.S_q, s.topk), dtype=torch.int32, device=device) \
            if s.kind == "csa" else None
        self.out = torch.empty_like(self.inp["q"])
        self.k_I = torch.empty((s.B, s.P, s.d_I), dtype=dt, device=device) \
            if s.pool_index_keys else self.inp["k_I"]
        self.q_I = torch.empty_like(self.inp["q_I"]) if s.index_rope else self.inp["q_I"]
        self.k_I_rot = torch.empty_like(self.k_I) if s.index_rope else self.k_I
        wsi = csa.csa_index_topk_workspace_bytes(s.B, s.S_q, s.q_pos0, s.P, s.H_I, s.d_I, s.m,
                                                 s.topk, dt) \
            if s.kind == "csa" else 0
        wsa = csa.csa_attend_workspace_bytes(0 if s.kind == "csa" else 1, s.B, s.S_q, s.S_kv, s.P,
                                             s.H, s.D, s.topk, dt)
        self.ws_i = torch.empty(max(wsi, 1), dtype=torch.uint8, device=device) if wsi else None
        self.ws_a = torch.empty(max(wsa, 1), dtype=torch.uint8, device=device) if wsa else None
        self.kv = self.inp["kv"]
        self.gate = self.inp["gate"]
        self.y = None
        if s.proj:
            import csa_synth as cs
            self.kv = torch.empty((s.B, s.S_kv, s.D), dtype=dt, device=device)
            self.gate = torch.empty_like(self.kv)
            self.y = torch.empty((s.B, s.S_q, cs.PROJ_HIDDEN), dtype=dt, device=device)
            wso = csa.csa_out_proj_workspace_bytes(s.B * s.S_q, cs.PROJ_GROUPS, cs.PROJ_RANK)
            self.ws_o = torch.empty(wso, dtype=torch.uint8, device=device)

    @property
    def result(self):
        """The step's output: y after the output projection, else the attention output."""
        return self.y if self.y is not None else self.out

    def stages(self):
        s = self.spec
        st = []
        if s.proj:
            st.append("proj_in")
        if not s.decode and s.kind != "sliding":
            st.append("compress")
        if s.pool_index_keys:
            st.append("compress_I")
        if s.index_rope:
            st.append("rope_I")
        if s.cache_update:
            st.append("append")
        if s.kind == "csa":
            st.append("index")
        st.append("attend")
        if s.proj:
            st.append("proj_out")
        return st

    def run_stage(self, name):
        s, i, csa = self.spec, self.inp, self.csa
        if name == "proj_in":
            csa.csa_kv_gate_proj(i["x"], i["w_kv"], i["w_gate"], i["kv_norm_w"], 1e-6, kv=self.kv,
                                 gate=self.gate)
        elif name == "proj_out":
            csa.csa_out_proj(self.out, i["w_a"], i["w_b"], y=self.y, workspace=self.ws_o)
        elif name == "compress":
            csa.csa_compress(self.kv, self.gate, s.m, s.overlap, pool=self.pool)
        elif name == "compress_I":
            csa.csa_compress(i["kI_tok"], i["gI_tok"], s.m, s.overlap, pool=self.k_I)
        elif name == "rope_I":
            csa.csa_rope_rows(i["q_I"], s.q_pos0, s.H_I, s.S_q, 1, s.index_rope, s.base, out=self.q_I)
            csa.csa_rope_rows(self.k_I, 0, 1, s.P, s.m, s.index_rope, s.base, out=self.k_I_rot)
        elif name == "append":
            import csa_synth as cs
            csa.csa_compress_append(cs.kv_new(s, i), i["gate_new"], i["state"], s.q_pos0, s.m,
                                    s.overlap, pool=self.pool)
            if s.kind == "csa":
                csa.csa_compress_append(i["kI_new"], i["gI_new"], i["state_I"], s.q_pos0, s.m,
                                        s.overlap, pool=i["k_I"])
        elif name == "index":
            csa.csa_index_topk(self.q_I, i["w"], self.k_I_rot, s.q_pos0, s.m, s.topk, idx=self.idx,
                               workspace=self.ws_i)
        elif s.kind == "csa":
            csa.csa_attend(i["q"], self.kv, s.kv_pos0, self.pool, self.idx, i["sink"], s.q_pos0, s.R,
                           s.base, s.W, s.m, s.scale, out=self.out, workspace=self.ws_a)
        else:
            csa.hca_attend(i["q"], self.kv, s.kv_pos0, self.pool if s.kind == "hca" else None,
                           i["sink"], s.q_pos0, s.R, s.base, s.W, s.m, s.scale, out=self.out,
                           workspace=self.ws_a)


def src_hash(names):
    h = hashlib.sha256()
    for n in names:
        p = os.path.join(ROOT, "sparse_attention_14_b200", "csrc", n)
        if os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


STAGE_SOURCES = {"compress": ["compress.cu", "common.cuh"],
                 "append": ["compress.cu", "common.cuh"],
                 "compress_I": ["compress.cu", "common.cuh"],
                 "rope_I": ["rope.cu", "common.cuh"],
                 "index": ["index_topk.cu", "topk.cuh", "index_tc.cu", "umma.cuh", "common.cuh"],
                 "attend": ["attend.cu", "attend_tc.cu", "umma.cuh", "common.cuh"],
                 "proj_in": ["proj_tc.cu", "umma.cuh", "common.cuh"],
                 "proj_out": ["proj_tc.cu", "umma.cuh", "common.cuh"]}


def ncu_traffic(stage, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current
    source of that kernel (else None)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get("workload%d" % workload, {}).get(stage)
    if not e or e.get("src_sha") != src_hash(STAGE_SOURCES[stage]):
        return None
    return e.get("dram_bytes_per_launch")


def gpu_arm(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import sparse_attention_14_b200 as csa

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    specs = [rank_spec(s, rank) for s in workload_specs(args.workload)]
    csa.load_library()
    stream = torch.cuda.current_stream()

    # mixed stack: allocate per layer inside the step would time allocation; instead keep
    # every layer resident when it fits, else run layers one at a time (generated per layer)
    runners = [LayerRunner(s, dev) for s in specs]
    tokens_per_step = sum(s.B * s.S_q for s in specs[:1])  # the block processes S tokens once
    stage_names = [(li, st) for li, r in enumerate(runners) for st in r.stages()]

    for _ in range(args.warmup):
        for li, st in stage_names:
            runners[li].run_stage(st)
    torch.cuda.synchronize()

    # The timed region is one CUDA graph holding all K steps (the library only enqueues work
    # on the current stream, so its calls are capturable): no host launch gaps between
    # kernels.  A second graph of the same K steps records timing events around every stage;
    # it is replayed after the timed region and gives the per-stage times (event nodes
    # between kernels add their own time, ~4 us per decode step, so they stay out of the
    # timed graph).  Fallbacks: one graph per stage replayed with events between them, then
    # eager launches.
    ev = {k: [(torch.cuda.Event(enable_timing=True, external=True),
               torch.cuda.Event(enable_timing=True, external=True))
              for _ in range(args.steps)] for k in stage_names}
    whole = None
    graphs = None
    launches_per_step = None
    launch_mode = "eager"
    if not args.eager:
        try:
            l0 = csa.launch_count()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for k in range(args.steps):
                    for key in stage_names:
                        runners[key[0]].run_stage(key[1])
            launches_per_step = (csa.launch_count() - l0) // args.steps
            gi = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gi):
                for k in range(args.steps):
                    for key in stage_names:
                        ev[key][k][0].record()
                        runners[key[0]].run_stage(key[1])
                        ev[key][k][1].record()
            torch.cuda.synchronize()
            g.replay()   # one untimed replay of each: first-launch costs of the graphs themselves
            gi.replay()
            torch.cuda.synchronize()
            whole = g
            launch_mode = ("one CUDA graph for the K timed steps; per-stage times from a second, "
                           "event-instrumented graph of the same steps replayed after it")
        except Exception as exc:  # pragma: no cover - falls back to per-stage graphs
            print("whole-run graph capture failed (%s); trying per-stage graphs" % exc, file=sys.stderr)
            whole = None
            torch.cuda.synchronize()
            ev = {k: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                      for _ in range(args.steps)] for k in stage_names}
            try:
                l0 = csa.launch_count()
                graphs = {}
                for key in stage_names:
                    gs = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(gs):
                        runners[key[0]].run_stage(key[1])
                    graphs[key] = gs
                launches_per_step = csa.launch_count() - l0
                torch.cuda.synchronize()
                launch_mode = "CUDA graph per stage"
            except Exception as exc2:  # pragma: no cover - falls back to eager launches
                print("graph capture failed (%s); timing eager launches" % exc2, file=sys.stderr)
                graphs = None
                torch.cuda.synchronize()

    def step(events=None):
        for key in stage_names:
            if events is not None:
                events[key][0].record(stream)
            if graphs is not None:
                graphs[key].replay()
            else:
                runners[key[0]].run_stage(key[1])
            if events is not None:
                events[key][1].record(stream)

    if whole is None:
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    launches0 = csa.launch_count()
    clk = ClockSampler(local_rank)
    clk.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0.record(stream)
    if whole is not None:
        whole.replay()
    else:
        for k in range(args.steps):
            step({key: ev[key][k] for key in stage_names})
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = clk.stop()
    if whole is not None:
        gi.replay()   # the instrumented copy: per-stage device times
        torch.cuda.synchronize()
    launches = csa.launch_count() - launches0
    if launches_per_step is not None:
        launches = launches_per_step * args.steps
    ms_total = max_over_ranks(t0.elapsed_time(t1), world, dev)
    ms_step = ms_total / args.steps
    stage_ms = {"%d:%s" % key: sum(a.elapsed_time(b) for a, b in ev[key]) / args.steps
                for key in stage_names}

    # end to end through the public API with host buffers: pinned inputs copied in, the
    # layer run, the output copied back, every step
    e2e = None
    if not args.no_e2e:
        e2e = e2e_arm(args, runners, stage_names, stream, world, dev)

    if rank != 0:
        return None
    peaks, peak_kind = load_peaks()
    spec0 = specs[0]
    work = [algorithmic_work(s) for s in specs]
    # dominant kernel = the stage with the largest device time
    (dom_layer, dom_stage), dom_ms = max(((k, stage_ms["%d:%s" % k]) for k in stage_names),
                                         key=lambda x: x[1])
    wk = work[dom_layer]
    dom_spec = specs[dom_layer]
    if dom_stage in ("compress", "append", "compress_I", "rope_I") \
            or (dom_stage == "attend" and (dom_spec.kind == "sliding" or dom_spec.decode)) \
            or (dom_stage == "index" and dom_spec.decode):
        key_b = {"compress": "compress_bytes", "attend": "attend_bytes", "index": "index_bytes",
                 "append": "append_bytes", "compress_I": "compress_I_bytes",
                 "rope_I": "rope_I_bytes"}[dom_stage]
        achieved = wk[key_b] / (dom_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "algorithmic_bytes_per_launch": wk[key_b]}
    else:
        key_f = {"attend": "attend_flops", "index": "index_flops", "proj_in": "proj_in_flops",
                 "proj_out": "proj_out_flops"}[dom_stage]
        achieved = wk[key_f] / (dom_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                "algorithmic_flops_per_launch": wk[key_f]}
    roof.update({"kernel": "%s (layer %d)" % (dom_stage, dom_layer),
                 "kernel_ms": round(dom_ms, 4), "peak_source": peak_kind + " (burst)",
                 "traffic": ncu_traffic(dom_stage, args.workload)})
    tokens = tokens_per_step * world
    value = tokens / (ms_step * 1e-3)
    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32" if spec0.dtype == "f32" else "bf16",
        "data": "synthetic (seeded N(0,1) q/kv/gate/q_I/k_I, w/sqrt(H_I), RMS-normalised kv)",
        "config": workload_config(args.workload, specs),
        "l2": "inputs larger than L2 (q/out/q_I > 126 MB per step); no flush",
        "launch": launch_mode,
        "stages_ms": {k: round(v, 4) for k, v in stage_ms.items()},
        "roofline": roof,
        "gpu_launches": int(launches),
        "clocks": clocks,
        "e2e": e2e,
    }
    return line


def workload_name(w, specs):
    return {0: "tiny CSA layer fp32 (S=256)", 1: "CSA prefill bf16 S=8192 (V4-Flash layer shape)",
            2: "HCA prefill bf16 S=65536", 3: "CSA decode bf16 B=64 at 65536 cached tokens",
            4: "mixed 4-layer stack bf16 S=131072",
            5: "CSA decode step with compressor cache update, bf16 B=64 at 65536 tokens",
            6: "CSA prefill bf16 S=8192 with the indexer key path (pooled index keys, indexer RoPE 64)",
            7: "CSA prefill bf16 S=8192 with its projections (kv/gate from hidden 4096, grouped "
               "output projection 8 groups x 1024 -> 4096)"}[w]


def workload_config(w, specs):
    """The workload part of the JSON line's config, shared by both arms."""
    spec0 = specs[0]
    return {"workload": workload_name(w, specs), "B": spec0.B, "S": spec0.S_q, "H": spec0.H,
            "D": spec0.D, "rope_dim": spec0.R, "window": spec0.W, "layers": [s.kind for s in specs],
            "m": [s.m for s in specs], "P": [s.P for s in specs], "topk": spec0.topk,
            "H_I": spec0.H_I, "d_I": spec0.d_I, "index_rope": spec0.index_rope,
            "parallelism": "independent layer instance per GPU"}


def e2e_arm(args, runners, stage_names, stream, world, dev):
    import torch
    import torch.distributed as dist
    host = []
    h2d = d2h = 0
    for r in runners:
        pairs = []
        for k, v in r.inp.items():
            if v is None:
                continue
            hv = torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
            hv.copy_(v)
            pairs.append((hv, v))
            h2d += v.numel() * v.element_size()
        ho = torch.empty(r.result.shape, dtype=r.result.dtype, pin_memory=True)
        d2h += r.result.numel() * r.result.element_size()
        host.append((pairs, ho))
    steps = max(1, min(args.steps, 5))

    def one():
        for (pairs, ho), r in zip(host, runners):
            for hv, dv in pairs:
                dv.copy_(hv, non_blocking=True)
        for li, st in stage_names:
            runners[li].run_stage(st)
        for (pairs, ho), r in zip(host, runners):
            ho.copy_(r.result, non_blocking=True)

    one()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        one()
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b) / steps, world, dev)
    tokens = runners[0].spec.B * runners[0].spec.S_q * world
    return {"value": round(tokens / (ms * 1e-3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 3),
            "steps": steps}


# ----------------------------------------------------------------------------- sharded prefill
def sharded_arm(args, rank, world, local_rank):
    """One CSA prefill sequence split over the ranks by query rows (zig-zag chunks), each
    rank pooling its share of the entries, one all-gather of the entries and one of the
    index keys (NCCL), then the indexer and attention on its own rows.  Total work is fixed
    (strong scaling); each step is timed on the device, max over ranks."""
    import torch
    import csa_synth as cs
    import sparse_attention_14_b200 as csa
    from sparse_attention_14_b200 import shard
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    spec = workload_specs(args.workload)[0]
    if spec.kind != "csa" or spec.decode or spec.proj or spec.pool_index_keys or len(workload_specs(args.workload)) > 1:
        raise SystemExit("--shard needs a single-layer CSA prefill workload (1)")
    csa.load_library()
    inp = cs.make_inputs(spec, device=dev)   # the same seeded sequence on every rank
    be = shard.LibraryBackend()
    for _ in range(args.warmup):
        shard.prefill_sharded(be, world, rank, inp, spec)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    l0 = csa.launch_count()
    clk = ClockSampler(local_rank)
    clk.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    t0.record()
    for _ in range(args.steps):
        shard.prefill_sharded(be, world, rank, inp, spec)
    t1.record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = clk.stop()
    launches = csa.launch_count() - l0
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev) / args.steps
    if rank != 0:
        return None
    cfg = dict(workload_config(args.workload, [spec]),
               parallelism="query-row shards (zig-zag) + NCCL all-gather of pool and k_I")
    return {"metric": METRIC, "value": round(spec.B * spec.S_q / (ms * 1e-3), 1), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded, the same sequence on every rank)", "config": cfg,
            "launch": "eager (collectives between the phases)", "gpu_launches": int(launches),
            "clocks": clocks, "roofline": None, "e2e": None}


# ----------------------------------------------------------------------------- CPU oracle
def oracle_sample_run(spec, rows, inp_cpu=None):
    """The fp64 oracle over the whole hot path for the given query rows (the compressor
    runs in full: every sampled row may attend to any entry).  Returns seconds."""
    import numpy as np
    import csa_synth as cs
    import oracle
    inp = cs.make_inputs(spec, device="cpu") if inp_cpu is None else inp_cpu
    f64 = lambda t: None if t is None else t.double().numpy()
    t0 = time.perf_counter()
    pool = None
    kv, gate = f64(inp["kv"]), f64(inp["gate"])
    if spec.proj:
        kv, gate = oracle.kv_gate_proj(f64(inp["x"]), f64(inp["w_kv"]), f64(inp["w_gate"]),
                                       f64(inp["kv_norm_w"]), 1e-6)
    k_I = oracle.compress(f64(inp["kI_tok"]), f64(inp["gI_tok"]), spec.m, spec.overlap) \
        if spec.pool_index_keys else f64(inp["k_I"])
    if spec.decode:
        pool = f64(inp["pool"])
        if spec.cache_update:
            j0 = spec.q_pos0 // spec.m
            comps = [(inp["state"], cs.kv_new(spec, inp), inp["gate_new"], pool)]
            if spec.kind == "csa":
                comps.append((inp["state_I"], inp["kI_new"], inp["gI_new"], k_I))
            for state, new_kv, new_g, cache in comps:
                kh, gh, s0 = cs.ring_history(state, spec.q_pos0, spec.m, spec.overlap)
                st = oracle.CompressorState.resume(f64(kh), f64(gh), s0, spec.m, spec.overlap)
                ent = st.append(f64(new_kv), f64(new_g))
                cache[:, j0:j0 + ent.shape[1]] = ent
    elif spec.kind != "sliding":
        pool = oracle.compress(kv, gate, spec.m, spec.overlap)
    tpos = np.asarray(rows, dtype=np.int64) + spec.q_pos0
    idx = None
    if spec.kind == "csa":
        if spec.index_rope:
            sc = oracle.index_scores_rope(f64(inp["q_I"][:, rows]), f64(inp["w"][:, rows]), k_I, tpos,
                                          spec.m, spec.index_rope, spec.base)
        else:
            sc = oracle.index_scores(f64(inp["q_I"][:, rows]), f64(inp["w"][:, rows]), k_I, tpos, spec.m)
        idx, _ = oracle.topk(sc, tpos, spec.m, spec.topk)
    o = oracle.attend(f64(inp["q"][:, rows]), tpos, kv, spec.kv_pos0, pool, spec.m, idx,
                      f64(inp["sink"]), spec.R, spec.base, spec.W, spec.scale,
                      "csa" if spec.kind == "csa" else "hca")
    if spec.proj:
        oracle.grouped_out_proj(o, f64(inp["w_a"]), f64(inp["w_b"]))
    return time.perf_counter() - t0


def compressor_note(spec):
    """How the sampled oracle run treats the compressor, for the sample description."""
    if spec.decode:
        return "cache update in full" if spec.cache_update else "resident pool (no compressor)"
    if spec.proj:
        return "kv/gate projections and compressor in full, output projection on the sampled rows"
    return "no compressor" if spec.kind == "sliding" else "compressor in full"


def oracle_rows(spec, n):
    # evenly spaced query rows: the same causal mix of window/entry counts as the workload
    S = spec.S_q
    n = min(n, S)
    return sorted({min(S - 1, int((k + 0.5) * S / n)) for k in range(n)})


def oracle_threads():
    v = os.environ.get("OMP_NUM_THREADS")
    return int(v) if v else (len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count())


def cpu_baseline(args):
    spec = workload_specs(args.workload)[0]
    if spec.B * spec.S_q * spec.D * spec.H > 4e9:
        spec = dataclasses.replace(spec)  # inputs generated per call below, bounded by rows
    import csa_synth as cs
    inp = cs.make_inputs(spec, device="cpu")
    rows = oracle_rows(spec, 16)
    dt = oracle_sample_run(spec, rows, inp)
    # size the sample to about 15 s of CPU work
    n = max(16, min(spec.S_q, int(16 * 15.0 / max(dt, 1e-3))))
    rows = oracle_rows(spec, n)
    dt = oracle_sample_run(spec, rows, inp)
    units = spec.B * len(rows)
    return {"value": round(units / dt, 3), "unit": "tokens/s", "cores": oracle_threads(),
            "kind": "oracle",
            "sample": "%d of %d query rows (evenly spaced) x B=%d of %s; %s; %.1f s"
                      % (len(rows), spec.S_q, spec.B, spec.name, compressor_note(spec), dt)}


def reference_arm(args, rank, world):
    if rank != 0:
        return None
    import csa_synth as cs
    spec = workload_specs(args.workload)[0]
    inp = cs.make_inputs(spec, device="cpu")
    rows = oracle_rows(spec, 16)
    dt = oracle_sample_run(spec, rows, inp)
    n = max(8, min(spec.S_q, int(16 * 6.0 / max(dt, 1e-3))))  # ~6 s per step
    rows = oracle_rows(spec, n)
    for _ in range(args.warmup):
        oracle_sample_run(spec, rows, inp)
    t = [oracle_sample_run(spec, rows, inp) for _ in range(args.steps)]
    ms = 1e3 * sum(t) / len(t)
    units = spec.B * len(rows)
    value = units / (ms * 1e-3)
    sample = "%d of %d query rows (evenly spaced) x B=%d of %s per step; %s" % (
        len(rows), spec.S_q, spec.B, spec.name, compressor_note(spec))
    return {"metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": workload_config(args.workload, workload_specs(args.workload)),
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s",
                             "cores": oracle_threads(), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- main
def _free_port() -> int:
    import socket
    sk = socket.socket()
    sk.bind(("127.0.0.1", 0))
    port = sk.getsockname()[1]
    sk.close()
    return port


def launch_ranks(n: int, limit_s: int = 1800) -> int:
    """`bench.py --gpus N` run without a launcher: re-run this command under
    torch.distributed.run with one rank per GPU (rendezvous on 127.0.0.1), bounded by
    `timeout`.  Returns the launcher's exit code; rank 0 prints the JSON line."""
    cmd = ["timeout", "-k", "60", str(limit_s), sys.executable, "-m", "torch.distributed.run",
           "--nnodes=1", "--nproc-per-node=%d" % n, "--master-addr", "127.0.0.1",
           "--master-port", str(_free_port()), os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=1, choices=[0, 1, 2, 3, 4, 5, 6, 7])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time eager launches instead of CUDA graphs")
    ap.add_argument("--shard", action="store_true",
                    help="split one CSA prefill sequence over the ranks by query rows (strong scaling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(launch_ranks(args.gpus))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = reference_arm(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        if args.shard:
            line = sharded_arm(args, rank, world, local_rank)
            if line is not None:
                print(json.dumps(line), flush=True)
            return
        line = gpu_arm(args, rank, world, local_rank)
        if line is not None:
            if world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline(args)
            else:
                line["cpu_baseline"] = None
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
