"""StagQ batch-one GEMV benchmark on B200.

Workload (one step): one Llama-3.1-8B layer's linears (q/k/v/o, gate/up, down;
out x in as in the model), synthetic weights, group 128, base + 2 refinement
planes, 0.5 % side record, x fp16 N(0,1), batch 1, at 2, then 3, then 4 bits.
Per precision the layer runs as a decode runs it: q/k/v in one launch (one
stacked handle: they share x), o, gate/up in one launch, down -- 4 launches,
12 per step, 21 GEMVs. Each precision pass reads its own device copy of the
layer, and a copy is read again only after at least 4x the L2 size of other
reads, so every byte comes from HBM. Every step is one CUDA-graph replay.

Prints one JSON line. ``value`` is the whole job's algorithmic HBM traffic
(planes read at the chosen precision + pairs + side record + x + y) divided by
device time, in GB/s. Per-launch microseconds for every launch and precision
are in ``per_launch``.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl stagq|reference]
                  [--workload llama31_8b_linears_b1 | phi4_olmo2_linears_b1 | precision_sweep |
                              llama31_8b_stack | llama31_8b_guarded | cublas_context]

The default workload is the Llama-3.1-8B layer above. The others print one
JSON line each with per-GEMV (or per-token) times:
  phi4_olmo2_linears_b1  Phi-4 and OLMo-2-7B linears at 2/3/4 bits, batch 1,
                         each alone and as one layer's chain (q k v o gate up
                         down, one CUDA graph);
  cublas_context         dense fp16 torch.mv (cuBLAS) on the Llama-3.1-8B shapes
                         beside the StagQ GEMVs: the speedups of the paper's
                         Table 5, as context;
  llama31_8b_guarded     the Llama-3.1-8B linears at group 32 with the paper's
                         side-record guards (ratio T = 4 + post-grid), each
                         alone and as a layer chain;
  precision_sweep        14336x4096 and 4096x14336 with base + 4 planes, read at
                         2..6 bits, group 16, 32, 64 and 128, side record
                         0 / 0.1 / 1 %;
  llama31_8b_stack       32 layers x 7 linears (6.98e9 weights) resident on the
                         GPU, per-token GEMV time at batch 1 and 4, 2/3/4 bits
                         read from one stored stream.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "batch-1 GEMV µs and achieved HBM GB/s (% of roofline) at 2/3/4 bits"
WORKLOAD = "llama31_8b_linears_b1"
BITS = (2, 3, 4)
GROUP, N_PLANES, DENSITY = 128, 2, 0.005
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ["quantized_gemv_stagq_b200/csrc/gemv.cu", "quantized_gemv_stagq_b200/csrc/gemv1.cu",
                  "quantized_gemv_stagq_b200/csrc/kernel_common.cuh", "quantized_gemv_stagq_b200/csrc/layout.cuh"]
SINGLE_MAX_IN = 15 * 2048  # up to this many columns, n = 1 runs the single-vector kernel (gemv1)


def _args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="stagq", choices=["stagq", "reference"])
    p.add_argument("--copies", type=int, default=6, help="least device copies of the layer rotated over")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--workload", default=WORKLOAD,
                   choices=[WORKLOAD, "phi4_olmo2_linears_b1", "precision_sweep", "llama31_8b_stack",
                            "llama31_8b_guarded", "cublas_context"])
    p.add_argument("--stack-distinct", type=int, default=4,
                   help="llama31_8b_stack: distinct encoded layers (the 32 resident layers cycle over them)")
    return p.parse_args()


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _kernel_hash():
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _ncu_traffic():
    """dram bytes per launch of the dominant kernel from the committed ncu
    summary, if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "gemv_dram_traffic.txt")
    try:
        kv = {}
        for line in open(path):
            if line.strip() and not line.startswith("#") and " " in line:
                k, v = line.split(None, 1)
                kv[k] = v.strip()
        if kv.get("kernel_source_sha256_16") != _kernel_hash():
            return None, None
        return float(kv["dram_bytes_per_launch_full"]), kv.get("kernel", "")
    except Exception:
        return None, None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [t.strip() for t in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


def _launch_kernel(key):
    """Name of the kernel that serves the step launch `name@pM` at n = 1."""
    from quantized_gemv_stagq_b200 import synth
    members = dict(LAYER_LAUNCHES)[key.split("@")[0]]
    return "gemv1_kernel" if synth.LLAMA31_8B_LINEARS[members[0]][1] <= SINGLE_MAX_IN else "gemv_kernel"


def _layer_shapes():
    from quantized_gemv_stagq_b200 import synth
    return list(synth.LLAMA31_8B_LINEARS.items())


# ------------------------------------------------------------------ reference arm

class OracleSample:
    """The oracle's GEMV (decode + fp64 dot) of the q_proj shape at 2/3/4 bits:
    the CPU statement of one precision sweep of the hot path."""

    def __init__(self):
        from oracle import stagq as O
        from quantized_gemv_stagq_b200 import synth
        self.O = O
        self.out, self.inp = synth.LLAMA31_8B_LINEARS["q_proj"]
        W = synth.weights(self.out, self.inp, seed=11)
        self.F = O.encode(W, GROUP, N_PLANES, DENSITY, "fast")
        self.x = synth.activations(1, self.inp, seed=12)
        try:
            from threadpoolctl import threadpool_info
            self.threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
        except Exception:
            self.threads = os.cpu_count() or 1

    def one(self, b):
        """One GEMV at b bits; returns (bytes, seconds)."""
        t0 = time.perf_counter()
        self.O.gemv(self.F, b, self.x)
        return self.O.model_bytes(self.out, self.inp, GROUP, self.F.nnz, b), time.perf_counter() - t0

    def text(self, n):
        return (f"oracle GEMV (decode + fp64 dot) of q_proj {self.out}x{self.inp}, {n} call(s) cycling "
                f"p2/p3/p4")


def cpu_oracle_sample(target_s: float = 12.0):
    """Bounded CPU baseline: rounds of OracleSample until ~target_s."""
    S = OracleSample()
    nb, el, n = 0, 0.0, 0
    while el < target_s or n % len(BITS):
        b, t = S.one(BITS[n % len(BITS)])
        nb, el, n = nb + b, el + t, n + 1
    return nb / el / 1e9, el, S.text(n), S.threads


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    S = OracleSample()
    for w in range(args.warmup):
        S.one(BITS[w % len(BITS)])
    nb, el = 0, 0.0
    for k in range(args.steps):       # a step: one oracle GEMV, precisions cycling
        b, t = S.one(BITS[k % len(BITS)])
        nb, el = nb + b, el + t
    value = nb / el / 1e9
    sample = S.text(args.steps)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * el / max(args.steps, 1), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD, "sample": sample, "group": GROUP,
                                        "n_planes": N_PLANES, "side_record_density": DENSITY, "batch": 1},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": S.threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm

def time_gemv(Q, torch, mats, bits, x, y, n, stream, reps=24, repeats=5):
    """Device time of one GEMV (µs): a CUDA graph of `reps` launches rotating
    over the device copies in `mats` (so reads come from HBM), replayed
    `repeats` times between CUDA events; median over 10 such measurements."""
    C = len(mats)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        Q.stagq_gemv_n(mats[0], bits, x, n, y, stream=stream)
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=stream):
        for r in range(reps):
            Q.stagq_gemv_n(mats[(r + 1) % C], bits, x, n, y, stream=stream)
    g.replay()
    torch.cuda.synchronize()
    us = _median_event_us(torch, stream, lambda: [g.replay() for _ in range(repeats)], 10) / (repeats * reps)
    del g
    return us


def job_ms(ms: float, dist=None, device: str = "cuda") -> float:
    """The job's device time: the max over ranks of each replica's CUDA-event
    time (ms), taken by an all-reduce on `device` (a GPU tensor for NCCL, the
    CPU for gloo); the local time without a process group."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, step_bytes: int, steps: int, ms: float) -> float:
    """Whole-job throughput in GB/s: every replica moves step_bytes per step
    (weak scaling), over the job's time."""
    return world * step_bytes * steps / (ms * 1e-3) / 1e9


def copies_for(Q, stored_bytes, l2, minimum=3):
    """Device copies so that one pass over them is at least 4x the L2 size."""
    return max(minimum, int(4 * l2 // max(stored_bytes, 1)) + 1)


def _extra_line(args, workload, results, extra_cfg, clocks, peak, peak_kind, value, unit, gemvs):
    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": 1, "steps": None, "warmup": None,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int32 dot (u8 codes x i16 x) + fp32", "data": "synthetic",
        "config": dict({"workload": workload}, **extra_cfg), "results": results,
        "peak": {"hbm_gbs": peak, "kind": peak_kind}, "gpu_launches": gemvs, "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def run_extra(args):
    """The other measured workloads (one JSON line each)."""
    import torch
    import quantized_gemv_stagq_b200 as Q
    from quantized_gemv_stagq_b200 import synth
    torch.cuda.set_device(0)
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    peak, peak_kind = _peaks()
    stream = torch.cuda.Stream()
    clocks = ClockSampler(0)
    clocks.start()
    results = {}
    launches = 0

    def per_gemv(shapes, bits_list, group, n_planes, density, batch=1, tag="", **enc):
        nonlocal launches
        for name, (out, inp) in shapes:
            S = Q.stagq_pack(Q.stagq_encode(synth.weights(out, inp, seed=out + 3 * inp), group, n_planes,
                                            density, "fast", **enc))
            m0 = Q.stagq_load(S, 0)
            C = copies_for(Q, m0.device_bytes, l2)
            mats = [m0] + [Q.stagq_load(S, 0) for _ in range(C - 1)]
            x = torch.from_numpy(synth.activations(batch, inp, seed=inp)).cuda()
            y = torch.empty(batch, out, dtype=torch.float16, device="cuda")
            for b in bits_list:
                us = time_gemv(Q, torch, mats, b, x, y, batch, stream)
                launches += 24 * 5 * 3
                nb = Q.stagq_bytes(m0, b, batch)
                results[f"{tag}{name} {out}x{inp} p{b}"] = {"us": round(us, 3), "bytes": nb,
                                                           "gbs": round(nb / us / 1e3, 1),
                                                           "frac": round(nb / us / 1e3 / peak, 4)}
            for m in mats:
                m.free()
            del S

    def layer_chain(model, linears, bits_list, group, n_planes, density, **enc):
        """One layer's linears as a decode runs them -- q/k/v stacked in one
        launch, o, gate/up stacked, down -- as one CUDA graph, rotating over
        enough device copies that reads come from HBM; µs per layer."""
        nonlocal launches
        streams = {}
        for _, (out, inp) in linears:
            if (out, inp) not in streams:
                streams[(out, inp)] = Q.stagq_pack(Q.stagq_encode(synth.weights(out, inp, seed=out + 3 * inp),
                                                                  group, n_planes, density, "fast", **enc))
        # linears come in the order q, k, v, o, gate, up, down
        assert len(linears) == 7
        groups = [(0, 1, 2), (3,), (4, 5), (6,)]

        def load():
            return [Q.stagq_load_stack([streams[linears[i][1]] for i in grp], 0) for grp in groups]
        first = load()
        C = copies_for(Q, sum(m.device_bytes for m in first), l2, minimum=2)
        mats = [first] + [load() for _ in range(C - 1)]
        xs = [torch.from_numpy(synth.activations(1, m.inp, seed=m.inp)).cuda() for m in first]
        ys = [torch.empty(1, m.out, dtype=torch.float16, device="cuda") for m in first]
        for b in bits_list:
            def body(c):
                for j, m in enumerate(mats[c]):
                    Q.stagq_gemv(m, b, xs[j], ys[j], stream=stream)
            with torch.cuda.stream(stream):
                body(0)
            torch.cuda.synchronize()
            reps = 2 * C
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for r in range(reps):
                    body(r % C)
            g.replay()
            torch.cuda.synchronize()
            us = _median_event_us(torch, stream, lambda: [g.replay() for _ in range(4)], 10) / (4 * reps)
            launches += len(groups) * (1 + 41 * reps)
            nb = sum(Q.stagq_bytes(m, b, 1) for m in first)
            results[f"{model} layer p{b}"] = {"us": round(us, 3), "bytes": nb, "gbs": round(nb / us / 1e3, 1),
                                              "frac": round(nb / us / 1e3 / peak, 4), "gemvs": len(linears),
                                              "launches": len(groups)}
            del g
        for L in mats:
            for m in L:
                m.free()

    if args.workload == "phi4_olmo2_linears_b1":
        shapes = [("phi4." + k, v) for k, v in synth.PHI4_LINEARS.items()] + \
                 [("olmo2." + k, v) for k, v in synth.OLMO2_7B_LINEARS.items()]
        per_gemv(shapes, BITS, GROUP, N_PLANES, DENSITY)
        P, O = synth.PHI4_LINEARS, synth.OLMO2_7B_LINEARS
        layer_chain("phi4", [("q", P["qo"]), ("k", P["kv"]), ("v", P["kv"]), ("o", P["qo"]),
                             ("gate", P["gate_up"]), ("up", P["gate_up"]), ("down", P["down"])],
                    BITS, GROUP, N_PLANES, DENSITY)
        layer_chain("olmo2", [("q", O["qkvo"]), ("k", O["qkvo"]), ("v", O["qkvo"]), ("o", O["qkvo"]),
                              ("gate", O["gate_up"]), ("up", O["gate_up"]), ("down", O["down"])],
                    BITS, GROUP, N_PLANES, DENSITY)
        cfg = {"linears_out_x_in": {k: list(v) for k, v in shapes}, "bits": list(BITS), "group": GROUP,
               "n_planes": N_PLANES, "side_record_density": DENSITY, "batch": 1}
    elif args.workload == "cublas_context":
        # Context only (the paper's Table 5 reports speedups over cuBLAS): the
        # dense fp16 GEMV of torch (cuBLAS) on the Llama-3.1-8B shapes, timed
        # like the StagQ GEMVs (a CUDA graph of launches rotating over device
        # copies larger than L2), and the StagQ times of the same shapes.
        shapes = _layer_shapes()
        per_gemv(shapes, BITS, GROUP, N_PLANES, DENSITY)
        for name, (out, inp) in shapes:
            nbytes = 2 * out * inp
            C = copies_for(Q, nbytes, l2, minimum=2)
            Ws = [torch.randn(out, inp, device="cuda", dtype=torch.float16) * 0.02 for _ in range(C)]
            xv = torch.from_numpy(synth.activations(1, inp, seed=inp)[0]).cuda()
            yv = torch.empty(out, dtype=torch.float16, device="cuda")
            with torch.cuda.stream(stream):
                torch.mv(Ws[0], xv, out=yv)
            torch.cuda.synchronize()
            reps = 24
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for r in range(reps):
                    torch.mv(Ws[(r + 1) % C], xv, out=yv)
            g.replay()
            torch.cuda.synchronize()
            ts = []
            for _ in range(3):
                a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(stream):
                    a0.record(stream)
                    for _ in range(5):
                        g.replay()
                    a1.record(stream)
                torch.cuda.synchronize()
                ts.append(a0.elapsed_time(a1) * 1e3 / (5 * reps))
            del g
            us = statistics.median(ts)
            nb = nbytes + 2 * inp + 2 * out
            r = {"us": round(us, 3), "bytes": nb, "gbs": round(nb / us / 1e3, 1), "frac": round(nb / us / 1e3 / peak, 4)}
            for b in BITS:
                st = results.get(f"{name} {out}x{inp} p{b}")
                if st:
                    r[f"speedup_p{b}"] = round(us / st["us"], 3)
            results[f"cublas_fp16 {name} {out}x{inp}"] = r
            del Ws
            torch.cuda.empty_cache()
        cfg = {"linears_out_x_in": {k: list(v) for k, v in shapes}, "bits": list(BITS), "group": GROUP,
               "n_planes": N_PLANES, "side_record_density": DENSITY, "batch": 1,
               "note": "context: dense fp16 torch.mv (cuBLAS) on random weights; speedup = t_cuBLAS / t_StagQ"}
    elif args.workload == "llama31_8b_guarded":
        # The paper's guards on every linear (pre-grid ratio criterion T = 4 and
        # the post-grid per-row guard, Table 6 / Appendix E) at its kernel
        # evaluation's group size 32 (Section 4.3).
        shapes = _layer_shapes()
        guard = dict(guard="ratio", ratio_T=4.0, post_guard=True)
        per_gemv(shapes, BITS, 32, N_PLANES, 0.0, **guard)
        L = synth.LLAMA31_8B_LINEARS
        layer_chain("llama31_8b_g32_guarded", [(k, L[k]) for k in ("q_proj", "k_proj", "v_proj", "o_proj",
                                                                    "gate_proj", "up_proj", "down_proj")],
                    BITS, 32, N_PLANES, 0.0, **guard)
        cfg = {"linears_out_x_in": {k: list(v) for k, v in shapes}, "bits": list(BITS), "group": 32,
               "n_planes": N_PLANES, "side_record": "pre-grid ratio guard T = 4 + post-grid guard (1 per row)",
               "batch": 1}
    elif args.workload == "precision_sweep":
        shapes = [("gate", (14336, 4096)), ("down", (4096, 14336))]
        for g in (16, 32, 64, 128):
            for d in (0.0, 0.001, 0.01):
                per_gemv(shapes, (2, 3, 4, 5, 6), g, 4, d, tag=f"g{g} d{d} ")
        cfg = {"shapes_out_x_in": [list(v) for _, v in shapes], "bits": [2, 3, 4, 5, 6], "n_planes": 4,
               "groups": [16, 32, 64, 128], "side_record_densities": [0.0, 0.001, 0.01], "batch": 1}
    else:  # llama31_8b_stack
        layers, K = 32, max(1, args.stack_distinct)
        shapes = _layer_shapes()
        names = [n for n, _ in shapes]
        enc = []
        for li in range(K):
            enc.append({n: Q.stagq_pack(Q.stagq_encode(synth.weights(o, i, seed=1000 * li + j), GROUP, N_PLANES,
                                                       DENSITY, "fast")) for j, (n, (o, i)) in enumerate(shapes)})
        # per layer the launches a decode runs: q/k/v stacked, o, gate/up stacked, down
        stack = [[Q.stagq_load_stack([enc[li % K][n] for n in members], 0) for _, members in LAYER_LAUNCHES]
                 for li in range(layers)]
        del enc
        weights = layers * sum(o * i for _, (o, i) in shapes)
        shapes = [(name, (stack[0][j].out, stack[0][j].inp)) for j, (name, _) in enumerate(LAYER_LAUNCHES)]
        for batch in (1, 4):
            xs = [torch.from_numpy(synth.activations(batch, i, seed=i + batch)).cuda() for _, (o, i) in shapes]
            ys = [torch.empty(batch, o, dtype=torch.float16, device="cuda") for _, (o, i) in shapes]
            for b in BITS:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.stream(stream):
                    for li in range(layers):
                        for j in range(len(shapes)):
                            Q.stagq_gemv_n(stack[li][j], b, xs[j], batch, ys[j], stream=stream)
                torch.cuda.synchronize()
                with torch.cuda.graph(g, stream=stream):
                    for li in range(layers):
                        for j in range(len(shapes)):
                            Q.stagq_gemv_n(stack[li][j], b, xs[j], batch, ys[j], stream=stream)
                for _ in range(3):
                    g.replay()
                torch.cuda.synchronize()
                ts = []
                for _ in range(5):
                    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    with torch.cuda.stream(stream):
                        a0.record(stream)
                        g.replay()
                        a1.record(stream)
                    torch.cuda.synchronize()
                    ts.append(a0.elapsed_time(a1) * 1e3)
                launches += 8 * layers * len(shapes)
                us = statistics.median(ts)
                nb = sum(Q.stagq_bytes(stack[0][j], b, batch) for j in range(len(shapes))) * layers
                results[f"p{b} batch{batch}"] = {"us_per_token_step": round(us, 1),
                                                 "us_per_token": round(us / batch, 1), "bytes": nb,
                                                 "gbs": round(nb / us / 1e3, 1), "frac": round(nb / us / 1e3 / peak, 4),
                                                 "gemvs": layers * len(names), "launches": layers * len(shapes)}
                del g
        stored = sum(m.device_bytes for L in stack for m in L)
        for L in stack:
            for m in L:
                m.free()
        cfg = {"layers": layers, "linears_out_x_in": {k: list(v) for k, v in _layer_shapes()},
               "launches_per_layer": {name: list(members) for name, members in LAYER_LAUNCHES}, "weights": weights,
               "distinct_encoded_layers": K, "stored_bytes": stored, "bits": list(BITS), "batches": [1, 4],
               "group": GROUP, "n_planes": N_PLANES, "side_record_density": DENSITY,
               "note": f"the 32 resident layers cycle over {K} distinct encodings (timing does not depend on "
                       f"the weight values; {stored / 1e9:.2f} GB resident >> L2)"}
    clk = clocks.stop()
    vals = [r["gbs"] for r in results.values()]
    value = round(statistics.median(vals), 1) if vals else None
    _extra_line(args, args.workload, results, cfg, clk, peak, peak_kind, value, "GB/s", launches)


# The layer step: per precision, the launches of one Llama-3.1-8B layer as a
# decode runs them -- q/k/v stacked in one handle (they share x), o, gate/up
# stacked (they share x), down -- each on its own input.
LAYER_LAUNCHES = [("qkv", ("q_proj", "k_proj", "v_proj")), ("o", ("o_proj",)),
                  ("gate_up", ("gate_proj", "up_proj")), ("down", ("down_proj",))]


def _median_event_us(torch, stream, fn, repeats):
    """Median of `repeats` CUDA-event timings (µs) of fn() on `stream`."""
    out = []
    for _ in range(repeats):
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a0.record(stream)
            fn()
            a1.record(stream)
        torch.cuda.synchronize()
        out.append(a0.elapsed_time(a1) * 1e3)
    return statistics.median(out)


def run_stagq(args):
    import torch
    import quantized_gemv_stagq_b200 as Q
    from quantized_gemv_stagq_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = local
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size

    # ---- encode the layer once (library encoder, fast pair rule) and pack
    shapes = _layer_shapes()
    packed = {}
    for li, (name, (out, inp)) in enumerate(shapes):
        W = synth.weights(out, inp, seed=100 + li)
        packed[name] = Q.stagq_pack(Q.stagq_encode(W, GROUP, N_PLANES, DENSITY, "fast"))
        del W

    def load_layer():
        return [Q.stagq_load_stack([packed[n] for n in members], dev) for _, members in LAYER_LAUNCHES]

    first = load_layer()
    stored = sum(m.device_bytes for m in first)
    step_bytes = sum(Q.stagq_bytes(first[i], b, 1) for b in BITS for i in range(len(first)))
    # Cold protocol: a step runs p2, p3, p4 each on its own copy of the layer,
    # and a copy comes back only after at least 4x the L2 size of other reads
    # (C / 3 - 1 whole steps in between).
    C = len(BITS) * max(-(-args.copies // len(BITS)), -(-4 * l2 // step_bytes) + 1)
    layers = [first] + [load_layer() for _ in range(C - 1)]
    xs = [torch.from_numpy(synth.activations(1, m.inp, seed=200 + i)).cuda() for i, m in enumerate(first)]
    ys = [torch.empty(1, m.out, dtype=torch.float16, device="cuda") for m in first]

    stream = torch.cuda.Stream()

    def step_launches(s):
        for k, b in enumerate(BITS):
            L = layers[(len(BITS) * s + k) % C]
            for i, m in enumerate(L):
                Q.stagq_gemv(m, b, xs[i], ys[i], stream=stream)

    # ---- one CUDA graph per distinct step (copies cycle every G steps)
    G = C // len(BITS)
    with torch.cuda.stream(stream):
        step_launches(0)  # warm the launch path outside capture
    torch.cuda.synchronize()
    graphs = []
    for s in range(G):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step_launches(s)
        graphs.append(g)
    torch.cuda.synchronize()
    for w in range(max(args.warmup, 3)):
        graphs[w % G].replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(torch.cuda.current_device() if world == 1 else local)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for s in range(args.steps):
            graphs[s % G].replay()
        e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)

    # ---- per launch: each launch of the step alone, a CUDA graph of launches
    # rotating over enough device copies of it that a pass over them is at
    # least 4x the L2 size (every read from HBM), median of 10 timings
    per = {}
    with torch.cuda.stream(stream):
        for i, (name, members) in enumerate(LAYER_LAUNCHES):
            pool = [layers[c][i] for c in range(C)]
            while len(pool) < copies_for(Q, first[i].device_bytes, l2):
                pool.append(Q.stagq_load_stack([packed[n] for n in members], dev))
            reps = 2 * len(pool)
            for b in BITS:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for r in range(reps):
                        Q.stagq_gemv(pool[r % len(pool)], b, xs[i], ys[i], stream=stream)
                g.replay()
                torch.cuda.synchronize()
                us = _median_event_us(torch, stream, g.replay, 10) / reps
                nb = Q.stagq_bytes(first[i], b, 1)
                per.setdefault(f"p{b}", {})[name] = {"us": round(us, 3), "bytes": nb, "gbs": round(nb / us / 1e3, 1),
                                                      "out_x_in": [first[i].out, first[i].inp], "copies": len(pool)}
                del g
            for m in pool[C:]:
                m.free()
    clk = clocks.stop()

    if dist:
        ms = job_ms(ms, dist, "cuda")
        dist.barrier()

    # ---- end to end through the C ABI with host buffers: a step's 12 GEMVs in
    # one stagq_gemv_host_many call (x copied in, GEMVs, y copied out, one sync)
    e2e_steps = max(2, min(args.steps, 10))
    xh = [x.cpu().pin_memory().numpy() for x in xs]
    yh = [[torch.empty((1, m.out), dtype=torch.float16).pin_memory().numpy() for m in first] for _ in BITS]

    def e2e_step(s):
        mats, bl, xl, yl = [], [], [], []
        for k, b in enumerate(BITS):
            for i, m in enumerate(layers[(len(BITS) * s + k) % C]):
                mats.append(m)
                bl.append(b)
                xl.append(xh[i])
                yl.append(yh[k][i])
        Q.stagq_gemv_host_many(mats, bl, xl, yl, stream=stream)

    e2e_step(0)
    h2d = sum(2 * m.inp for b in BITS for m in first)
    d2h = sum(2 * m.out for b in BITS for m in first)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for s in range(e2e_steps):
        e2e_step(s)
    e2e_s = time.perf_counter() - t0
    e2e_gbs = step_bytes * e2e_steps / e2e_s / 1e9

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peak, peak_kind = _peaks()
    value = job_value(world, step_bytes, args.steps, ms)
    # dominant kernel: the launch with the largest share of a step
    dom_key, dom = max(((f"{name}@{pb}", d) for pb, dd in per.items() for name, d in dd.items()),
                       key=lambda kv: kv[1]["us"])
    traffic, _ = _ncu_traffic()
    cpu = None
    if not args.no_cpu_baseline:
        v, s, sample, threads = cpu_oracle_sample()
        cpu = {"value": round(v, 4), "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": sample}
    step_us = {pb: round(sum(d["us"] for d in dd.values()), 2) for pb, dd in per.items()}
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int32 dot (u8 codes x i16 x) + fp32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "linears_out_x_in": {n: [o, i] for n, (o, i) in shapes}, "bits": list(BITS),
                   "group": GROUP, "n_planes": N_PLANES, "side_record_density": DENSITY, "batch": 1,
                   "pair_rule": "fast",
                   "launches_per_step": {name: list(members) for name, members in LAYER_LAUNCHES},
                   "gemvs_per_step": len(BITS) * len(shapes), "kernel_launches_per_step": len(BITS) * len(first),
                   "l2": f"inputs larger than L2: each precision pass of a step reads its own layer copy; {C} copies x "
                         f"{stored / 1e6:.0f} MB stored, {step_bytes / 1e6:.0f} MB read per step vs L2 {l2 / 1e6:.0f} MB",
                   "parallelism": "replicas" if world > 1 else "single"},
        "frac_of_hbm": round(value / world / peak, 4),
        "per_launch": per, "us_per_precision_layer": step_us,
        "roofline": {"bound": "hbm", "kernel": f"{_launch_kernel(dom_key)} {dom_key}", "achieved": dom["gbs"], "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(dom["gbs"] / peak, 4),
                     "traffic": traffic, "algorithmic_bytes": dom["bytes"]},
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_gbs, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": "stagq_gemv_host_many (the step's 12 GEMVs with host x/y, one sync per step)"},
        "gpu_launches": len(BITS) * len(first) * args.steps,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


def main():
    args = _args()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload != WORKLOAD:
        run_extra(args)
    else:
        run_stagq(args)


if __name__ == "__main__":
    main()
