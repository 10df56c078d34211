"""Benchmark of the routed 2-bit MoE FFN layer on B200.

One step = one moe_layer_forward (router, top-k, permutation, routed expert
FFNs, shared expert, combine) over one batch of synthetic tokens, with all
inputs resident in HBM. Several layers with distinct weights are resident and
used in rotation, so the bytes a step reads are not served from L2 (L2 is
126 MB; one decode step touches ~190 MB and the rotation keeps >= 570 MB in
flight between reuses).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config decode1|decode32|prefill|stack]
                  [--impl ours|reference]

Under torchrun each rank runs its own batches (weak scaling, no collective on
the data path); the step time is the max over ranks. ``--impl reference``
times the CPU oracle (the baseline arm) on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import tempfile
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

HBM_FALLBACK_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="decode1", choices=["decode1", "decode32", "prefill", "stack"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=0, help="resident layers in rotation (0 = config default)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="launch every step directly instead of replaying CUDA graphs")
    ap.add_argument("--experts", type=int, default=0,
                    help="override the routed expert count (small cases for profiling; not a bench workload)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the tokens per step (small cases for profiling; not a bench workload)")
    ap.add_argument("--workloads", default="auto",
                    help="other workloads measured in the same run and reported under 'workloads': 'all' "
                         "(decode32, prefill, stack, decode1_mxfp4, decode1_q4, prefill_mxfp4, prefill_q4, decode1_cached, "
                         "quantize), 'none', or a comma list; "
                         "'auto' = all on one GPU")
    ap.add_argument("--workload-steps", type=int, default=20, help="timed steps of each extra workload")
    ap.add_argument("--workloads-only", action="store_true",
                    help="profiling aid: skip the main configuration and print only the 'workloads' object")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p.get("bf16_tflops", 0.0)), "measured"
    except Exception:
        return HBM_FALLBACK_GBS, 1590.0, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index
        self.path = None

    def start(self):
        try:
            # raw samples go to a temporary folder unless MOE_BENCH_CLOCKS_DIR names one to keep them
            out_dir = os.environ.get("MOE_BENCH_CLOCKS_DIR") or tempfile.gettempdir()
            os.makedirs(out_dir, exist_ok=True)
            self.path = os.path.join(out_dir, f"clocks_bench_{os.getpid()}.csv")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------- bytes
def expert_bytes(cfg) -> dict:
    nb = cfg.I * cfg.H // 256
    return {"gateup": 2 * nb * (64 + 2), "down": nb * (80 + 4), "shared": 3 * cfg.Is * cfg.H * 2,
            "router": cfg.E * cfg.H * 2}


def traffic_record(workload: str, kernel: str):
    """dram bytes per launch of `kernel` in `workload` from a committed ncu
    summary (key "workload:kernel"), if its source hash matches the current
    kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        rec = json.load(open(p)).get(f"{workload}:{kernel}")
        if not rec:
            return None
        src = os.path.join(ROOT, rec["source"])
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()
        return rec if h == rec["sha256"] else None
    except Exception:
        return None


# ------------------------------------------------------------ multi-rank
def max_over_ranks(vals, world, device):
    """Element-wise max of per-rank timings; every rank calls it at the same
    point (one all-reduce of a few scalars, outside the data path)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor(vals, dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def job_tokens_per_s(tokens_per_rank_step, world, ms_per_step):
    """Whole-job throughput: every rank processes its own tokens (replicas)."""
    return tokens_per_rank_step * world / (ms_per_step * 1e-3)


def rank_seed(cfg_seed, rank):
    """Input seed of a rank: replicas work on distinct synthetic tokens."""
    return cfg_seed + 7919 * rank


# --------------------------------------------------------------- reference
def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_tokens(cfg, x, budget_s, tokens_per_call):
    """Oracle throughput on a bounded sample: calls of `tokens_per_call` tokens
    until `budget_s` seconds have passed (at least one call)."""
    import oracle

    lw = synth.make_layer(cfg)
    n, t0 = 0, time.perf_counter()
    while n + tokens_per_call <= x.shape[0]:
        oracle.layer_forward(lw, np.ascontiguousarray(x[n:n + tokens_per_call]))
        n += tokens_per_call
        if time.perf_counter() - t0 > budget_s:
            break
    return n, time.perf_counter() - t0


def run_reference(args, cfg):
    """The reference arm: the CPU oracle as it stands (OpenMP build, every host
    core), one bounded sample of the workload per step."""
    import oracle

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    oracle.build()
    lw = synth.make_layer(cfg)
    per_step_tokens = 1 if cfg.T < 64 else 16
    x = synth.make_x_fast(cfg, max(args.steps + args.warmup, 1) * per_step_tokens)
    for i in range(args.warmup):
        oracle.layer_forward(lw, np.ascontiguousarray(x[i * per_step_tokens:(i + 1) * per_step_tokens]))
    t0 = time.perf_counter()
    for i in range(args.steps):
        j = args.warmup + i
        oracle.layer_forward(lw, np.ascontiguousarray(x[j * per_step_tokens:(j + 1) * per_step_tokens]))
    dt = time.perf_counter() - t0
    value = per_step_tokens * args.steps / dt
    cores = oracle.threads()
    sample = (f"{per_step_tokens} token(s) per step through the full {cfg.name} layer (router, {cfg.k} experts, "
              f"shared), C oracle on {cores} threads")
    line = {
        "impl": "reference", "metric": "moe_layer_tokens_per_s", "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "tokens_per_step": per_step_tokens, "H": cfg.H, "I": cfg.I, "E": cfg.E,
                   "k": cfg.k, "I_s": cfg.Is},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample,
                         "cpu_model": cpu_model(), "nproc": os.cpu_count()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline(cfg, budget_s=12.0):
    """The oracle timed on the host cores: the OpenMP build on every core (the
    reported value) and the single-threaded build (context), each on a bounded
    sample of the workload's tokens."""
    import subprocess as sp

    x = synth.make_x_fast(cfg, 64)
    import oracle

    oracle.build()
    n, dt = oracle_tokens(cfg, x, budget_s, 1)
    out = {"value": n / dt, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
           "sample": f"{n} tokens of the {cfg.name} layer one at a time, C oracle (OpenMP) on {oracle.threads()} "
                     f"threads ({dt:.1f} s)",
           "cpu_model": cpu_model(), "nproc": os.cpu_count()}
    # the single-threaded build, in a child process (the OpenMP build is loaded here)
    code = ("import sys, json; sys.path.insert(0, sys.argv[1]); import bench, synth; "
            "cfg = synth.CONFIGS[sys.argv[2]]; x = synth.make_x_fast(cfg, 64); "
            "n, dt = bench.oracle_tokens(cfg, x, float(sys.argv[3]), 1); print(json.dumps([n, dt]))")
    try:
        r = sp.run([sys.executable, "-c", code, ROOT, cfg.name, str(budget_s / 2)], capture_output=True, text=True,
                   env=dict(os.environ, MOEREF_OPENMP="0"), timeout=600)
        n1, dt1 = json.loads(r.stdout.strip().splitlines()[-1])
        out["single_thread"] = {"value": n1 / dt1, "unit": "tokens/s", "cores": 1,
                                "sample": f"{n1} tokens one at a time ({dt1:.1f} s)"}
    except Exception as exc:  # the figure is context only
        out["single_thread"] = {"unavailable": str(exc)[:200]}
    return out


# -------------------------------------------------------------------- ours
def measure(args, cfg, world, rank, local, steps):
    """Time `steps` steps of one workload (CUDA-graph replay, device events, max
    over ranks), then the same steps with per-kernel events, then end to end
    with host buffers. Returns the JSON fields of that workload."""
    import torch

    from bit_quantized_routed_iq2_b200 import moe2bit

    n_layers = args.layers or {"decode1": 4, "decode32": 4, "prefill": 2, "stack": cfg.layers}.get(cfg.name, 1)
    is_stack = cfg.name.startswith("stack")
    T = cfg.T
    layers = []
    for l in range(n_layers):
        lw = synth.make_layer(cfg, layer=l)
        layers.append(moe2bit.to_device(lw))
        del lw
    n_slots = 4
    xs_host = [synth.make_x_fast(cfg, T, layer=100 + s, cfg_seed=rank_seed(cfg.seed, rank)) for s in range(n_slots)]

    def dev_x(a):
        t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()
        return t.view(torch.bfloat16) if a.dtype == np.uint16 else t

    xs = [dev_x(a) for a in xs_host]
    res = None
    if is_stack:
        res = torch.from_numpy(synth.make_residual(cfg, T, cfg_seed=cfg.seed + rank)).cuda()
    y = torch.empty((T, cfg.H), dtype=torch.float32, device="cuda")
    ws = moe2bit.alloc_workspace(layers[0].desc, T)
    stream = torch.cuda.current_stream()
    # the next layer's bf16 input, written by the library beside y (two buffers: a layer's output may not
    # overlap its own input)
    xa = [torch.empty((T, cfg.H), dtype=torch.bfloat16, device="cuda") for _ in range(2)] if is_stack else None

    side = torch.cuda.Stream() if is_stack else None

    def chain(first_x, st, out=None):
        """The layers in order; while layer l runs, layer l+1's router and shared expert are prefetched
        into L2 on a side stream (they do not depend on routing). The residual stream is `out` (default y)."""
        yo = y if out is None else out
        cur = first_x
        for l, dl in enumerate(layers):
            if l + 1 < len(layers):
                side.wait_stream(st)
                moe2bit.prefetch_layer(layers[l + 1], side)
            nxt = xa[l % 2] if l + 1 < len(layers) else None  # bf16 of the residual stream, for layer l + 1
            moe2bit.layer_forward(dl, cur, res if l == 0 else yo, yo, ws, st, y_next=nxt)
            cur = nxt
        st.wait_stream(side)

    if is_stack:
        # one step = a 16-token decode step through all resident layers chained by the residual stream
        def step_on(i, st):
            chain(xs[i % n_slots], st)
    else:
        def step_on(i, st):
            moe2bit.layer_forward(layers[i % n_layers], xs[i % n_slots], None, y, ws, st)

    warm = max(args.warmup, 3)
    for i in range(warm):
        step_on(i, stream)
    torch.cuda.synchronize()
    # The timed steps replay CUDA graphs of the same library calls (the library
    # launches nothing that a graph cannot hold); one graph per distinct
    # (layer, input) slot of the rotation.
    period = n_slots if is_stack else int(np.lcm(n_layers, n_slots))
    graphs = []
    if args.graph:
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        for j in range(period):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                step_on(j, cap)
            graphs.append(g)
        torch.cuda.synchronize()
        for j in range(period):
            graphs[j].replay()
        torch.cuda.synchronize()

    def timed_step(i):
        if graphs:
            graphs[i % period].replay()
        else:
            step_on(i, stream)

    import torch.distributed as dist

    if world > 1:
        dist.barrier()
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        timed_step(warm + i)
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = e0.elapsed_time(e1) / steps

    # per-kernel durations (CUDA events around each library launch, same workload)
    moe2bit.profile_enable(True)
    for i in range(steps):
        step_on(warm + i, stream)
    torch.cuda.synchronize()
    prof = moe2bit.profile_read()
    moe2bit.profile_enable(False)

    # end to end through the public API with host buffers: pinned x -> device, layer, y -> pinned host
    xh = [torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).pin_memory() for a in xs_host]
    yh = torch.empty((T, cfg.H), dtype=torch.float32).pin_memory()
    xd = torch.empty((T, cfg.H), dtype=torch.int16 if cfg.x_dtype == "bf16" else torch.float32, device="cuda")
    xdv = xd.view(torch.bfloat16) if cfg.x_dtype == "bf16" else xd

    # Every step copies its own x from pinned host memory and reads its own y back into pinned host memory.
    # Step i's graph holds three independent branches: the input copy of step i + 1, the layer of step i and the
    # read-back of step i - 1 (x and y double-buffered), so the copies overlap the neighbouring steps' layers as
    # a serving loop would run; an input copy before the first step and a read-back after the last complete the
    # timed region (one copy of each kind more than the steps need).
    xdb = [xd, torch.empty_like(xd)]
    yb = [y, torch.empty_like(y)]
    yhb = [yh, torch.empty_like(yh).pin_memory()]
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    eperiod = int(np.lcm(2, period))

    def xview(b):
        return xdb[b].view(torch.bfloat16) if cfg.x_dtype == "bf16" else xdb[b]

    def e2e_step(i, st):
        h2d.wait_stream(st)
        d2h.wait_stream(st)
        with torch.cuda.stream(h2d):
            xdb[(i + 1) % 2].copy_(xh[(i + 1) % n_slots], non_blocking=True)
        with torch.cuda.stream(d2h):
            yhb[(i + 1) % 2].copy_(yb[(i + 1) % 2], non_blocking=True)  # the read-back of step i - 1
        if is_stack:
            chain(xview(i % 2), st, out=yb[i % 2])
        else:
            moe2bit.layer_forward(layers[i % n_layers], xview(i % 2), None, yb[i % 2], ws, st)
        st.wait_stream(h2d)
        st.wait_stream(d2h)

    def e2e_first(st):
        with torch.cuda.stream(st):
            xdb[0].copy_(xh[0], non_blocking=True)

    def e2e_last(i, st):
        with torch.cuda.stream(st):
            yhb[i % 2].copy_(yb[i % 2], non_blocking=True)

    e2e_first(stream)
    for i in range(warm):
        e2e_step(i, stream)
    torch.cuda.synchronize()
    e2e_graphs = []
    if args.graph:
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        for j in range(eperiod):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                e2e_step(j, cap)
            e2e_graphs.append(g)
        torch.cuda.synchronize()
    e0.record(stream)
    e2e_first(stream)
    for i in range(steps):
        if e2e_graphs:
            e2e_graphs[i % eperiod].replay()
        else:
            e2e_step(i, stream)
    e2e_last(steps - 1, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = e0.elapsed_time(e1) / steps
    del e2e_graphs
    clocks = clk.stop()
    ms, ms_e2e = max_over_ranks([ms, ms_e2e], world, "cuda")

    # realised active experts per layer step, from the library's own routing
    act = []
    for sl in range(n_slots):
        for l in range(min(n_layers, 4)):
            dl = layers[l]
            idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
            w = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
            off = torch.empty(cfg.E + 1, dtype=torch.int32, device="cuda")
            perm = torch.empty(T * cfg.k, dtype=torch.int32, device="cuda")
            inv = torch.empty(T * cfg.k, dtype=torch.int32, device="cuda")
            moe2bit.route(dl.desc, dl.tensors["router_w"], dl.tensors["router_bias"], xs[sl], idx, w, off, perm, inv,
                          ws)
            o = off.cpu().numpy()
            act.append(int(np.count_nonzero(np.diff(o))))
    n_active = float(np.mean(act))
    del graphs, layers, xs, ws
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    hbm, bf16_tf, peak_kind = peaks()
    eb = expert_bytes(cfg)
    lps = n_layers if is_stack else 1  # library layer calls per step
    launches_per_step = {k: v[1] / steps for k, v in prof.items()}
    avg_ms = {k: v[0] / max(v[1], 1) for k, v in prof.items()}
    # the dominant kernel among those with an algorithmic model (the combine's span also covers its wait for
    # the side stream, so it is not a candidate)
    modeled = [k for k in prof if k in ("gateup", "down", "prefill_gateup", "prefill_down", "shared_gateup",
                                        "shared_down")]
    dom = max(modeled or list(prof), key=lambda k: prof[k][0])
    if dom in ("gateup", "prefill_gateup"):
        alg = n_active * eb["gateup"] + T * cfg.H * (2 if cfg.x_dtype == "bf16" else 4)
    elif dom in ("down", "prefill_down"):
        alg = n_active * eb["down"] + T * cfg.k * cfg.I * 2 + T * cfg.k * cfg.H * 4
    elif dom in ("shared_gateup",):
        alg = 2 * cfg.Is * cfg.H * 2
    elif dom in ("shared_down",):
        alg = cfg.Is * cfg.H * 2
    else:
        alg = 0
    tr = traffic_record(cfg.name, dom)
    if cfg.name.startswith("prefill") and dom in ("prefill_gateup", "prefill_down") and bf16_tf > 0:
        # the grouped GEMM is a dense contraction: fp16 operands (the same tensor rate as
        # bf16), FLOPs = 2 * assignments * output rows * K
        nA = T * cfg.k
        flops = 2.0 * nA * 2 * cfg.I * cfg.H if dom == "prefill_gateup" else 2.0 * nA * cfg.H * cfg.I
        achieved = flops / (avg_ms[dom] * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": bf16_tf, "unit": "TFLOP/s",
                "frac": achieved / bf16_tf,
                "peak_source": f"{peak_kind} bf16_tflops (burst; fp16 runs at the bf16 rate)",
                "traffic": tr["bytes_per_launch"] if tr else None, "algorithmic_flops_per_launch": flops,
                "algorithmic_bytes_per_launch": alg, "avg_launch_ms": avg_ms[dom]}
    else:
        achieved = alg / (avg_ms[dom] * 1e-3) / 1e9 if alg else 0.0
        roof = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "peak_source": f"{peak_kind} hbm_gbs",
                "traffic": tr["bytes_per_launch"] if tr else None,
                "algorithmic_bytes_per_launch": alg, "avg_launch_ms": avg_ms[dom]}
    layer_bytes = n_active * (eb["gateup"] + eb["down"]) + eb["shared"] + eb["router"] + T * cfg.H * 6
    step_bytes = layer_bytes * lps
    bytes_x = T * cfg.H * (2 if cfg.x_dtype == "bf16" else 4)
    return {
        "value": job_tokens_per_s(T, world, ms), "unit": "tokens/s", "ms_per_step": ms,
        "config": {"workload": cfg.name, "tokens_per_step": T, "H": cfg.H, "I": cfg.I, "E": cfg.E, "k": cfg.k,
                   "I_s": cfg.Is, "x_dtype": cfg.x_dtype, "resident_layers": n_layers,
                   "layers_per_step": lps, "routing": "zipf(1.1) router bias" if cfg.zipf else "plain",
                   "l2": f"inputs larger than L2: {n_layers} resident layers in rotation",
                   "active_experts_per_layer": n_active, "layer_bytes_touched": layer_bytes,
                   "launch": "cuda_graph" if args.graph else "direct"},
        "roofline": roof,
        # whole-step HBM rate over the realised touched bytes (router, active experts, shared, activations)
        "step_hbm": {"achieved_gbs": step_bytes / (ms * 1e-3) / 1e9, "peak": hbm,
                     "frac": step_bytes / (ms * 1e-3) / 1e9 / hbm, "bytes_per_step": step_bytes},
        "kernels": {k: {"avg_ms": avg_ms[k], "launches_per_step": launches_per_step[k]} for k in prof},
        "gpu_launches": int(round(sum(launches_per_step.values()) * steps)),
        "clocks": clocks,
        "e2e": {"value": job_tokens_per_s(T, world, ms_e2e), "unit": "tokens/s",
                "h2d_bytes_per_step": bytes_x, "d2h_bytes_per_step": T * cfg.H * 4,
                "copies": "every step: x from pinned host, y to pinned host; in step i's graph the input copy of "
                          "step i+1 and the read-back of step i-1 run beside the layer (double-buffered)"},
        "dtype": "fp16" if "prefill_gateup" in prof else "int8",
        "steps": steps,
    }


def h2d_gbs(nbytes=256 << 20, reps=5):
    """Host-to-device copy rate from page-locked memory, measured here (the
    denominator of the expert cache's miss traffic)."""
    import torch

    h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    d = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    d.copy_(h, non_blocking=True)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        d.copy_(h, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    return nbytes * reps / (e0.elapsed_time(e1) * 1e-3) / 1e9


def measure_cached(args, steps, n_slots=64):
    """One-token decode steps with every routed expert in page-locked host
    memory and n_slots of them cached in HBM (moe_layer_forward_cached), under
    Zipf(1.1) routing: steady-state tokens/s, hit rate and the miss traffic's
    host-to-device rate. The call synchronises once per step (it reads the
    routing back), so steps are launched directly and timed with events."""
    import torch

    from bit_quantized_routed_iq2_b200 import moe2bit

    cfg = synth.Config("decode1_cached", 1, 7168, 2048, 256, 8, 2048, "bf16", 1.0, True, 1, 0xD5400006)
    lw = synth.make_layer(cfg)
    shared = moe2bit.to_device_shared_only(lw)
    cache = moe2bit.ExpertCache(lw, n_slots)
    del lw
    ws = moe2bit.alloc_workspace(shared.desc, 1)
    xs_host = synth.make_x_fast(cfg, steps + 64)
    xs = torch.from_numpy(xs_host.view(np.int16)).cuda().view(torch.bfloat16)
    y = torch.empty((1, cfg.H), dtype=torch.float32, device="cuda")
    warm = 48  # fills the cache
    for i in range(warm):
        cache.forward(shared, xs[i:i + 1], None, y, ws)
    torch.cuda.synchronize()
    st0 = cache.stats()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        cache.forward(shared, xs[warm + i:warm + i + 1], None, y, ws)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    st1 = cache.stats()
    hits, misses = st1["hits"] - st0["hits"], st1["misses"] - st0["misses"]
    copied = st1["bytes_copied"] - st0["bytes_copied"]
    peak = h2d_gbs()
    achieved = copied / steps / (ms * 1e-3) / 1e9
    cache.close()
    del cache, shared, ws
    torch.cuda.empty_cache()
    return {
        "value": 1.0 / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
        "config": {"workload": cfg.name, "tokens_per_step": 1, "H": cfg.H, "I": cfg.I, "E": cfg.E, "k": cfg.k,
                   "I_s": cfg.Is, "routing": "zipf(1.1) router bias", "slots": n_slots,
                   "host_pool": "all routed experts in page-locked host memory",
                   "launch": "direct (the call reads the routing back once per step)"},
        "hit_rate": hits / max(hits + misses, 1), "misses_per_step": misses / steps,
        # while misses occur the step is bound by the host-to-device link
        "roofline": {"bound": "h2d", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": "pinned host-to-device copy measured in this run",
                     "bytes_per_step": copied / steps},
    }


def measure_mxfp4(args, steps, fmt="mxfp4"):
    """One-token decode with block-32 routed experts: MXFP4 (moe_layer_forward_mxfp4,
    4.25 bits per weight) or Q4-style (moe_layer_forward_q4, 4.5 bits per weight);
    the decode1 shapes (H=7168, I=2048, E=256, k=8, I_s=2048), 2 resident layers
    of all 256 experts and 4 inputs in rotation (inputs larger than L2),
    CUDA-graph replay; roofline of the gate/up GEMV over the bytes of the 8
    active experts' gate and up planes."""
    import torch

    from bit_quantized_routed_iq2_b200 import moe2bit

    q4 = fmt == "q4"
    E = args.experts or 256  # a smaller E (profiling captures) keeps the 8 active experts per step
    cfg = synth.Config("decode1_" + fmt + ("" if E == 256 else f"_E{E}"), 1, 7168, 2048, E, 8, 2048, "bf16", 1.0,
                       False, 1, 0xD5400008 if q4 else 0xD5400007)
    make = synth.make_layer_q4 if q4 else synth.make_layer_mxfp4
    upload = moe2bit.to_device_q4 if q4 else moe2bit.to_device_mxfp4
    forward = moe2bit.layer_forward_q4 if q4 else moe2bit.layer_forward_mxfp4
    scale_bytes = 2.0 if q4 else 1.0  # per 32-weight block
    layers = []
    for l in range(2):
        lw = make(cfg, layer=l)
        layers.append(upload(lw))
        del lw
    n_slots = 4
    xs = [torch.from_numpy(synth.make_x_fast(cfg, 1, layer=100 + s).view(np.int16)).cuda().view(torch.bfloat16)
          for s in range(n_slots)]
    y = torch.empty((1, cfg.H), dtype=torch.float32, device="cuda")
    ws = moe2bit.alloc_workspace_mxfp4(layers[0].desc, 1)  # moe_workspace_size_q4 is the same size
    stream = torch.cuda.current_stream()

    def step_on(i, st):
        forward(layers[i % 2], xs[i % n_slots], None, y, ws, st)

    for i in range(max(args.warmup, 3)):
        step_on(i, stream)
    torch.cuda.synchronize()
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    graphs = []
    for j in range(n_slots):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            step_on(j, cap)
        graphs.append(g)
    torch.cuda.synchronize()
    for g in graphs:
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        graphs[i % n_slots].replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    moe2bit.profile_enable(True)
    for i in range(steps):
        step_on(i, stream)
    torch.cuda.synchronize()
    prof = moe2bit.profile_read()
    moe2bit.profile_enable(False)
    assert moe2bit.read_status(ws) == 0
    del graphs, layers, xs, ws
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    hbm, _, peak_kind = peaks()
    avg_ms = {k: v[0] / max(v[1], 1) for k, v in prof.items()}
    # gate + up codes and scales of the 8 active experts, plus the activations
    alg = cfg.k * 2 * cfg.I * cfg.H * (0.5 + scale_bytes / 32) + cfg.H * 2
    achieved = alg / (avg_ms["gateup"] * 1e-3) / 1e9
    dn_alg = cfg.k * cfg.H * cfg.I * (0.5 + scale_bytes / 32)
    tr = traffic_record("decode1_" + fmt, "gateup")
    return {
        "value": 1.0 / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
        "config": {"workload": cfg.name, "tokens_per_step": 1, "H": cfg.H, "I": cfg.I, "E": cfg.E, "k": cfg.k,
                   "I_s": cfg.Is, "experts": ("Q4-style (32 x 4-bit codes + fp16 d, w = d (q - 8))" if q4 else
                                              "MXFP4 (OCP MX: E2M1 x 32 + E8M0)") + ", all three routed matrices",
                   "resident_layers": 2, "l2": "inputs larger than L2: 2 resident layers of all experts",
                   "launch": "cuda_graph"},
        "kernels": {k: {"avg_ms": v, "launches_per_step": prof[k][1] / steps} for k, v in avg_ms.items()},
        "roofline": {"bound": "hbm", "kernel": "gateup", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "peak_source": peak_kind, "algorithmic_bytes_per_launch": alg,
                     "avg_launch_ms": avg_ms["gateup"], "traffic": tr["bytes_per_launch"] if tr else None,
                     "down_frac": dn_alg / (avg_ms["down"] * 1e-3) / 1e9 / hbm},
    }


def measure_blk32_prefill(args, steps, fmt="mxfp4"):
    """2048 bf16 tokens with block-32 routed experts (the prefill shapes H=7168, I=2048, E=256, k=8,
    I_s=2048; every expert active), one resident layer of 6-6.6 GB (weights larger than L2).
    MXFP4: FP4 weights x MXFP8 activations on the block-scaled tensor cores; roofline of the gate/up
    grouped GEMM against HBM (every active expert's gate and up codes and scales, the MXFP8 activations it
    reads and the MXFP8 h it writes), the tensor-pipe fraction (FP8 x FP4 flops over twice the bf16 peak,
    the nominal fp8 : bf16 ratio) beside it.
    Q4-style: the dequantising grouped GEMM (fp16 weight tiles, tcgen05 kind::f16); roofline of its gate/up
    launch against the bf16 tensor peak, the HBM fraction of its weight bytes beside it."""
    import torch

    from bit_quantized_routed_iq2_b200 import moe2bit

    q4 = fmt == "q4"
    E = args.experts or 256
    name = "prefill_" + fmt + ("" if E == 256 else f"_E{E}")
    cfg = synth.Config(name, 2048 * E // 256, 7168, 2048, E, 8, 2048, "bf16", math.sqrt(0.5), False, 1,
                       0xD540000B if q4 else 0xD540000A)
    lw = (synth.make_layer_q4 if q4 else synth.make_layer_mxfp4)(cfg)
    dl = (moe2bit.to_device_q4 if q4 else moe2bit.to_device_mxfp4)(lw)
    del lw
    forward = moe2bit.layer_forward_q4 if q4 else moe2bit.layer_forward_mxfp4
    x = torch.from_numpy(synth.make_x_fast(cfg, cfg.T).view(np.int16)).cuda().view(torch.bfloat16)
    y = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device="cuda")
    if q4:
        import ctypes

        n = ctypes.c_size_t(0)
        assert moe2bit.load().moe_workspace_size_q4(ctypes.byref(dl.desc), cfg.T, ctypes.byref(n)) == 0
        ws = torch.empty(max(int(n.value), 16), dtype=torch.uint8, device="cuda")
    else:
        ws = moe2bit.alloc_workspace_mxfp4(dl.desc, cfg.T)
    stream = torch.cuda.current_stream()
    for _ in range(max(args.warmup, 3)):
        forward(dl, x, None, y, ws, stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        forward(dl, x, None, y, ws, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    moe2bit.profile_enable(True)
    for _ in range(steps):
        forward(dl, x, None, y, ws, stream)
    torch.cuda.synchronize()
    prof = moe2bit.profile_read()
    moe2bit.profile_enable(False)
    assert moe2bit.read_status(ws) == 0
    del dl, ws, x, y
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    hbm, bf16_tf, peak_kind = peaks()
    avg_ms = {k: v[0] / max(v[1], 1) for k, v in prof.items()}
    nA = cfg.T * cfg.k
    wb = 0.5 + (2.0 if q4 else 1.0) / 32  # bytes per weight: codes + scales
    flops = 2.0 * nA * 2 * cfg.I * cfg.H
    gu_s = avg_ms["prefill_gateup"] * 1e-3
    if q4:
        alg = cfg.E * 2 * cfg.I * cfg.H * wb + nA * cfg.H * 2 + nA * cfg.I * 2  # weights, fp16 x in, fp16 h out
        dn_alg = cfg.E * cfg.H * cfg.I * wb + nA * cfg.I * 2 + nA * cfg.H * 2
    else:
        alg = cfg.E * 2 * cfg.I * cfg.H * wb + nA * cfg.H * (1 + 1 / 32) + nA * cfg.I * (1 + 1 / 32)
        dn_alg = cfg.E * cfg.H * cfg.I * wb + nA * cfg.I * (1 + 1 / 32) + nA * cfg.H * 4
    fp8_tf = 2.0 * bf16_tf
    hbm_ach = alg / gu_s / 1e9
    if q4:
        tf = flops / gu_s / 1e12
        roof = {"bound": "tensor", "kernel": "prefill_gateup", "achieved": tf, "peak": bf16_tf, "unit": "TFLOP/s",
                "frac": tf / bf16_tf, "peak_source": peak_kind, "algorithmic_flops_per_launch": flops,
                "hbm_frac": hbm_ach / hbm}
    else:
        roof = {"bound": "hbm", "kernel": "prefill_gateup", "achieved": hbm_ach, "peak": hbm, "unit": "GB/s",
                "frac": hbm_ach / hbm, "peak_source": peak_kind, "algorithmic_bytes_per_launch": alg,
                "tensor_frac": flops / gu_s / 1e12 / fp8_tf, "tensor_peak_tflops": fp8_tf}
    roof.update({"avg_launch_ms": avg_ms["prefill_gateup"],
                 "traffic": (traffic_record(cfg.name, "prefill_gateup") or {}).get("bytes_per_launch"),
                 "down_hbm_frac": dn_alg / (avg_ms["prefill_down"] * 1e-3) / 1e9 / hbm})
    return {
        "value": cfg.T / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
        "config": {"workload": cfg.name, "tokens_per_step": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E, "k": cfg.k,
                   "I_s": cfg.Is,
                   "experts": ("Q4-style (32 x 4-bit codes + fp16 d, w = d (q - 8))" if q4 else
                               "MXFP4 (OCP MX: E2M1 x 32 + E8M0)") + ", all three routed matrices",
                   "activations": ("routed: fp16 with a power-of-2 scale per token" if q4 else
                                   "routed: MXFP8 (E4M3 x 32 + E8M0)") + "; shared expert: bf16",
                   "l2": "inputs larger than L2: one resident layer of 6 GB or more", "launch": "stream"},
        "kernels": {k: {"avg_ms": v, "launches_per_step": prof[k][1] / steps} for k, v in avg_ms.items()},
        "roofline": roof,
    }


def measure_quantize(args, reps=3):
    """Float -> 2-bit codes for one expert (gate and up to IQ2, down to Q2K,
    2048 x 7168 weights each): weights per second. The IQ2 search is bound by
    fp32 arithmetic: 256 codebook rows x 8 weights x 3 operations per group of
    8, against 148 SMs x 128 lanes x the median SM clock."""
    import torch

    from bit_quantized_routed_iq2_b200 import moe2bit

    n = 2048 * 7168
    w = torch.randn(n, dtype=torch.float32, device="cuda") / math.sqrt(7168)
    nb = n // 256
    ci = torch.empty((nb, 64), dtype=torch.uint8, device="cuda")
    di = torch.empty(nb, dtype=torch.int16, device="cuda")
    cq = torch.empty((nb, 80), dtype=torch.uint8, device="cuda")
    dq = torch.empty(nb, dtype=torch.int32, device="cuda")
    for _ in range(2):
        moe2bit.quantize_iq2(w, ci, di)
        moe2bit.quantize_q2k(w, cq, dq)
    torch.cuda.synchronize()
    e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    e0.record()
    for _ in range(2 * reps):
        moe2bit.quantize_iq2(w, ci, di)
    e1.record()
    for _ in range(reps):
        moe2bit.quantize_q2k(w, cq, dq)
    e2.record()
    torch.cuda.synchronize()
    ms_iq2 = e0.elapsed_time(e1) / (2 * reps)
    ms_q2k = e1.elapsed_time(e2) / reps
    ms_expert = 2 * ms_iq2 + ms_q2k
    ops = (n // 8) * 256 * 8 * 3
    clk = 1965e6
    peak = 148 * 128 * clk / 1e12
    achieved = ops / (ms_iq2 * 1e-3) / 1e12
    return {
        "value": 3 * n / (ms_expert * 1e-3), "unit": "weights/s", "ms_per_expert": ms_expert,
        "ms_iq2_matrix": ms_iq2, "ms_q2k_matrix": ms_q2k,
        "config": {"workload": "quantize_expert", "matrices": "gate, up (IQ2), down (Q2K)", "rows_x_K": "2048 x 7168"},
        "roofline": {"bound": "alu", "kernel": "quantize_iq2", "achieved": achieved, "peak": peak, "unit": "Tops/s",
                     "frac": achieved / peak,
                     "peak_source": "148 SMs x 128 fp32 lanes x 1965 MHz (nominal clock), unfused fp32 operations"},
    }


def run_ours(args, cfg):
    import torch
    import torch.distributed as dist

    from bit_quantized_routed_iq2_b200 import build as moebuild
    from bit_quantized_routed_iq2_b200 import moe2bit

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    moebuild.build()
    moe2bit.load()

    if args.workloads_only:  # profiling aid: the listed workloads alone, no main line
        assert world == 1 and args.workloads not in ("auto", "all", "none")
        m = {"value": None, "ms_per_step": None, "dtype": None, "gpu_launches": 0,
             **{k: None for k in ("config", "roofline", "step_hbm", "kernels", "clocks", "e2e")}}
    else:
        m = measure(args, cfg, world, rank, local, args.steps)
    line = {
        "metric": "moe_layer_tokens_per_s", "value": m["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": m["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        # routed experts: exact 2-bit integer weights times 12-bit activation digits (two int8 digits) on the
        # decode GEMVs; fp16 operands with fp32 accumulation on the grouped GEMM
        "dtype": m["dtype"], "data": "synthetic",
        **{k: m[k] for k in ("config", "roofline", "step_hbm", "kernels", "gpu_launches", "clocks", "e2e")},
    }
    # the rest of the metric (decode batch, prefill, the 8-layer stack), measured in the same run
    want = args.workloads
    if want == "auto":
        want = "all" if (world == 1 and not args.experts and not args.tokens) else "none"
    if want != "none":
        names = ([n for n in ("decode32", "prefill", "stack") if n != cfg.name] +
                 ["decode1_mxfp4", "decode1_q4", "prefill_mxfp4", "prefill_q4", "decode1_cached", "quantize"]
                 if want == "all"
                 else want.split(","))
        line["workloads"] = {}
        for name in names:
            if name == "decode1_cached":
                w = measure_cached(args, args.workload_steps * 10)
            elif name == "quantize":
                w = measure_quantize(args)
            elif name in ("decode1_mxfp4", "decode1_q4"):
                w = measure_mxfp4(args, args.workload_steps, name.split("_")[1])
            elif name in ("prefill_mxfp4", "prefill_q4"):
                w = measure_blk32_prefill(args, max(3, args.workload_steps // 4), name.split("_")[1])
            else:
                w = measure(args, synth.CONFIGS[name], world, rank, local, args.workload_steps)
                line["gpu_launches"] += w["gpu_launches"]
            line["workloads"][name] = w
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    cfg = synth.CONFIGS[args.config]
    if args.experts:
        cfg = synth.Config(**{**cfg.__dict__, "E": args.experts, "name": f"{cfg.name}_E{args.experts}"})
    if args.tokens:
        cfg = synth.Config(**{**cfg.__dict__, "T": args.tokens, "name": f"{cfg.name}_T{args.tokens}"})
    if args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
