#!/usr/bin/env python3
"""Benchmark: EXL3 trellis GEMV / verify GEMM over a 64-layer 27B-class stack.

One step = one pass of every matrix product of the stack (64 layers x
{q, k, v, o, gate, up, down}, bits per layer drawn from seed 4) at M = 32 rows
(the draft-verification batch), each product running the whole hot path:
input rotation, packed-stream load, trellis decode, contraction, split-K
reduction, scale and output rotation.  Each layer's seven products are one
grouped library call (one rotation pre-pass and one product launch), unless
--separate.  The same stack at M = 1 (decode), 8 and 16 is timed too and
reported as us/layer, and so is the chained stack (each layer's output is the
next layer's input, one CUDA graph) at M = 32 and M = 1.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0).  Value = packed-weight bytes streamed per
second (GB/s), whole job (all ranks).  Under torchrun each rank runs its own
replica of the stack (independent problems, weak scaling, no collective on
the data path); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gemm_exl3_gemv_b200 import synth  # noqa: E402

METRIC = "packed-weight HBM GB/s (% of roofline) and us/layer at M=1 and M=32"
UNIT = "GB/s"
WORKLOAD = "64-layer 27B-class stack (q/k/v/o 5120x5120, 5120x1024 x2, gate/up 5120x17408, down 17408x5120), 2/3/4 bpw per layer from seed 4"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--m", type=int, default=32,
                    help="input rows; above 32 the products go through the many-row (prefill) call, "
                         "with the synthetic rows repeated to m")
    ap.add_argument("--layers", type=int, default=64)
    ap.add_argument("--first-layer", type=int, default=0,
                    help="start the stack at this layer (e.g. a 2-bit layer for a profile capture)")
    ap.add_argument("--separate", action="store_true", help="one library call per matrix instead of per layer")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="time only the main row count (no M=1/8/16, no chain)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-budget", type=float, default=None,
                    help="seconds of oracle work per step for --impl reference (default: about 90 s per run)")
    ap.add_argument("--only", default=None,
                    help="restrict the stack to one matrix kind (q,k,v,o,gate,up,down), e.g. for ncu captures")
    ap.add_argument("--oracle-sample", nargs=2, type=float, default=None, help=argparse.SUPPRESS)
    return ap.parse_args()


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ------------------------------------------------- committed ncu counters ----

def counters(name):
    """A committed ncu counter record (profiles/<name>.json) -- only if the
    kernel sources it was measured on are unchanged (else None, reason)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", name + ".json")
    if not os.path.exists(p):
        return None, "no committed capture"
    with open(p) as f:
        d = json.load(f)
    h = hashlib.sha256()
    for rel in d.get("sources", []):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    if d.get("source_sha256") != h.hexdigest():
        return None, "kernel sources changed since the capture"
    return d, None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def load_tensor_peak():
    """Dense fp16/bf16 tensor peak (the same nominal rate for both), burst."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured (bf16 burst)"
    return 1590.0, "fallback"


# --------------------------------------------------------------- clocks ----

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.path = os.path.join("/tmp", f"exl3_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ reference ----

def cores_used():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


_INPUT_CACHE = {}


def oracle_sample(budget_s: float, m: int):
    """Time the fp64 oracle on layer-0 matrices (smallest first: k, v, q, o,
    gate, up, down) until `budget_s` is spent; returns (packed bytes, seconds,
    [(name, us)]).  Input generation is outside the timed region."""
    import oracle
    oracle.build()
    specs = [s for s in synth.workload(5, m=m) if s.layer == 0]
    specs = sorted(specs, key=lambda s: s.n_weights)
    done_b, done_t, per = 0, 0.0, []
    for spec in specs:
        if spec not in _INPUT_CACHE:
            _INPUT_CACHE[spec] = synth.make_inputs(spec)
        inp = _INPUT_CACHE[spec]
        t0 = time.perf_counter()
        oracle.gemm(inp.x, inp.packed, inp.scale, inp.su, inp.sv, spec.k_in, spec.n_out, spec.bits)
        dt = time.perf_counter() - t0
        done_b += spec.packed_bytes
        done_t += dt
        per.append((spec.name, round(dt * 1e6, 1)))
        if done_t >= budget_s:
            break
    return done_b, done_t, per


def oracle_sample_threads(budget_s: float, m: int, threads: int):
    """oracle_sample in a fresh process limited to `threads` OpenMP threads."""
    env = dict(os.environ, OMP_NUM_THREADS=str(threads))
    out = subprocess.run([sys.executable, os.path.abspath(__file__), "--oracle-sample", str(budget_s), str(m)],
                         env=env, capture_output=True, text=True, timeout=600)
    if out.returncode != 0:
        return None
    return json.loads(out.stdout.strip().splitlines()[-1])


def cpu_baseline(m: int, budget_s: float, single_budget_s: float):
    """The fp64 oracle as it stands, on this host's cores (all, and one)."""
    cores = cores_used()
    allc = oracle_sample_threads(budget_s, m, cores)
    one = oracle_sample_threads(single_budget_s, m, 1)
    if allc is None:
        return None
    layer_bytes = sum(s.packed_bytes for s in synth.workload(5, m=m) if s.layer == 0)
    gbs = allc["bytes"] / allc["seconds"] / 1e9
    d = {"value": round(gbs, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
         "sample": f"fp64 oracle (C, OpenMP) on layer-0 matrices {','.join(n for n, _ in allc['per'])} at M={m}",
         "cpu_model": cpu_model(),
         "us_per_matrix": dict(allc["per"]),
         "us_per_layer_est": round(layer_bytes / (gbs * 1e9) * 1e6, 1)}
    if one is not None:
        g1 = one["bytes"] / one["seconds"] / 1e9
        d["single_thread"] = {"value": round(g1, 6), "unit": UNIT, "us_per_matrix": dict(one["per"]),
                              "us_per_layer_est": round(layer_bytes / (g1 * 1e9) * 1e6, 1)}
    return d


def run_reference(args, world, rank):
    if rank != 0:
        return
    os.environ.setdefault("OMP_NUM_THREADS", str(cores_used()))
    steps, warmup = args.steps, args.warmup
    # size each step so the whole run stays within a few minutes
    per_step_budget = args.ref_budget if args.ref_budget is not None else max(1.0, 90.0 / max(1, steps + warmup))
    vals, samples = [], None
    for i in range(warmup + steps):
        b, t, per = oracle_sample(per_step_budget, args.m)
        if i >= warmup:
            vals.append(b / t / 1e9)
        samples = [n for n, _ in per]
    value = statistics.median(vals)
    sample = f"fp64 oracle on layer-0 matrices {','.join(samples)} at M={args.m}, per step"
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
            "n_gpus": args.gpus, "steps": steps, "warmup": warmup, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "m": args.m, "layers": args.layers},
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores_used(),
                             "kind": "oracle", "sample": sample, "cpu_model": cpu_model()},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ ours ----

def make_weights(torch, device, layers, only=None, first=0):
    """Packed trellis words of the stack, generated on the device (SplitMix64)."""
    specs = [s for s in synth.workload(5, m=32) if first <= s.layer < first + layers]
    if only:
        specs = [s for s in specs if s.name.split(".")[1] == only]
    return specs, [synth.splitmix64_words_torch(s.stream_id, s.n_words, device) for s in specs]


def max_over_ranks(torch, dist, v: float, device) -> float:
    """The largest of every rank's v (all ranks get it); v itself on one rank.
    Each rank's step time is its own CUDA-event measurement; the job's step
    time is the slowest rank's."""
    if dist is None:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def timed(torch, fn, steps, warmup, barrier):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    return e0.elapsed_time(e1) / steps          # ms per step


def time_configs(torch, ex, device, steps, warmup):
    """Workloads 2-4 (single matrices): each matrix timed as single library
    calls replayed from one CUDA graph over R copies of its packed words,
    R chosen so the copies total more than 4x the L2 (no cache reuse between
    calls); us and packed GB/s per call."""
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    out = {}
    for cfg, m_list in ((2, (1,)), (3, (1,)), (4, (8, 16))):
        for m in m_list:
            for spec in synth.workload(cfg):         # workload 4 at M = 8 takes the first 8 of its 16 rows
                R = max(2, -(-4 * l2 // spec.packed_bytes))
                words = torch.stack([synth.splitmix64_words_torch(spec.stream_id, spec.n_words, device)] * R)
                scale, x, su, sv = synth.small_inputs(spec)
                dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
                xs, scs, sus, svs = dev(x[:m]), dev(scale), dev(su), dev(sv)
                y = torch.empty((m, spec.n_out), dtype=torch.float16, device=device)
                ws = ex.alloc_workspace(m, spec.k_in, spec.n_out, spec.bits, device=device)
                run = lambda: [ex.gemm(xs, words[r], scs, sus, svs, spec.bits, out=y, workspace=ws) for r in range(R)]
                run()
                torch.cuda.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    run()
                ms = timed(torch, g.replay, max(3, steps // 4), warmup, lambda: None)
                us = ms * 1e3 / R
                out[f"c{cfg}.m{m}.{spec.name}"] = {"us": round(us, 2), "gbs": round(spec.packed_bytes / (us * 1e-6) / 1e9, 1),
                                                   "shape": f"{spec.k_in}x{spec.n_out}", "bits": spec.bits}
                assert ex.workspace_status(ws) == ex.EXL3_OK
                del g, words
    return out


def run_ours(args, world, rank, local):
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    barrier = (lambda: dist.barrier()) if dist else (lambda: None)

    from gemm_exl3_gemv_b200 import exl3 as ex
    from gemm_exl3_gemv_b200.stack import Stack

    def rank_max(v):
        return max_over_ranks(torch, dist, v, device)

    specs, weights = make_weights(torch, device, args.layers, args.only, args.first_layer)
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    full_layers = args.only is None
    extra = not args.no_extra and args.m <= 32
    rows = [args.m]
    if extra:
        rows += [m for m in (1, 16, 8) if m != args.m]

    def graph_or_eager(st, fn):
        fn()                                            # the configuring first call, outside any capture
        torch.cuda.synchronize()
        if args.no_graph:
            return fn, None, "eager"
        try:
            g = st.capture(fn)
            return g.replay, g, "cuda_graph"
        except Exception as e:  # capture unsupported: time eager launches
            print(f"# graph capture failed ({e}); timing eager launches", file=sys.stderr)
            return fn, None, "eager"

    results = {}
    main_stack = None
    for m in rows:
        st = Stack(ex, torch, device, m, specs, weights, mode="sweep", grouped=not args.separate)
        fn, g, launch = graph_or_eager(st, st.run)
        sampler = ClockSampler(gpu_id) if m == args.m else None
        if sampler:
            sampler.start()
            time.sleep(0.5)                             # let nvidia-smi start sampling
        ms = rank_max(timed(torch, fn, args.steps, args.warmup, barrier))
        clocks = sampler.stop() if sampler else None
        res = {"ms": ms, "launch": launch, "clocks": clocks, "launches": st.launches()}
        if m == args.m:
            # end to end through the binding from pinned host buffers: graphed, then eager
            fe, ge, elaunch = graph_or_eager(st, st.run_e2e)
            res["e2e_ms"] = rank_max(timed(torch, fe, args.steps, max(1, args.warmup), barrier))
            res["e2e_launch"] = elaunch
            res["e2e_eager_ms"] = rank_max(timed(torch, st.run_e2e, args.steps, max(1, args.warmup), barrier))
            assert ex.workspace_status(st.ws) == ex.EXL3_OK
            assert torch.equal(st.y_pin, st.y_dev.cpu()), "end-to-end outputs differ from the device outputs"
            del ge
            main_stack = st
        assert ex.workspace_status(st.ws) == ex.EXL3_OK
        del g
        results[m] = res
        if m != args.m:
            del st
        torch.cuda.synchronize()

    chain = {}
    if extra and full_layers:
        for m in ([args.m, 1] if args.m != 1 else [1]):
            st = Stack(ex, torch, device, m, specs, weights, mode="chain")
            fn, g, launch = graph_or_eager(st, st.run)
            chain[m] = rank_max(timed(torch, fn, args.steps, args.warmup, barrier))
            assert ex.workspace_status(st.ws) == ex.EXL3_OK
            del g, st

    configs = time_configs(torch, ex, device, args.steps, args.warmup) if extra and rank == 0 and world == 1 else None

    main = results[args.m]
    st = main_stack
    layers = len(st.layers)
    gbs = st.packed_bytes / (main["ms"] * 1e-3) / 1e9
    peak, peak_kind = load_peaks()
    algo_bytes = st.packed_bytes + st.io_bytes
    achieved = algo_bytes / (main["ms"] * 1e-3) / 1e9
    n_weights = sum(s.n_weights for s in st.specs)
    sm_mhz = (main["clocks"] or {}).get("sm_mhz") or 1965.0
    # one launch of the dominant kernel = one library call of the step: a whole
    # layer (grouped) or one matrix (separate calls)
    per_launch = len(st.layers) if st.grouped else len(st.specs)

    def issue_record(m, ms):
        """Instruction-issue roofline: committed instructions per weight (ncu)
        x weights/s against 4 issue slots x 148 SMs x the sampled clock x 32 lanes."""
        c, why = counters("gemv_m1_counters" if m == 1 else "gemm_tc_counters")
        if c is None or "thread_instructions_per_weight" not in c:
            return {"bound": "alu-issue", "frac": None, "why": why}, c, why
        ipw = float(c["thread_instructions_per_weight"])
        wps = n_weights / (ms * 1e-3)
        peak_ti = 4 * 148 * sm_mhz * 1e6 * 32
        return ({"bound": "alu-issue", "instr_per_weight": ipw, "weights_per_s_T": round(wps / 1e12, 4),
                 "achieved": round(ipw * wps / 1e12, 3), "peak": round(peak_ti / 1e12, 3),
                 "unit": "T thread-instr/s", "frac": round(ipw * wps / peak_ti, 4), "sm_mhz": sm_mhz,
                 "source": c.get("capture")}, c, None)

    if args.m <= 32:
        issue, cnt, cnt_why = issue_record(args.m, main["ms"])
    else:
        issue, cnt, cnt_why = {"bound": "alu-issue", "frac": None, "why": "many-row path"}, None, "many-row path"
    traffic = None
    if cnt is not None and "dram_bytes_per_packed_byte" in cnt:
        traffic = round(cnt["dram_bytes_per_packed_byte"] * st.packed_bytes / per_launch)
    line = {
        "metric": METRIC, "value": round(gbs * world, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(main["ms"], 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16-f32acc",
        "data": "synthetic (SplitMix64 packed words, PCG64 activations/scales/signs)",
        "config": {"workload": WORKLOAD if not args.only else f"{WORKLOAD}; only {args.only}",
                   "m": args.m, "layers": layers,
                   "packed_bytes_per_step": st.packed_bytes,
                   "l2": "inputs larger than L2: %.2f GB of packed weights per step" % (st.packed_bytes / 1e9),
                   "calls": "one grouped call per layer" if st.grouped else "one call per matrix",
                   "launch": main["launch"], "parallelism": f"replicas x{world}"},
        "us_per_layer_m%d" % args.m: round(main["ms"] * 1e3 / layers, 3),
        "pct_of_8TBps": round(100 * gbs / 8000.0, 2),
        "pct_of_measured_hbm": round(100 * gbs / peak, 2),
        "gpu_launches": main["launches"] * args.steps,
        "e2e": {"value": round(world * st.packed_bytes / (main["e2e_ms"] * 1e-3) / 1e9, 3), "unit": UNIT,
                "h2d_bytes_per_step": st.h2d, "d2h_bytes_per_step": st.d2h,
                "ms_per_step": round(main["e2e_ms"], 4),
                "pipeline": "inputs up in growing chunks of layers, products, outputs down in shrinking chunks, on three streams, overlapped; " + main["e2e_launch"],
                "eager": {"value": round(world * st.packed_bytes / (main["e2e_eager_ms"] * 1e-3) / 1e9, 3),
                          "ms_per_step": round(main["e2e_eager_ms"], 4),
                          "launch": "eager: every library call through the binding and the C ABI each step"}},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_kind": peak_kind,
                     "kernel": ("verify product (rotation pre-pass + gemm_tc_kernel)" if args.m > 1 else
                                "single-row product (gemv_m1_kernel)") +
                               ": algorithmic bytes per step / CUDA-event step time; one launch = " +
                               ("one grouped layer call" if st.grouped else "one matrix"),
                     "algorithmic_bytes_per_launch": round(algo_bytes / per_launch),
                     "traffic_per": "launch (measured DRAM bytes per packed byte x the launch's packed bytes)",
                     "traffic_source": cnt.get("capture") if cnt else cnt_why,
                     "launches_per_step": main["launches"],
                     "issue": issue},
    }
    if st.large:
        flops = sum(2.0 * args.m * s.k_in * s.n_out for s in st.specs)
        tflops = flops / (main["ms"] * 1e-3) / 1e12
        tpeak, tkind = load_tensor_peak()
        line["tflops"] = round(tflops, 1)
        line["roofline"] = {"bound": "tensor", "achieved": round(tflops, 1), "peak": tpeak, "unit": "TFLOP/s",
                            "frac": round(tflops / tpeak, 4), "traffic": None, "peak_kind": tkind,
                            "kernel": "many-row product (decode image + input rotation + tcgen05 GEMM), "
                                      "2 m k n flops per product / (CUDA-event step time / products)",
                            "traffic_source": None, "launches_per_step": main["launches"]}
    m1_ms = results[1]["ms"] if 1 in results else None
    for m, r in results.items():
        if m == args.m:
            continue
        line["us_per_layer_m%d" % m] = round(r["ms"] * 1e3 / layers, 3)
        line["gbs_m%d" % m] = round(st.packed_bytes / (r["ms"] * 1e-3) / 1e9, 3)
    if m1_ms:
        line["pct_of_measured_hbm_m1"] = round(100 * line.get("gbs_m1", gbs) / peak, 2)
        if args.m != 1:
            io1 = sum(2 * (s.k_in + s.n_out) + 2 * (s.k_in + 2 * s.n_out) for s in st.specs)
            line["roofline_m1"] = {"bound": "hbm", "achieved": round((st.packed_bytes + io1) / (m1_ms * 1e-3) / 1e9, 2),
                                   "peak": peak, "unit": "GB/s", "kernel": "gemv_m1_kernel (one grouped call per layer)",
                                   "issue": issue_record(1, m1_ms)[0]}
            line["roofline_m1"]["frac"] = round(line["roofline_m1"]["achieved"] / peak, 4)
        line["step_vs_m1"] = {("m%d" % m): round(r["ms"] / m1_ms, 3) for m, r in results.items() if m != 1}
    for m, ms in chain.items():
        line["us_per_layer_chain_m%d" % m] = round(ms * 1e3 / layers, 3)
    if configs:
        line["configs_2_to_4"] = configs
    if main["clocks"]:
        line["clocks"] = main["clocks"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(args.m, 12.0, 6.0)
        if cb:
            line["cpu_baseline"] = cb
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    if args.oracle_sample is not None:
        b, t, per = oracle_sample(args.oracle_sample[0], int(args.oracle_sample[1]))
        print(json.dumps({"bytes": b, "seconds": t, "per": per}))
        return
    world, rank, local = dist_env()
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
