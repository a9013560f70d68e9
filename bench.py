#!/usr/bin/env python3
"""Benchmark: EXL3 trellis GEMV / verify GEMM over a 64-layer 27B-class stack.

One step = one pass of every matrix product of the stack (64 layers x
{q, k, v, o, gate, up, down}, bits per layer drawn from seed 4) at M = 32 rows
(the draft-verification batch), each product running the whole hot path:
input rotation, packed-stream load, trellis decode, contraction, split-K
reduction, scale and output rotation.  The same stack at M = 1 (decode) is
timed too and reported as us/layer.

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
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-budget", type=float, default=None,
                    help="seconds of oracle work per step for --impl reference (default: about 90 s per run)")
    ap.add_argument("--only", default=None,
                    help="restrict the stack to one matrix kind (q,k,v,o,gate,up,down), e.g. for ncu captures")
    return ap.parse_args()


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


KERNEL_SOURCES = ["gemm_exl3_gemv_b200/csrc/gemm_tc.cu", "gemm_exl3_gemv_b200/csrc/exl3_aop.cuh",
                  "gemm_exl3_gemv_b200/csrc/exl3_decode.cuh",
                  "gemm_exl3_gemv_b200/csrc/exl3_common.cuh", "gemm_exl3_gemv_b200/csrc/exl3_tc.cuh"]


def kernel_source_hash():
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic_ratio():
    """DRAM bytes per packed-weight byte of the verify-GEMM kernel, from the
    committed ncu capture in profiles/ -- only if the kernel's sources are the
    ones that capture measured (else None)."""
    p = os.path.join(ROOT, "profiles", "gemm_tc_traffic.json")
    if not os.path.exists(p):
        return None, None
    with open(p) as f:
        d = json.load(f)
    if d.get("source_sha256") != kernel_source_hash():
        return None, None
    return float(d["dram_bytes_per_packed_byte"]), d.get("capture")


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


_INPUT_CACHE = {}


def oracle_sample(budget_s: float, m: int):
    """Time the fp64 oracle on layer-0 matrices (smallest first: k, v, q, o,
    gate, up, down) until `budget_s` is spent; returns (packed bytes, seconds,
    names).  Input generation is outside the timed region."""
    import oracle
    oracle.build()
    specs = [s for s in synth.workload(5, m=m) if s.layer == 0]
    # smallest first so that a short budget still covers at least one matrix
    specs = sorted(specs, key=lambda s: s.n_weights)
    done_b, done_t, names = 0, 0.0, []
    for spec in specs:
        if spec not in _INPUT_CACHE:
            _INPUT_CACHE[spec] = synth.make_inputs(spec)
        inp = _INPUT_CACHE[spec]
        t0 = time.perf_counter()
        oracle.gemm(inp.x, inp.packed, inp.scale, inp.su, inp.sv, spec.k_in, spec.n_out, spec.bits)
        dt = time.perf_counter() - t0
        done_b += spec.packed_bytes
        done_t += dt
        names.append(spec.name)
        if done_t >= budget_s:
            break
    return done_b, done_t, names


def run_reference(args, world, rank):
    if rank != 0:
        return
    os.environ.setdefault("OMP_NUM_THREADS", str(cores_used()))
    steps, warmup = args.steps, args.warmup
    # size each step so the whole run stays within a few minutes
    per_step_budget = args.ref_budget if args.ref_budget is not None else max(1.0, 90.0 / max(1, steps + warmup))
    vals, samples = [], None
    for i in range(warmup + steps):
        b, t, names = oracle_sample(per_step_budget, args.m)
        if i >= warmup:
            vals.append(b / t / 1e9)
        samples = names
    value = statistics.median(vals)
    sample = f"fp64 oracle on layer-0 matrices {','.join(samples)} at M={args.m}, per step"
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
            "n_gpus": args.gpus, "steps": steps, "warmup": warmup, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "m": args.m, "layers": args.layers},
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores_used(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ ours ----

def make_weights(torch, device, layers, only=None):
    """Packed trellis words of the stack, generated on the device (SplitMix64)."""
    specs = [s for s in synth.workload(5, m=32) if s.layer < layers]
    if only:
        specs = [s for s in specs if s.name.split(".")[1] == only]
    return specs, [synth.splitmix64_words_torch(s.stream_id, s.n_words, device) for s in specs]


class Stack:
    """The stack's products.  Inputs x and outputs y of all matrices live in one
    flat device buffer each (and one pinned host buffer each), with a layer's
    matrices contiguous, so that the end-to-end step moves one slice per layer."""

    def __init__(self, ex, torch, device, m, specs, weights):
        self.specs = specs
        self.m = m
        self.mats = []
        ws_need = 0
        x_off, y_off, xo, yo = [], [], 0, 0
        for spec in specs:
            x_off.append(xo)
            y_off.append(yo)
            xo += m * spec.k_in
            yo += m * spec.n_out
        self.x_dev = torch.empty(xo, dtype=torch.float16, device=device)
        self.y_dev = torch.empty(yo, dtype=torch.float16, device=device)
        self.x_pin = torch.empty(xo, dtype=torch.float16).pin_memory()
        self.y_pin = torch.empty(yo, dtype=torch.float16).pin_memory()
        self.large = m > 32
        for i, (spec, packed) in enumerate(zip(specs, weights)):
            scale, x, su, sv = synth.small_inputs(spec)
            if x.shape[0] < m:                          # many-row runs: the synthetic rows repeated
                x = np.tile(x, ((m + x.shape[0] - 1) // x.shape[0], 1))
            t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
            xs = slice(x_off[i], x_off[i] + m * spec.k_in)
            ys = slice(y_off[i], y_off[i] + m * spec.n_out)
            self.x_pin[xs].copy_(torch.from_numpy(np.ascontiguousarray(x[:m]).reshape(-1)))
            self.x_dev[xs].copy_(self.x_pin[xs])
            self.mats.append({"spec": spec, "packed": packed, "scale": t(scale), "su": t(su), "sv": t(sv),
                              "x": self.x_dev[xs].view(m, spec.k_in), "y": self.y_dev[ys].view(m, spec.n_out)})
            ws_need = max(ws_need, int(ex.lib.exl3_large_m_workspace_bytes(m, spec.k_in, spec.n_out, spec.bits))
                          if self.large else ex.workspace_bytes(m, spec.k_in, spec.n_out, spec.bits))
        # per layer: its matrices and its contiguous x and y slices
        self.layers = []
        for i, spec in enumerate(specs):
            if not self.layers or self.layers[-1]["layer"] != spec.layer:
                self.layers.append({"layer": spec.layer, "mats": [], "x0": x_off[i], "y0": y_off[i]})
            lay = self.layers[-1]
            lay["mats"].append(self.mats[i])
            lay["x1"] = x_off[i] + m * spec.k_in
            lay["y1"] = y_off[i] + m * spec.n_out
        self.s_in = torch.cuda.Stream(device=device)
        self.s_out = torch.cuda.Stream(device=device)
        self.ws = torch.zeros(ws_need, dtype=torch.uint8, device=device)
        self.ex = ex
        self.packed_bytes = sum(s.packed_bytes for s in self.specs)
        # the many-row call launches three kernels (decode image, input rotation, GEMM)
        self.launches = sum(3 if self.large else ex.kernel_launches(m, s.k_in, s.n_out, s.bits)
                            for s in self.specs)
        self.io_bytes = sum(2 * m * (s.k_in + s.n_out) + 2 * (s.k_in + 2 * s.n_out) for s in self.specs)
        self.h2d = self.x_pin.numel() * 2
        self.d2h = self.y_pin.numel() * 2

    def run_mats(self, mats):
        ex = self.ex
        call = ex.gemm_large if self.large else ex.gemm
        for mt in mats:
            call(mt["x"], mt["packed"], mt["scale"], mt["su"], mt["sv"], mt["spec"].bits, out=mt["y"],
                 workspace=self.ws)

    def run(self):
        self.run_mats(self.mats)

    def run_e2e(self, torch):
        """One end-to-end step from pinned host buffers: per layer, its inputs go
        up on one stream, its products run on the current stream, its outputs come
        down on a third, so the copies of one layer overlap the products of its
        neighbours.  Every copy is inside the step; the step ends when the last
        output has landed on the host."""
        cs = torch.cuda.current_stream()
        start = torch.cuda.Event()
        start.record(cs)
        self.s_in.wait_event(start)
        self.s_out.wait_event(start)
        for lay in self.layers:
            xs, ys = slice(lay["x0"], lay["x1"]), slice(lay["y0"], lay["y1"])
            with torch.cuda.stream(self.s_in):
                self.x_dev[xs].copy_(self.x_pin[xs], non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(self.s_in)
            cs.wait_event(ev_in)
            self.run_mats(lay["mats"])
            ev_out = torch.cuda.Event()
            ev_out.record(cs)
            self.s_out.wait_event(ev_out)
            with torch.cuda.stream(self.s_out):
                self.y_pin[ys].copy_(self.y_dev[ys], non_blocking=True)
        cs.wait_stream(self.s_in)
        cs.wait_stream(self.s_out)


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

    def max_over_ranks(v):
        if not dist:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    results = {}
    graphs = []
    specs, weights = make_weights(torch, device, args.layers, args.only)
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    for m in ([args.m, 1] if args.m != 1 else [1]):
        st = Stack(ex, torch, device, m, specs, weights)
        st.run()                                        # first call configures kernels
        torch.cuda.synchronize()
        fn = st.run
        launch = "eager"
        if not args.no_graph:
            try:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    st.run()
                graphs.append(g)
                fn = g.replay
                launch = "cuda_graph"
            except Exception as e:  # capture unsupported: time eager launches
                print(f"# graph capture failed ({e}); timing eager launches", file=sys.stderr)
        sampler = ClockSampler(gpu_id) if m == args.m else None
        if sampler:
            sampler.start()
            time.sleep(0.5)                             # let nvidia-smi start sampling
        ms = timed(torch, fn, args.steps, args.warmup, barrier)
        clocks = sampler.stop() if sampler else None
        ms = max_over_ranks(ms)
        res = {"stack": st, "ms": ms, "launch": launch, "clocks": clocks}
        if m == args.m:
            st.run_e2e(torch)
            torch.cuda.synchronize()
            fn_e2e = lambda: st.run_e2e(torch)
            res["e2e_launch"] = "eager"
            if not args.no_graph:
                try:
                    ge = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(ge):
                        st.run_e2e(torch)
                    graphs.append(ge)
                    fn_e2e = ge.replay
                    res["e2e_launch"] = "cuda_graph"
                except Exception as e:  # capture unsupported: time eager launches
                    print(f"# e2e graph capture failed ({e}); timing eager launches", file=sys.stderr)
            res["e2e_ms"] = max_over_ranks(timed(torch, fn_e2e, args.steps, max(1, args.warmup), barrier))
            assert ex.workspace_status(st.ws) == ex.EXL3_OK
            assert torch.equal(st.y_pin, st.y_dev.cpu()), "end-to-end outputs differ from the device outputs"
        results[m] = res
        if m != args.m:
            del st
        torch.cuda.synchronize()

    main = results[args.m]
    st = main["stack"]
    layers = args.layers
    gbs = st.packed_bytes / (main["ms"] * 1e-3) / 1e9
    peak, peak_kind = load_peaks()
    algo_bytes = st.packed_bytes + st.io_bytes
    achieved = algo_bytes / (main["ms"] * 1e-3) / 1e9
    ratio, traffic_src = measured_traffic_ratio() if 1 < args.m <= 32 else (None, None)
    traffic = round(ratio * st.packed_bytes / len(st.specs)) if ratio else None
    line = {
        "metric": METRIC, "value": round(gbs * world, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(main["ms"], 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16-f32acc",
        "data": "synthetic (SplitMix64 packed words, PCG64 activations/scales/signs)",
        "config": {"workload": WORKLOAD if not args.only else f"{WORKLOAD}; only {args.only}",
                   "m": args.m, "layers": layers,
                   "packed_bytes_per_step": st.packed_bytes,
                   "l2": "inputs larger than L2: %.2f GB of packed weights per step" % (st.packed_bytes / 1e9),
                   "launch": main["launch"], "parallelism": f"replicas x{world}"},
        "us_per_layer_m%d" % args.m: round(main["ms"] * 1e3 / layers, 3),
        "pct_of_8TBps": round(100 * gbs / 8000.0, 2),
        "pct_of_measured_hbm": round(100 * gbs / peak, 2),
        "gpu_launches": st.launches * args.steps,
        "e2e": {"value": round(world * st.packed_bytes / (main["e2e_ms"] * 1e-3) / 1e9, 3), "unit": UNIT,
                "h2d_bytes_per_step": st.h2d, "d2h_bytes_per_step": st.d2h,
                "ms_per_step": round(main["e2e_ms"], 4),
                "pipeline": "per layer: H2D stream -> products -> D2H stream, overlapped; " + main["e2e_launch"]},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_kind": peak_kind,
                     "kernel": "verify product (input-rotation pre-pass + gemm_tc_kernel), per product: "
                               "algorithmic bytes / (CUDA-event step time / products)",
                     "algorithmic_bytes_per_product": round(algo_bytes / len(st.specs)),
                     "traffic_source": traffic_src,
                     "launches_per_step": st.launches},
    }
    if st.large:
        # many rows: a dense contraction on the tensor cores (fp16 in, fp32 accumulate)
        flops = sum(2.0 * args.m * s.k_in * s.n_out for s in st.specs)
        tflops = flops / (main["ms"] * 1e-3) / 1e12
        tpeak, tkind = load_tensor_peak()
        line["tflops"] = round(tflops, 1)
        line["roofline"] = {"bound": "tensor", "achieved": round(tflops, 1), "peak": tpeak, "unit": "TFLOP/s",
                            "frac": round(tflops / tpeak, 4), "traffic": None, "peak_kind": tkind,
                            "kernel": "many-row product (decode image + input rotation + tcgen05 GEMM), "
                                      "2 m k n flops per product / (CUDA-event step time / products)",
                            "traffic_source": None, "launches_per_step": st.launches}
    if 1 in results and args.m != 1:
        r1 = results[1]
        line["us_per_layer_m1"] = round(r1["ms"] * 1e3 / layers, 3)
        line["gbs_m1"] = round(st.packed_bytes / (r1["ms"] * 1e-3) / 1e9, 3)
        line["pct_of_measured_hbm_m1"] = round(100 * line["gbs_m1"] / peak, 2)
    if main["clocks"]:
        line["clocks"] = main["clocks"]
    del graphs
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        os.environ.setdefault("OMP_NUM_THREADS", str(cores_used()))
        b, t, names = oracle_sample(15.0, args.m)
        line["cpu_baseline"] = {"value": round(b / t / 1e9, 6), "unit": UNIT, "cores": cores_used(),
                                "kind": "oracle",
                                "sample": f"fp64 oracle, layer-0 matrices {','.join(names)} at M={args.m}"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    world, rank, local = dist_env()
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
