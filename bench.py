#!/usr/bin/env python
"""Benchmark of the fused decode FFN half-layer ("mono" kernel) on B200.

One step = one fused MoE layer-step of the chosen workload (all rows, every
stage of the layer, n_layers persistent launches).  Inputs are seeded and
synthetic; the weights are generated on the device and packed before timing.
L2 is flushed before every timed step (a 512 MiB write, then a 512 MiB read,
so that the write-back of the flush's dirty lines is not charged to the
step), and four hc_in sets rotate so the routed experts change from step to
step.

Prints ONE JSON line (rank 0).  Its headline (`value`, `roofline`, `e2e`)
is the --config workload (default: the bf16 layer at one row); `per_config`
then holds every configuration of the metric (rows 1, 6 and 8 bf16, FP8 at
4 rows, the 4-layer MXFP4 chain at 8 rows), each timed the same way, with
the CPU oracle on a bounded sample at one thread and on every host core.
`--impl reference` times the CPU oracle on a bounded sample of the same
workload instead.
"""

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "µs per fused MoE layer-step and achieved HBM GB/s (% of peak), rows=1..8"
UNIT = "us/layer-step"
FLUSH_BYTES = 512 << 20
N_INPUT_SETS = 4
KERNEL_SOURCES = ["moe_decode_layer_sm_b200/csrc/mono_ffn.cu", "moe_decode_layer_sm_b200/csrc/common.cuh",
                  "moe_decode_layer_sm_b200/csrc/cc_kernel.cuh", "moe_decode_layer_sm_b200/csrc/tc_kernel.cuh",
                  "moe_decode_layer_sm_b200/csrc/ptx.cuh", "moe_decode_layer_sm_b200/csrc/tq_kernel.cuh"]


def kernel_sha():
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


L2_MODE = ["flush"]
TRACE_DUMP = [None]


def workload(name):
    from synth import configs as C
    return C.BY_NAME[name]


def wl_config(wl, extra=None):
    cfg = {"workload": wl.name, "rows": wl.rows, "hidden": wl.hidden, "hc_streams": wl.hc,
           "routed_experts": wl.n_routed, "top_k": wl.top_k, "shared_experts": 1, "inter": wl.inter,
           "layers_per_step": wl.n_layers, "expert_format": wl.w_dtype, "hc_format": wl.hc_dtype,
           "activations": "mxfp8 (e4m3, e8m0 per 32)" if getattr(wl, "act_mx8", False) else "as the layer defines",
           "l2": "flushed before every timed step (512 MiB write, then a 512 MiB read so that the "
                 "written lines are back in HBM and L2 holds only clean lines of an unrelated buffer)"
                 if L2_MODE[0] == "flush" else
                 "not flushed: every step streams its weights (larger than the 126 MB L2) through it",
           "inputs": f"{N_INPUT_SETS} rotating seeded hc_in sets"}
    if extra:
        cfg.update(extra)
    return cfg


def dtype_of(wl):
    d = {"f32": "f32", "bf16": "bf16", "fp8": "fp8e4m3", "mxfp4": "mxfp4"}[wl.w_dtype]
    return d + "+mxfp8act" if getattr(wl, "act_mx8", False) else d


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"mono_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        self.proc.wait()
        self.f.close()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------ CPU baseline --

def _omp_threads(n):
    """Thread count of the oracle's OpenMP regions started from this thread."""
    import ctypes
    try:
        ctypes.CDLL("libgomp.so.1").omp_set_num_threads(int(n))
        return True
    except OSError:
        return False


def _oracle_case(wl):
    """The oracle's inputs for a bounded sample of the workload: the whole
    step when it has one row and one layer, else row 0 of layer 0 (the
    oracle works row by row, so a row's time times the rows is the step's,
    per layer).  Only the experts the sample touches are generated, before
    any clock starts.  Returns (layer weights, hc rows, scale, description)."""
    from oracle import oracle as O
    from synth import synth as S
    hc = S.cpu_hc_in(wl)
    scale = 1
    what = f"one full layer-step of {wl.name} ({wl.rows} rows)"
    if wl.rows > 1 or wl.n_layers > 1:
        hc = hc[:1]
        scale = wl.rows
        what = (f"row 0 of layer 0 of {wl.name}, times {wl.rows} rows (the oracle computes rows one by one)")
    w1 = wl.with_(rows=hc.shape[0])
    dense = S.cpu_dense(wl, 0)
    t = O.route(w1, O.LayerWeights(w1, dense, {}), hc)
    slots = sorted(set(int(e) for e in t.idx.ravel()) | {wl.n_routed})
    lw = O.LayerWeights(w1, dense, {e: S.cpu_expert(wl, 0, e) for e in slots})
    return w1, lw, hc, scale, what


def cpu_oracle_sample(wl, budget_s=12.0, threads=None, case=None):
    """Time the CPU oracle (as it stands) on a bounded sample of the
    workload (_oracle_case), in µs per layer-step.  threads: None = every
    host core, else that many OpenMP threads.  Repeats (up to 5) while the
    budget lasts; the median counts."""
    from oracle import oracle as O
    w1, lw, hc, scale, what = case if case is not None else _oracle_case(wl)
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    if threads is not None and _omp_threads(threads):
        cores = threads
    elif threads is None:
        _omp_threads(cores)
    O.layer(w1, lw, hc)   # untimed: first touch of the weights
    times = []
    t_end = time.time() + budget_s
    while time.time() < t_end or not times:
        t0 = time.perf_counter()
        O.layer(w1, lw, hc)
        times.append(time.perf_counter() - t0)
        if len(times) >= 5:
            break
    _omp_threads(int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1)))
    us = statistics.median(times) * 1e6 * scale
    return {"value": us, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{what}; median of {len(times)}; touched experts generated before timing"}


def cpu_baselines(wl, budget_s=12.0):
    """The oracle on every host core and on one thread, same sample."""
    case = _oracle_case(wl)
    return {"all_cores": cpu_oracle_sample(wl, budget_s, None, case),
            "one_thread": cpu_oracle_sample(wl, budget_s, 1, case)}


def parallelism(world):
    return "replicas" if world > 1 else "none (one replica)"


def run_reference(args):
    """The oracle, as it stands, on the host cores: W untimed steps, then
    exactly K timed steps, each one layer step of the bounded sample
    (_oracle_case: the whole step at one row, else row 0 scaled to the
    rows).  Rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import oracle as O
    wl = workload(args.config)
    w1, lw, hc, scale, what = _oracle_case(wl)
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    _omp_threads(cores)
    O.layer(w1, lw, hc)   # first touch of the weights
    for _ in range(args.warmup):
        O.layer(w1, lw, hc)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        O.layer(w1, lw, hc)
        times.append(time.perf_counter() - t0)
    us = sum(times) / len(times) * 1e6 * scale
    cb = {"value": us, "unit": UNIT, "cores": cores, "kind": "oracle",
          "sample": f"{what}; {args.warmup} warm-up and {args.steps} timed steps, mean; touched experts generated "
                    f"before timing"}
    line = {"metric": METRIC, "value": cb["value"], "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": cb["value"] / 1000.0, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generator)",
            "config": wl_config(wl, {"parallelism": parallelism(args.gpus)}), "impl": "reference",
            "cpu_baseline": cb, "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------- GPU path --

TRACE_NAMES = ["start", "mix published", "mix totals seen", "n ready", "logits published", "lists ready",
               "shared gate/up done", "routed gate/up done", "1st down expert ready", "down done", "end",
               "producer saw lists", "producer issued all", "issuer: 1st routed stage", "issuer: routed issued",
               "issuer: 1st down operand", "issuer: all issued", "mix: partials computed", "producer: 1st routed",
               "producer: 1st down", "epilogue: 1st shared", "ctl: logits complete", "ctl: top-k done",
               "pre/post ready", "collapse: all slices", "router: dots done", "top-k: loads done",
               "collapse: slice out", "mix: inputs in smem", "collapse: slices in smem", "norm: n done"]
TRACE_POINTS = 32


def print_trace(plan, wl, sets, out, flush_l2):
    """One extra traced step: stage timestamps relative to the earliest CTA
    start, min / median / max over CTAs (µs), to stderr."""
    import numpy as np
    import torch
    info = plan.info()
    G = info["grid"]
    buf = torch.zeros(wl.n_layers * G * TRACE_POINTS, dtype=torch.int64, device="cuda")
    plan.set_trace(buf)
    flush_l2()
    plan.step(wl.rows, sets[0], out)
    torch.cuda.synchronize()
    plan.set_trace(None)
    t = buf.view(wl.n_layers, G, TRACE_POINTS).cpu().numpy().astype("float64")
    if TRACE_DUMP[0]:
        np.save(TRACE_DUMP[0], t)
    for l in range(wl.n_layers):
        t0 = t[l, :, 0].min()
        print(f"layer {l}: stage times in us from the first CTA start (min / median / max over CTAs)", file=sys.stderr)
        for i, nm in enumerate(TRACE_NAMES[:31]):
            col = t[l, :, i]
            col = col[col > 0]
            if len(col) == 0:
                continue
            d = (col - t0) / 1000.0
            print(f"  {i:2d} {nm:22s} {d.min():9.2f} {statistics.median(d):9.2f} {d.max():9.2f}  (n={len(col)})",
                  file=sys.stderr)

def job_times(tot_ms, tot_e2e, world, device):
    """Max over ranks of each rank's timed totals (ms).  Every rank calls it,
    at the same point, on the initialised process group."""
    if world > 1:
        import torch
        import torch.distributed as dist
        t = torch.tensor([tot_ms, tot_e2e], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        tot_ms, tot_e2e = t.tolist()
    return tot_ms, tot_e2e


def job_value(tot_ms, steps, layers, world):
    """µs per layer-step of the whole job: the layer-steps of all ranks in the
    max-over-ranks time (replicas: the work grows with the ranks)."""
    return tot_ms * 1000.0 / steps / layers / world


PER_CONFIG = ["v41flash-bf16-r1", "v41flash-bf16-r6", "v41flash-bf16-r8", "v41flash-fp8b128-r4",
              "v41flash-mxfp4-chain4-r8", "v41flash-mxfp4-mx8act-chain4-r8"]


def traffic_of(wl):
    """ncu DRAM bytes per launch from profiles/, if captured at these sources."""
    tr_path = os.path.join(ROOT, "profiles", f"traffic_{wl.name}.json")
    if os.path.exists(tr_path):
        tr = json.load(open(tr_path))
        if tr.get("kernel_sha") == kernel_sha():
            return tr.get("dram_bytes_per_launch")
    return None


def measure(wl, args, ctx):
    """Plan, pack and time one workload: K steps with inputs resident (CUDA
    events on the launching stream, L2 flushed before each), then K steps
    end to end through mono_ffn_step_host.  Every rank runs it at the same
    point (the barriers and the max over ranks)."""
    import numpy as np
    import torch

    from moe_decode_layer_sm_b200 import Plan
    from synth import synth as S
    rank, world, local, barrier, flush_l2 = ctx["rank"], ctx["world"], ctx["local"], ctx["barrier"], ctx["flush"]
    plan = Plan.for_workload(wl, device=local)
    info = plan.info()
    for l in range(wl.n_layers):
        d = S.gpu_dense(wl, l)
        ex = S.gpu_experts(wl, l)
        plan.pack(l, d["mix_w"], d["norm_w"], d["router_w"], d["router_bias"], ex["gate"][0], ex["up"][0],
                  ex["down"][0], ex["gate"][1], ex["up"][1], ex["down"][1])
        torch.cuda.synchronize()
        del ex, d
        torch.cuda.empty_cache()
    # input sets: seeds differ per set and per rank (independent replicas)
    sets = [S.gpu_hc_in(wl.with_(seed=wl.seed + 1000 * i + 7919 * rank)) for i in range(N_INPUT_SETS)]
    out = torch.empty_like(sets[0])
    idx_taps = [torch.zeros((wl.rows, wl.top_k), dtype=torch.int32, device="cuda") for _ in range(wl.n_layers)]
    for l in range(wl.n_layers):
        plan.set_taps(l, idx=idx_taps[l])
    # unique experts touched per input set (for the byte count)
    uniq = []
    for i in range(N_INPUT_SETS):
        plan.step(wl.rows, sets[i], out)
        rc, st = plan.query_error()
        if rc != 0:
            raise SystemExit(f"device error {rc} stage {st.stage}")
        uniq.append([len(set(t.cpu().numpy().ravel().tolist())) for t in idx_taps])
    for l in range(wl.n_layers):
        plan.clear_taps(l)
    hc_bytes = wl.rows * wl.hc * wl.hidden * (2 if wl.hc_dtype == "bf16" else 4)
    bytes_per_set = [sum(info["dense_bytes"] + (u + 1) * info["expert_bytes"] + 2 * hc_bytes for u in us)
                     for us in uniq]
    stream = torch.cuda.current_stream()
    for k in range(args.warmup):
        flush_l2()
        plan.step(wl.rows, sets[k % N_INPUT_SETS], out)
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed")   # lets a profiler capture exactly the timed launches
    for k in range(K):
        flush_l2()
        ev[k][0].record(stream)
        plan.step(wl.rows, sets[k % N_INPUT_SETS], out)
        ev[k][1].record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]

    # end to end through the host-buffer entry point: H2D of the step's hc_in
    # from pinned memory, the step, D2H of the result, per step
    host_in = [x.cpu().pin_memory() for x in sets]
    host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    KE = min(K, args.e2e_steps)
    ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(KE)]
    barrier()
    torch.cuda.synchronize()
    for k in range(KE):
        flush_l2()
        ev2[k][0].record(stream)
        plan.step_host(wl.rows, host_in[k % N_INPUT_SETS], host_out)
        ev2[k][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = [a.elapsed_time(b) for a, b in ev2]
    clk = clocks.stop()
    if args.trace:
        print_trace(plan, wl, sets, out, flush_l2)
    rc, st = plan.query_error()
    if rc != 0:
        raise SystemExit(f"device error {rc} stage {st.stage}")
    plan.close()
    del plan, sets, out, host_in, host_out
    torch.cuda.empty_cache()

    tot_ms, tot_e2e = job_times(sum(step_ms), sum(e2e_ms), world, "cuda")
    mean_bytes = sum(bytes_per_set[k % N_INPUT_SETS] for k in range(K)) / K
    achieved = mean_bytes / (tot_ms / 1000.0 / K) / 1e9
    pk, pk_kind = peaks()
    return {
        "workload": wl.name, "rows": wl.rows, "layers_per_step": wl.n_layers, "expert_format": wl.w_dtype,
        "value": job_value(tot_ms, K, wl.n_layers, world), "unit": UNIT, "ms_per_step": tot_ms / K,
        "step_us_p10_p50_p90": [float(np.percentile(step_ms, q)) * 1000.0 for q in (10, 50, 90)],
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / pk["hbm_gbs"], "traffic": traffic_of(wl),
                     "peak_kind": f"{pk_kind} HBM copy", "frac_of_8tbs_nominal": achieved / 8000.0,
                     "algorithmic_bytes_per_step": mean_bytes,
                     "unique_routed_experts_per_layer": statistics.mean(x for us in uniq for x in us)},
        "e2e": {"value": job_value(tot_e2e, KE, wl.n_layers, world), "unit": UNIT, "h2d_bytes_per_step": hc_bytes,
                "d2h_bytes_per_step": hc_bytes},
        "gpu_launches": K * wl.n_layers,
        "clocks": clk,
        "plan": {k: info[k] for k in ("grid", "threads", "smem_bytes", "ring_stages", "ring_slot_bytes")},
    }


def run_gpu(args):
    import torch
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    flush_rd = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    flush_acc = torch.zeros((), dtype=torch.float32, device="cuda")

    def flush_l2():
        # a write pass evicts everything, a read pass then writes the dirty
        # lines back before the timed region instead of inside it
        if args.l2 == "flush":
            flush.zero_()
            torch.sum(flush_rd, dim=0, out=flush_acc)

    ctx = {"rank": rank, "world": world, "local": local, "barrier": barrier, "flush": flush_l2}
    wl = workload(args.config)
    if args.routed:
        wl = wl.with_(name=f"{wl.name}-e{args.routed}", n_routed=args.routed)
    if args.inter:
        wl = wl.with_(name=f"{wl.name}-i{args.inter}", inter=args.inter)
    head = measure(wl, args, ctx)
    others = []
    if not args.no_per_config and not args.routed and not args.inter:
        # every configuration of the metric (rows = 1..8, each expert format),
        # in the same run, each with its own plan
        for name in PER_CONFIG:
            if name != wl.name:
                others.append(measure(workload(name), args, ctx))
    cpu_on = rank == 0 and world == 1 and not args.no_cpu_baseline
    line = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": dtype_of(wl),
        "data": "synthetic (seeded generator, random-init weights of the layer's shape)",
        "config": wl_config(wl, {"parallelism": parallelism(world)}),
        "roofline": head["roofline"], "e2e": head["e2e"], "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"], "step_us_p10_p50_p90": head["step_us_p10_p50_p90"], "plan": head["plan"],
    }
    if cpu_on:
        cb = cpu_baselines(wl)
        line["cpu_baseline"] = cb["all_cores"]
        line["cpu_baseline_one_thread"] = cb["one_thread"]
    if others or cpu_on:
        per = {}
        for m in [head] + others:
            entry = {k: m[k] for k in ("rows", "layers_per_step", "expert_format", "value", "unit",
                                       "step_us_p10_p50_p90", "roofline", "e2e", "clocks")}
            if cpu_on:
                entry["cpu_baseline"] = cpu_baselines(workload(m["workload"])) if m is not head else \
                    {"all_cores": line["cpu_baseline"], "one_thread": line["cpu_baseline_one_thread"]}
            per[m["workload"]] = entry
        line["per_config"] = per
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="mono", choices=["mono", "reference"])
    ap.add_argument("--config", default="v41flash-bf16-r1")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only --config (by default every configuration of the metric follows it)")
    ap.add_argument("--routed", type=int, default=0, help="override the routed-expert count (small profiling cases)")
    ap.add_argument("--inter", type=int, default=0, help="override the expert width (small profiling cases)")
    ap.add_argument("--trace-dump", default=None, help="with --trace: save the raw [layers][grid][32] stamps (.npy)")
    ap.add_argument("--trace", action="store_true", help="print per-stage device timestamps (stderr) after the run")
    ap.add_argument("--l2", default="flush", choices=["flush", "none"],
                    help="flush: write, then read, 512 MiB before every step; none: rely on the step's weights "
                         "exceeding L2")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    L2_MODE[0] = args.l2
    TRACE_DUMP[0] = args.trace_dump
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
