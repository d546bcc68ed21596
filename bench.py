"""Benchmark of the int4 expert-grouped MoE layer on B200.

One step = one whole MoE layer (routing, top-k, prefix scan, scatter, block
map, gate/up grouped GEMM with SwiGLU, down grouped GEMM with the weighted
combine, bf16 output) over one batch of seeded synthetic tokens, through the
C-ABI entry point moe_forward_timed.  Default workload: the 8192-token
prefill layer (d=2048, E=128, k=8, f=768, int4 group 64).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   (the CPU oracle, timed on host cores)

With N > 1 (torchrun, one process per GPU) every rank runs its own replica of
the layer on its own batch: the token batches are independent and the
weights are replicated, so there is no collective on the data path
("replicas only", weak scaling); timing is the max over ranks.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402

METRIC = "MoE-layer prefill tokens/s (int4 fused grouped GEMM) and % of roofline"
L2_FLUSH_BYTES = 256 << 20  # > 126 MB L2
L2_BYTES = 126 << 20
# kernels one layer call launches, by moe_forward_path: fp32 router (logits,
# top-k), scan, scatter, dispatch, gate/up GEMM, down GEMM, combine; the
# small-batch kernel; the int8 tensor-core router (prep, approximate logits,
# selection) and the rest as for the first
KERNELS_PER_PATH = {0: 8, 1: 1, 2: 9}


def build_library():
    """Compile libmoe_b200.so when its sources are newer (build.py by path:
    the package refuses to import until the library exists)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "moe_libbuild", os.path.join(ROOT, "int4_expert_grouped_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def workload_desc(name, s, seed, zipf):
    kind = "decode" if s.T <= 8 else "prefill"
    return ("%s T=%d, d=%d, E=%d, top-k=%d, f=%d, int4 group %d, SwiGLU, seed %d%s"
            % (kind, s.T, s.d, s.E, s.k, s.f, s.group, seed, ", Zipf(1.1) router bias" if zipf else ""))


def algorithmic(s, counts):
    """Algorithmic work of one layer: GEMM flops and int4-weight + activation bytes."""
    touched = int(np.count_nonzero(counts))
    per_expert = 3 * s.f * s.d // 2 + 3 * s.f * (s.d // s.group) * 4
    flops_gateup = 4.0 * s.T * s.k * s.d * s.f
    flops_down = 2.0 * s.T * s.k * s.d * s.f
    bytes_layer = touched * per_expert + 2 * s.T * s.d * 2
    bytes_gateup = touched * (2 * s.f * s.d // 2 + 2 * s.f * (s.d // s.group) * 4) \
        + s.T * s.d * 2 + s.T * s.k * s.f * 2
    return dict(touched=touched, per_expert=per_expert, flops_gateup=flops_gateup,
                flops_down=flops_down, flops=flops_gateup + flops_down, bytes=bytes_layer,
                bytes_gateup=bytes_gateup)


class ColdL2:
    """Keeps every timed step's weights cold in L2.

    Layers that touch more weight bytes than L2 holds get a 256 MiB write
    before each step (outside the step's events); the write also keeps the
    stream busy while the host enqueues the step.  Layers that touch few
    (the small batches: 8 experts, 21 MB at one token) instead rotate over R
    copies of the packed weights and W_r, R - 1 >= 2 x L2 / touched bytes, so
    that each step reads a copy whose bytes left L2 R - 1 steps ago; no
    other kernel runs between two steps."""

    def __init__(self, layer, work, flush):
        import torch
        self.layer, self.flush = layer, flush
        self.packs = self.wrs = None
        touched = work["bytes"]
        if 4 * work["touched"] <= layer.E and touched < L2_BYTES:
            r = 1 + -(-2 * L2_BYTES // touched)
            self.packs = [layer.packed] + [layer.packed.clone() for _ in range(r - 1)]
            self.wrs = [layer.w_r] + [layer.w_r.clone() for _ in range(r - 1)]
            torch.cuda.synchronize()
            self.desc = ("weights rotated over %d copies of the packed experts and W_r (%.1f GB), "
                         "each step's %.1f MB cold in L2; no flush kernel" %
                         (r, r * layer.packed.numel() / 1e9, touched / 1e6))
        else:
            self.desc = "flushed between steps (256 MiB write outside the step events)"

    def before(self, i):
        import torch
        if self.packs is None:
            self.flush.fill_(i & 0xFF)
        else:
            self.layer.packed = self.packs[i % len(self.packs)]
            self.layer.w_r = self.wrs[i % len(self.wrs)]
            # keep the stream busy while the host enqueues the step, so that
            # the step's start event is taken when the GPU reaches it, not
            # while the host is still launching (about 25 us of spinning)
            torch.cuda._sleep(50000)

    def release(self):
        if self.packs is not None:
            self.layer.packed, self.layer.w_r = self.packs[0], self.wrs[0]
            self.packs = self.wrs = None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled while the timed loop runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def cpu_oracle_rate(inp, budget_s=15.0, min_tokens=16):
    """Time the CPU oracle (as it stands) on the first tokens of the workload,
    growing the sample until it takes a few seconds; returns tokens/s."""
    import oracle
    s = inp.shape
    n = min(min_tokens, s.T)
    while True:
        sub = mi.Inputs(mi.Shape(n, s.d, s.E, s.k, s.f, s.group), inp.seed, inp.x[:n], inp.w_r,
                        inp.b_r, inp.gate, inp.up, inp.down)
        t0 = time.perf_counter()
        oracle.forward(sub)
        dt = time.perf_counter() - t0
        if dt >= budget_s / 4 or n >= s.T:
            return n / dt, n, dt
        n = min(s.T, max(n * 2, int(n * budget_s / 4 / max(dt, 1e-3))))


def run_reference(args, name):
    shape, seed, zipf = mi.WORKLOADS[name]
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = mi.workload(name)
    import oracle
    cores = os.cpu_count()
    rate, n, dt = cpu_oracle_rate(inp, budget_s=8.0)
    # each step: the oracle on a bounded sample of n tokens of the workload
    sub = mi.Inputs(mi.Shape(n, shape.d, shape.E, shape.k, shape.f, shape.group), seed,
                    inp.x[:n], inp.w_r, inp.b_r, inp.gate, inp.up, inp.down)
    for _ in range(args.warmup):
        oracle.forward(sub)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.forward(sub)
    total = time.perf_counter() - t0
    value = args.steps * n / total
    sample = "first %d tokens of the workload per step (CPU oracle, float64, OpenMP)" % n
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(name, shape, seed, zipf), "tokens_per_step": n},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def layer_launches(layer, T):
    """Kernels one layer call launches (the library's launch sequence)."""
    return KERNELS_PER_PATH[layer.plan.forward_path(T)]


def max_over_ranks(value, world, device="cuda"):
    """The largest of every rank's value (the slowest rank sets a replicated
    step's time); every rank must call it, in the same order."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def time_layer(layer, x, y, K, repeats, cold, stream, world=1):
    """K layer calls with the weights cold in L2 (`cold`), `repeats` times.

    Each call is bracketed by two CUDA events on the launching stream (the
    L2 flush, when there is one, runs before the first); returns the
    per-repeat mean step times (ms, max over ranks) and their median.  The
    per-stage split comes from a separate pass (stage_times): the four events
    moe_forward_timed records inside a call add their own gaps, a few us
    each, which the step time must not carry."""
    import torch
    import torch.distributed as dist
    reps = []
    for _ in range(repeats):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for i in range(K):
            cold.before(i)  # outside the step's events
            evs[i][0].record(stream)
            layer.forward(x, y)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        total = max_over_ranks(float(sum(r[0].elapsed_time(r[1]) for r in evs)), world)
        reps.append(total / K)
    return reps, sorted(reps)[repeats // 2]


def stage_times(layer, x, y, K, cold, stream):
    """Mean stage times (ms) over K calls of moe_forward_timed, which records
    events after routing, after each GEMM and after the combine.  The
    small-batch kernel is one launch: its whole time is under "routing"."""
    import torch
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    for row in evs:
        for e in row:
            e.record(stream)  # create the handles before they are passed to the C API
    torch.cuda.synchronize()
    for i in range(K):
        cold.before(i)
        layer.forward(x, y, events=evs[i])
    torch.cuda.synchronize()
    return {
        "routing": float(np.mean([r[0].elapsed_time(r[1]) for r in evs])),
        "gate_up_gemm": float(np.mean([r[1].elapsed_time(r[2]) for r in evs])),
        "down_gemm": float(np.mean([r[2].elapsed_time(r[3]) for r in evs])),
        "combine": float(np.mean([r[3].elapsed_time(r[4]) for r in evs])),
    }


def layer_roofline(work, ms, peaks):
    t_tensor = work["flops"] / (peaks["bf16_tflops"] * 1e12)
    t_hbm = work["bytes"] / (peaks["hbm_gbs"] * 1e9)
    roof = max(t_tensor, t_hbm)
    return {"frac": roof / (ms * 1e-3), "time_us": roof * 1e6,
            "bound": "tensor" if t_tensor >= t_hbm else "hbm",
            "flops": work["flops"], "bytes": work["bytes"], "experts_touched": work["touched"],
            "peak": "bf16 %.1f TFLOP/s burst, HBM %.1f GB/s (%s)"
            % (peaks["bf16_tflops"], peaks["hbm_gbs"], peaks["source"])}


def other_configs(args, main_name, flush, stream, peaks):
    """The other layer configurations, each timed the same way (median of
    repeats of K steps, weights cold in L2 as ColdL2 says), for the same JSON line."""
    import torch
    from int4_expert_grouped_b200.layer import MoeLayer, bf16_tensor
    out = {}
    for name in ("tiny", "decode_t1", "decode_t4", "prefill_t512", "prefill_t8192",
                 "prefill_t32768_zipf"):
        if name == main_name:
            continue
        inp = mi.workload(name)
        s = inp.shape
        layer = MoeLayer.from_inputs(inp)
        x = bf16_tensor(inp.x, "cuda")
        y = torch.empty((max(s.T, 1), s.d), dtype=torch.bfloat16, device="cuda")
        bufs = layer.route_buffers(s.T)
        layer.forward(x, y, route_out=bufs)
        torch.cuda.synchronize()
        code, detail = layer.read_status()
        if code != 0:
            raise RuntimeError("%s: device status %d (%d)" % (name, code, detail))
        work = algorithmic(s, bufs["counts"].cpu().numpy())
        cold = ColdL2(layer, work, flush)
        for i in range(3):
            cold.before(i)
            layer.forward(x, y)
        torch.cuda.synchronize()
        K = args.steps if s.T < 32768 else max(3, args.steps // 2)
        clocks = ClockSampler(torch.cuda.current_device())
        clocks.start()
        reps, ms = time_layer(layer, x, y, K, args.repeats, cold, stream)
        clk = clocks.stop()
        stages = stage_times(layer, x, y, K, cold, stream)
        cold.release()
        roof = layer_roofline(work, ms, peaks)
        entry = {"workload": workload_desc(name, s, *mi.WORKLOADS[name][1:]), "tokens": s.T,
                 "ms_per_step": ms, "repeats_ms": reps, "tokens_per_s": s.T / (ms * 1e-3),
                 "layer_roofline": roof, "stages_ms": stages, "steps": K, "l2": cold.desc,
                 "gpu_launches_per_step": layer_launches(layer, s.T), "clocks": clk,
                 "kernels": "small-batch (decode)" if layer.plan.forward_path(s.T) == 1 else "batched"}
        if roof["bound"] == "hbm":
            entry["hbm_gbs_achieved"] = work["bytes"] / (ms * 1e-3) / 1e9
        out[name] = entry
        del layer
        torch.cuda.empty_cache()
    return out


def run_ours(args, name):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    build_library()
    from int4_expert_grouped_b200.layer import MoeLayer, bf16_tensor

    shape, seed, zipf = mi.WORKLOADS[name]
    inp = mi.workload(name)
    if args.tokens:
        # the first `tokens` tokens of the workload (a smaller case of the same layer)
        n = min(args.tokens, inp.shape.T)
        inp = mi.Inputs(mi.Shape(n, *[getattr(inp.shape, f) for f in ("d", "E", "k", "f", "group")]),
                        inp.seed, inp.x[:n], inp.w_r, inp.b_r, inp.gate, inp.up, inp.down)
    s = inp.shape
    layer = MoeLayer.from_inputs(inp)
    x = bf16_tensor(inp.x, "cuda")
    y = torch.empty((s.T, s.d), dtype=torch.bfloat16, device="cuda")
    bufs = layer.route_buffers(s.T)
    layer.forward(x, y, route_out=bufs)
    torch.cuda.synchronize()
    code, detail = layer.read_status()
    if code != 0:
        raise RuntimeError("device status %d (%d) after the first call" % (code, detail))
    if args.profile:
        # a few plain layer calls for a profiler to capture; no timing, no output
        for _ in range(args.profile):
            layer.forward(x, y)
        torch.cuda.synchronize()
        return
    counts = bufs["counts"].cpu().numpy()
    work = algorithmic(s, counts)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    cold = ColdL2(layer, work, flush)
    for i in range(max(args.warmup, 3)):
        cold.before(i)
        layer.forward(x, y)
    torch.cuda.synchronize()

    K = args.steps
    clocks = ClockSampler(local)
    clocks.start()
    reps, ms_per_step = time_layer(layer, x, y, K, args.repeats, cold, stream, world)
    clk = clocks.stop()
    stage_ms = stage_times(layer, x, y, K, cold, stream)
    cold.release()
    value = world * s.T / (ms_per_step * 1e-3)

    # end to end through the host-buffer entry point (pinned host memory)
    xh = torch.from_numpy(inp.x.view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = torch.empty((s.T, s.d), dtype=torch.bfloat16).pin_memory()
    layer.forward_host(xh, yh)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    KE = max(3, min(K, 10))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(KE):
        layer.forward_host(xh, yh)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / KE, world)
    code, detail = layer.read_status()
    if code != 0:
        raise RuntimeError("device status %d (%d) after timing" % (code, detail))

    peaks = load_peaks()
    lroof = layer_roofline(work, ms_per_step, peaks)
    decode = layer.plan.forward_path(s.T) == 1
    if decode:
        # one launch does the whole layer: its bytes are the touched experts'
        # weights, W_r, x and y; its time is the step's
        achieved = (work["bytes"] + 4 * s.d * s.E) / (ms_per_step * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                "kernel": "decode_layer_kernel", "peak_kind": "HBM copy, %s" % peaks["source"]}
    elif work["flops_gateup"] / (peaks["bf16_tflops"] * 1e12) >= \
            work["bytes_gateup"] / (peaks["hbm_gbs"] * 1e9):
        # the gate/up GEMM, timed alone with cold weights, well under a second:
        # the burst bf16 peak is its denominator; the sustained one is reported too
        t_gu = stage_ms["gate_up_gemm"] * 1e-3
        achieved = work["flops_gateup"] / t_gu / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                "traffic": TRAFFIC_GATEUP.get(name), "kernel": "grouped_gemm_kernel<gate/up>",
                "peak_kind": "bf16 burst, %s" % peaks["source"],
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"]}
    else:
        t_gu = stage_ms["gate_up_gemm"] * 1e-3
        achieved = work["bytes_gateup"] / t_gu / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": TRAFFIC_GATEUP.get(name),
                "kernel": "grouped_gemm_kernel<gate/up>", "peak_kind": "HBM copy, %s" % peaks["source"]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, n, dt = cpu_oracle_rate(inp)
        cpu = {"value": rate, "unit": "tokens/s", "cores": os.cpu_count(), "kind": "oracle",
               "sample": "first %d tokens of the workload, %.1f s (CPU oracle, float64, OpenMP)"
               % (n, dt)}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_desc(name, s, seed, zipf), "tokens_per_gpu": s.T,
                   "parallelism": "replicas" if world > 1 else "single GPU",
                   "l2": cold.desc,
                   "repeats": "median of %d repeats of %d steps" % (args.repeats, K)},
        "pct_of_layer_roofline": 100.0 * lroof["frac"],
        "layer_roofline": lroof,
        "repeats_ms": reps,
        "roofline": roof,
        "stages_ms": stage_ms,
        "cpu_baseline": cpu,
        "e2e": {"value": world * s.T / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(s.T * s.d * 2), "d2h_bytes_per_step": int(s.T * s.d * 2)},
        "gpu_launches": args.repeats * K * layer_launches(layer, s.T),
        "clocks": clk,
    }
    if world == 1 and not args.no_configs:
        del layer
        torch.cuda.empty_cache()
        line["configs"] = other_configs(args, name, flush, stream, peaks)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# dram__bytes_read.sum + dram__bytes_write.sum (bytes) of one gate/up GEMM
# launch from an ncu capture of the current kernel build (a one-pass metric
# set on the full workload, profiles/ncu_grouped_gemm_t2048.md); workloads
# without such a capture report None.
TRAFFIC_GATEUP: dict = {"prefill_t8192": 495.87e6 + 85.25e6}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="prefill_t8192", choices=sorted(mi.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--repeats", type=int, default=3,
                    help="repeats of the timed loop of K steps; the median is reported")
    ap.add_argument("--no-configs", action="store_true",
                    help="time only the main workload (not the other layer configurations)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="use only the first TOKENS tokens of the workload (smaller cases for profilers)")
    ap.add_argument("--profile", type=int, default=0,
                    help="run this many extra layer calls after set-up and exit (for ncu)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    args.repeats = max(1, args.repeats)
    if args.impl == "reference":
        run_reference(args, args.workload)
    else:
        run_ours(args, args.workload)


if __name__ == "__main__":
    main()
