#!/usr/bin/env python
"""Switch-FFN layer forward benchmark on B200.

One step = one whole layer forward through the C ABI (router, dispatch,
expert FFNs, gate-scaled combine with residual, load-balancing loss) on one
batch of synthetic input already resident in HBM.  The default workload is
the Switch-Base-like bf16 layer (T = 65536 tokens = batch 128 x seq 512,
d_model 768, d_ff 3072, 128 experts, capacity factor 1.25).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     (the CPU oracle, timed)

With N > 1 (torchrun) every rank runs an independent replica on its own
batch (its own routing group): weak scaling, no collective on the data path.
Rank 0 prints one JSON line.
"""
import argparse
import datetime
import json
import os
import select
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from switch_inputs import (WORKLOADS, PROFILE_WORKLOADS, make_x, make_router, make_w1,  # noqa: E402
                           make_w2, Inputs)
ALL_WORKLOADS = {**WORKLOADS, **PROFILE_WORKLOADS}

METRIC = "Switch-layer fwd tokens/s"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20

# DRAM bytes (read + written) of one GEMM1 + GEMM2 launch pair on the Base
# workload, from a one-pass ncu capture of those kernels (dram__bytes_read.sum
# + dram__bytes_write.sum, caches flushed before each kernel), valid only for
# the kernel sources they were taken on: the bench reports them as `traffic`
# while the sources hash the same, and null once a kernel has changed.
GEMM_SOURCES = ("common.cuh", "gemm_common.cuh", "gemm_pair.cuh", "expert_ffn.cu",
                "expert_ffn_pair.cu", "expert_ffn_pair_rows.cu")
GEMM_TRAFFIC = {"workload": "base",
                "sources_sha256": "c4fce9f41a3dd7e284f8129f86b81096d3c4c9f22e2d073bac49b74f260f4f6a",
                # GEMM1 715.75 MB read + 368.88 MB written; GEMM2 1197.38 + 89.05 MB
                # (mean of four forwards of one capture)
                "bytes": 715.75e6 + 368.88e6 + 1197.38e6 + 89.05e6}


def gemm_sources_sha256():
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_mixture_experts_switch_b200", "csrc")
    for name in GEMM_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def gemm_traffic(workload):
    if workload != GEMM_TRAFFIC["workload"] or GEMM_TRAFFIC["bytes"] is None:
        return None
    return GEMM_TRAFFIC["bytes"] if gemm_sources_sha256() == GEMM_TRAFFIC["sources_sha256"] \
        else None


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="base",
                    choices=sorted(WORKLOADS) + sorted(PROFILE_WORKLOADS),
                    help="the headline workload (default base); base_e64, Base's per-expert "
                         "shape at half the tokens and experts, is for counter captures")
    ap.add_argument("--parallel", default="replicas", choices=["replicas", "ep"],
                    help="N > 1: independent replicas (default), or expert parallelism "
                         "(each rank N/G experts and its own T tokens, one routing group)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workloads", default=None,
                    help="comma-separated extra workloads timed after the headline one "
                         "('all' = every bf16 workload, 'none'; default: all at N=1, none at N>1)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="budget of the oracle sample timed for cpu_baseline")
    ap.add_argument("--stage", default=None, choices=sorted(STAGES),
                    help="time one staged call alone on --workload (--steps replays after "
                         "--warmup) and print its line instead of the layer's")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(wl):
    return (f"{wl.name}: Switch-FFN layer, T={wl.T} tokens, d_model={wl.d_model}, "
            f"d_ff={wl.d_ff}, N={wl.n_experts} experts, capacity_factor={wl.capacity_factor}, "
            f"{wl.dtype} (fp32 router)")


# ------------------------------------------------------------ CPU oracle

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_sample(inp, budget_s, fixed_experts=None):
    """Time the oracle on a bounded sample of the workload.

    The router (fp64 logits, softmax, top-1) and the dispatch run on every
    token; the expert FFNs run for experts 0, 1, ... until the time budget is
    spent (or for `fixed_experts` of them); the combine and the loss run on
    every token.  The expert time is scaled by N / (experts run) to estimate
    the whole layer.  Returns (estimated seconds for the layer, experts run).
    """
    import oracle.switch_oracle as orc
    wl = inp.wl
    t0 = time.perf_counter()
    r = orc.router(inp.x, inp.w_r, inp.b_r)
    C = orc.capacity(wl.T, wl.n_experts, wl.capacity_factor)
    dsp = orc.dispatch(r["idx"], wl.n_experts, C)
    t1 = time.perf_counter()
    Y = np.zeros((wl.n_experts, C, wl.d_model))
    done = 0
    t_exp0 = time.perf_counter()
    limit = fixed_experts if fixed_experts is not None else wl.n_experts
    while done < limit:
        part = orc.expert_ffn(inp.x, inp.w1, inp.w2, dsp["slot_token"], dsp["counts"], C,
                              experts=[done])
        Y[done] = part[done]
        done += 1
        if fixed_experts is None and time.perf_counter() - t0 > budget_s:
            break
    t_exp = time.perf_counter() - t_exp0
    t2 = time.perf_counter()
    orc.combine(inp.x, r["idx"], dsp["rank"], dsp["drop"], r["gate"], Y)
    orc.aux_loss(dsp["counts"], r["probs"], wl.alpha)
    t3 = time.perf_counter()
    est = (t1 - t0) + (t3 - t2) + t_exp * wl.n_experts / done
    return est, done


def host_inputs(wl, rank=0):
    w_r, b_r = make_router(wl)
    x = make_x(wl.with_(seed=wl.seed + 7919 * rank))
    return Inputs(wl, x, w_r, b_r, make_w1(wl), make_w2(wl))


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = ALL_WORKLOADS[args.workload]
    inp = host_inputs(wl)
    per_step_budget = max(1.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    est, n_exp = oracle_sample(inp, per_step_budget)          # sizes the sample
    for _ in range(max(0, args.warmup - 1)):
        oracle_sample(inp, per_step_budget, fixed_experts=n_exp)
    ests = [oracle_sample(inp, per_step_budget, fixed_experts=n_exp)[0]
            for _ in range(args.steps)]
    sec = statistics.mean(ests)
    value = wl.T / sec
    sample = (f"oracle (numpy float64) on all {wl.T} tokens for router, dispatch, combine "
              f"and loss; expert FFNs for experts 0..{n_exp - 1} of {wl.n_experts}, "
              f"time scaled by {wl.n_experts}/{n_exp}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(wl)},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# -------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock, power and clock-event reasons sampled while the GPU works.

    Reads NVML directly every few milliseconds (read-only queries), so that a
    timed region of a few tens of milliseconds still gets several samples;
    falls back to `nvidia-smi -lms 100` when NVML is not importable."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id, uuid=None, period_s=0.0005):
        self.gpu_id = gpu_id
        self.uuid = uuid
        self.period_s = period_s
        self.rows = []            # (time, sm_mhz, max_mhz, power_w, reasons)
        self.proc = None
        self.stop_evt = threading.Event()
        self.thread = None
        self.source = None

    # The NVML loop runs in a child process of its own, so that the bench
    # process's interpreter lock (held while it launches and waits) cannot
    # starve it; each line carries the child's wall-clock time of the sample.
    NVML_CHILD = r"""
import sys, time, pynvml
pynvml.nvmlInit()
uuid, idx, period = sys.argv[1], int(sys.argv[2]), float(sys.argv[3])
h = pynvml.nvmlDeviceGetHandleByUUID(uuid) if uuid else pynvml.nvmlDeviceGetHandleByIndex(idx)
bits = (pynvml.nvmlClocksEventReasonHwSlowdown, pynvml.nvmlClocksEventReasonHwThermalSlowdown,
        pynvml.nvmlClocksEventReasonSwThermalSlowdown, pynvml.nvmlClocksEventReasonSwPowerCap)
mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
pw, n = 0.0, 0
for _ in range(3):          # the first queries are slow: make them before reporting ready
    pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
    pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
    pynvml.nvmlDeviceGetPowerUsage(h)
print("ready", flush=True)
while True:
    try:
        sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
        rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
        if n % 8 == 0:
            pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
        n += 1
        flags = "".join("1" if rs & b else "0" for b in bits)
        print(f"{time.time():.6f},{sm},{mx},{pw:.1f},{flags}", flush=True)
    except pynvml.NVMLError:
        pass
    time.sleep(period)
"""

    def start(self):
        try:
            import pynvml  # noqa: F401 -- the child needs it too
            self.proc = subprocess.Popen(
                [sys.executable, "-c", self.NVML_CHILD, self.uuid or "", str(self.gpu_id or 0),
                 str(self.period_s)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            ready, _, _ = select.select([self.proc.stdout], [], [], 30.0)
            if not ready or self.proc.stdout.readline().strip() != "ready":
                raise RuntimeError("NVML sampler did not start")
            self.source = "nvml"
            self.thread = threading.Thread(target=self._nvml_lines, daemon=True)
            self.thread.start()
            return
        except Exception:
            if self.proc is not None:
                self.proc.kill()
                self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu_id)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi"
            self.thread = threading.Thread(target=self._smi, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _nvml_lines(self):
        for ln in self.proc.stdout:
            r = ln.strip().split(",")
            try:
                self.rows.append((float(r[0]), float(r[1]), float(r[2]), float(r[3]),
                                  [n for n, f in zip(self.REASONS, r[4]) if f == "1"]))
            except (ValueError, IndexError):
                pass

    def _smi(self):
        names = self.REASONS
        for ln in self.proc.stdout:
            r = [c.strip() for c in ln.split(",")]
            try:
                self.rows.append((time.time(), float(r[1]), float(r[2]), float(r[3]),
                                  [n for n, v in zip(names, r[5:9]) if v == "Active"]))
            except (ValueError, IndexError):
                pass

    def stop(self):
        self.stop_evt.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        rows = [r for r in self.rows if t0 <= r[0] <= t1]
        if not rows:   # region shorter than the sampling period: nearest samples
            rows = sorted(self.rows, key=lambda r: abs(r[0] - (t0 + t1) / 2))[:3]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(r[1] for r in rows),
                "sm_max_mhz": max(r[2] for r in rows),
                "reasons": sorted({n for r in rows for n in r[4]}),
                "samples": len(rows), "source": self.source,
                "power_w_max": max(r[3] for r in rows)}


# ------------------------------------------------------------- GPU arm

def run_expert_parallel(args):
    """--parallel ep: the layer expert-parallel over the torchrun ranks.  Each
    rank holds N / G experts and its own batch of the workload's T tokens
    (weak scaling: G * T tokens in one routing group); a step is one
    ExpertParallelSwitch.forward (route, record all-gather, dispatch with peer
    stores, barrier, experts with the combine stored on the home ranks,
    barrier), launched eagerly; device time by CUDA events, max over ranks."""
    import torch
    import torch.distributed as dist
    from sparse_mixture_experts_switch_b200.expert_parallel import ExpertParallelSwitch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    wl = ALL_WORKLOADS[args.workload]
    inp = host_inputs(wl, rank)
    T, d, F, N = wl.T, wl.d_model, wl.d_ff, wl.n_experts
    E = N // world

    def to_dev(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    x, w_r, b_r = to_dev(inp.x), to_dev(inp.w_r), to_dev(inp.b_r)
    w1 = to_dev(inp.w1[rank * E:(rank + 1) * E])
    w2 = to_dev(inp.w2[rank * E:(rank + 1) * E])
    layer = ExpertParallelSwitch(T, d, F, N, wl.capacity_factor, alpha=wl.alpha, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(3, args.warmup)):
        layer.forward(x, w_r, b_r, w1, w2)
    torch.cuda.synchronize(dev)
    st, where, info = layer.lib.switch_get_device_error(layer.ws)
    if st != 0:
        raise RuntimeError(f"device error {st} at {where} ({info}) during warm-up")
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    dist.barrier()
    torch.cuda.synchronize(dev)
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        layer.forward(x, w_r, b_r, w1, w2)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    total_ms = max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in evs), dev, world)
    st, where, info = layer.lib.switch_get_device_error(layer.ws)
    if st != 0:
        raise RuntimeError(f"device error {st} at {where} ({info}) in the timed region")
    value = job_throughput(T, args.steps, world, total_ms)
    if rank == 0:
        C = layer.lib.switch_capacity(world * T, N, wl.capacity_factor)
        print(json.dumps({
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": workload_desc(wl), "T_per_rank": T, "d_model": d,
                       "d_ff": F, "n_experts": N, "capacity_factor": wl.capacity_factor,
                       "capacity": C, "parallelism": f"expert parallel x{world}",
                       "l2": "flushed (256 MiB write) before every timed step, outside the events",
                       "launch": "eager launches of ExpertParallelSwitch.forward"},
            "gpu_launches": 10 * args.steps}), flush=True)
    dist.barrier()
    dist.destroy_process_group()


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.stage is not None:
        return run_stage(args)
    if args.parallel == "ep" and int(os.environ.get("WORLD_SIZE", "1")) > 1:
        return run_expert_parallel(args)

    import torch
    import torch.distributed as dist
    from sparse_mixture_experts_switch_b200 import switch_moe as sm

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    wl = ALL_WORKLOADS[args.workload]
    inp = host_inputs(wl, rank)
    T, d, F, N = wl.T, wl.d_model, wl.d_ff, wl.n_experts
    C = sm.switch_capacity(T, N, wl.capacity_factor)
    bf = wl.dtype == "bf16"
    tdt = torch.bfloat16 if bf else torch.float32

    def to_dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    x = to_dev(inp.x)
    w_r = to_dev(inp.w_r)
    b_r = None if inp.b_r is None else to_dev(inp.b_r)
    w1 = to_dev(inp.w1)
    w2 = to_dev(inp.w2)
    cfg = sm.config(T, d, F, N, wl.capacity_factor, dtype=wl.dtype, alpha=wl.alpha)
    ws = sm.workspace(cfg, device=dev)
    out = torch.empty_like(x)
    idx = torch.empty(T, dtype=torch.int32, device=dev)
    gate = torch.empty(T, dtype=torch.float32, device=dev)
    counts = torch.empty(N, dtype=torch.int32, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        sm.switch_layer_forward(cfg, x, w_r, b_r, w1, w2, out, idx, gate, counts, loss, ws)

    # One forward = 6 kernel launches with no host synchronisation inside, so
    # it is captured once as a CUDA graph and replayed: the timed region then
    # measures the kernels, not the host's launch latency.
    step_graph = make_graph(step)

    def barrier():
        if world > 1:
            dist.barrier()

    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    clocks = ClockSampler(local if not os.environ.get("CUDA_VISIBLE_DEVICES")
                          else os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local], uuid)
    clocks.start()
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    st, where, info = sm.switch_get_device_error(ws)
    if st != 0:
        raise RuntimeError(f"device error {st} at {where} ({info}) during warm-up")

    # ------------------------------------------------ timed region (device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    for e0, e1 in evs:
        flush.zero_()                      # L2 flush, outside the events
        e0.record(stream)
        step_graph()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    t_wall1 = time.time()
    ms = [e0.elapsed_time(e1) for e0, e1 in evs]
    total_ms = max_over_ranks(sum(ms), dev, world)
    st, where, info = sm.switch_get_device_error(ws)
    if st != 0:
        raise RuntimeError(f"device error {st} at {where} ({info}) in the timed region")
    ms_per_step = total_ms / args.steps
    value = job_throughput(T, args.steps, world, total_ms)

    # ------------------------------------------- end to end (host buffers)
    # Each step copies its input from pinned host memory, runs the layer
    # through the public call, and copies its output and loss back, as a
    # serving loop would: on three streams, so that step i's input copy and
    # step i-1's output copy (separate copy engines, both PCIe directions)
    # run while step i-1 / step i compute; two device input and output
    # buffers alternate, and events order every reuse.
    x_host = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    x_host.copy_(x)
    out_host = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    loss_host = [torch.empty(1, dtype=torch.float32, pin_memory=True) for _ in range(2)]
    xb = [x, torch.empty_like(x)]
    ob = [out, torch.empty_like(out)]
    lb = [loss, torch.empty_like(loss)]
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()                        # noqa: E731

    def e2e_run(n, compute=True):
        """n pipelined steps; returns (first event, last event) for timing.
        compute=False runs the same copies and ordering without the layer:
        the copy-bound ceiling of this loop on this host."""
        t_first = torch.cuda.Event(enable_timing=True)
        t_last = torch.cuda.Event(enable_timing=True)
        in_done, comp_done, out_done = {}, {}, {}
        t_first.record(s_in)
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(comp_done[i - 2])      # step i-2 has read xb[b]
                xb[b].copy_(x_host, non_blocking=True)
                in_done[i] = ev()
                in_done[i].record(s_in)
            stream.wait_event(in_done[i])
            if i >= 2:
                stream.wait_event(out_done[i - 2])         # ob[b] copied out
            if compute:
                sm.switch_layer_forward(cfg, xb[b], w_r, b_r, w1, w2, ob[b], None, None, None,
                                        lb[b], ws)
            comp_done[i] = ev()
            comp_done[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[i])
                out_host[b].copy_(ob[b], non_blocking=True)
                loss_host[b].copy_(lb[b], non_blocking=True)
                out_done[i] = ev()
                out_done[i].record(s_out)
        s_in.wait_stream(s_out)
        s_in.wait_stream(stream)
        t_last.record(s_in)
        return t_first, t_last

    e2e_run(max(3, args.warmup))
    barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = e2e_run(args.steps)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_value = job_throughput(T, args.steps, world,
                               max_over_ranks(e0.elapsed_time(e1), dev, world))
    e2e_bytes = (x_host.numel() * x_host.element_size(),
                 out_host[0].numel() * out_host[0].element_size() + loss_host[0].numel() * 4)
    # the same loop with the copies alone: what the host link allows
    e2e_run(max(3, args.warmup), compute=False)
    torch.cuda.synchronize(dev)
    c0, c1 = e2e_run(args.steps, compute=False)
    torch.cuda.synchronize(dev)
    copy_ms = max_over_ranks(c0.elapsed_time(c1), dev, world)
    copy_bound = job_throughput(T, args.steps, world, copy_ms)
    del x_host, out_host, step_graph, xb, ob

    # --------------------------------------- per-kernel roofline (rank 0)
    line = None
    if rank == 0:
        pk, pk_kind = peaks()
        kern = kernel_rooflines(sm, cfg, wl, C, x, w_r, b_r, w1, w2, ws, flush, stream, dev,
                                pk, pk_kind)
        T_kept = kern.pop("_T_kept")
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            est, n_exp = oracle_sample(inp, args.cpu_seconds)
            cpu = {"value": wl.T / est, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                   "sample": (f"numpy float64 oracle: router, dispatch, combine and loss on "
                              f"all {wl.T} tokens; expert FFNs of experts 0..{n_exp - 1} of "
                              f"{wl.n_experts}, their time scaled by {wl.n_experts}/{n_exp}"),
                   "host_cpus": os.cpu_count()}
        ffn = kern["expert_ffn"]
        bounds = layer_bounds(wl, T_kept, pk)
        t_layer_min = bounds["t_min_us"] * 1e-6
        extra = extra_workloads(args, world, wl.name)
        table = {wl.name: workload_row(wl, C, ms_per_step, ffn["us"] * 1e-6, T_kept, pk)}
        del x, w1, w2, ws, out
        torch.cuda.empty_cache()
        for name in extra:
            tw0 = time.time()
            table[name] = time_workload(sm, WORKLOADS[name], dev, stream, flush, pk,
                                        max(5, min(args.steps, 20)))
            # the SM clock while this workload's layer and expert FFN were timed
            # (a long tensor-bound workload can reach the power cap)
            table[name]["clocks"] = clocks.summary(tw0, time.time())
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if bf else "f32", "data": "synthetic",
            "config": {"workload": workload_desc(wl), "T": T, "d_model": d, "d_ff": F,
                       "n_experts": N, "capacity_factor": wl.capacity_factor, "capacity": C,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "flushed (256 MiB write) before every timed step, outside the events",
                       "launch": "each step replays a CUDA graph of one switch_layer_forward "
                                 "call (all its kernels); e2e calls the C ABI directly"},
            "roofline": {"kernel": "expert FFN grouped GEMM (GEMM1 + GEMM2, tcgen05)",
                         "bound": "tensor", "achieved": ffn["tflops"],
                         "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": ffn["tflops"] / pk["bf16_tflops"],
                         "peak_kind": f"{pk_kind} bf16 burst",
                         "traffic": gemm_traffic(args.workload),
                         "useful_flops": 4.0 * T_kept * d * F},
            "layer_roofline": {**bounds, "tokens_per_s": T / t_layer_min,
                               "frac": value / world / (T / t_layer_min)},
            "kernels": kern,
            "workloads": table,
            "routing": {"T_kept": T_kept, "drop_rate": 1.0 - T_kept / T,
                        "padding": 1.0 - T_kept / (N * C)},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": e2e_bytes[0],
                    "d2h_bytes_per_step": e2e_bytes[1],
                    # the same pipelined loop with its copies only (no layer)
                    "copy_bound": copy_bound,
                    "frac_of_copy_bound": e2e_value / copy_bound,
                    "h2d_gbs_per_gpu": e2e_bytes[0] * args.steps / (copy_ms * 1e-3) / 1e9},
            "clocks": clocks.summary(t_wall0, t_wall1),
            "gpu_launches": launches_per_step(cfg, wl) * args.steps,
        }
    clocks.stop()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


# staged calls that --stage times alone: algorithmic bytes as in the kernel table
STAGES = ("router", "router_probs", "dispatch", "dispatch_gather", "combine", "aux_loss",
          "expert_ffn")


def run_stage(args):
    """One staged call on one GPU, on the workload's synthetic inputs: the
    router (with probabilities) and the dispatch run once to give it real
    routing; then `steps` graph replays of the call, each after an L2 flush."""
    import torch
    from sparse_mixture_experts_switch_b200 import switch_moe as sm
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = ALL_WORKLOADS[args.workload]
    w_r_h, b_r_h = make_router(wl)          # expert weights only for the expert FFN stage
    T, d, N = wl.T, wl.d_model, wl.n_experts
    C = sm.switch_capacity(T, N, wl.capacity_factor)
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32

    def to_dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    x, w_r = to_dev(make_x(wl)), to_dev(w_r_h)
    b_r = None if b_r_h is None else to_dev(b_r_h)
    cfg = sm.config(T, d, wl.d_ff, N, wl.capacity_factor, dtype=wl.dtype, alpha=wl.alpha)
    ws = sm.workspace(cfg, device=dev)
    i32 = dict(dtype=torch.int32, device=dev)
    idx, rank, counts = torch.empty(T, **i32), torch.empty(T, **i32), torch.empty(N, **i32)
    gate = torch.empty(T, dtype=torch.float32, device=dev)
    probs = torch.empty(T, N, dtype=torch.float32, device=dev)
    drop = torch.empty(T, dtype=torch.uint8, device=dev)
    slot = torch.empty(N * C, **i32)
    x_disp = torch.empty(N * C, d, dtype=tdt, device=dev)
    y = torch.empty(N * C, d, dtype=tdt, device=dev).normal_()
    out = torch.empty_like(x)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    sm.switch_router(cfg, x, w_r, b_r, idx, gate, probs, ws)
    sm.switch_dispatch(cfg, idx, None, rank, drop, counts, slot, x, x_disp, ws)
    torch.cuda.synchronize(dev)
    T_kept = int(np.minimum(counts.cpu().numpy().astype(np.int64), C).sum())
    ffn = None
    if args.stage == "expert_ffn":
        w1, w2 = to_dev(make_w1(wl)), to_dev(make_w2(wl))
        cfg_rows = sm.config(T, d, wl.d_ff, N, wl.capacity_factor, dtype=wl.dtype,
                             alpha=wl.alpha, flags=sm.FLAG_ROWS_DISPATCHED)
        ffn = lambda: sm.switch_expert_ffn(cfg_rows, x_disp, None, counts, w1, w2, y, ws)  # noqa: E731
    es = x.element_size()
    calls = {
        "router": (lambda: sm.switch_router(cfg, x, w_r, b_r, idx, gate, None, ws),
                   T * d * es + N * d * 4 + T * 8),
        "router_probs": (lambda: sm.switch_router(cfg, x, w_r, b_r, idx, gate, probs, ws),
                         T * d * es + N * d * 4 + T * 8 + T * N * 4),
        "dispatch": (lambda: sm.switch_dispatch(cfg, idx, None, rank, drop, counts, slot, None,
                                                None, ws),
                     T * 4 + T * 5 + N * 4 + N * C * 4),
        "dispatch_gather": (lambda: sm.switch_dispatch(cfg, idx, None, rank, drop, counts, slot,
                                                       x, x_disp, ws),
                            T * 9 + N * 4 + N * C * 4 + T_kept * d * es + N * C * d * es),
        "combine": (lambda: sm.switch_combine(cfg, x, idx, rank, drop, gate, y, out),
                    2 * T * d * es + T_kept * d * es + T * 13),
        "aux_loss": (lambda: sm.switch_aux_loss(cfg, counts, probs, loss, None, None, ws),
                     T * N * 4 + N * 4),
        # FLOPs, not bytes: the line's "gbs" is then useful GFLOP/s
        "expert_ffn": (ffn, 4.0 * T_kept * d * wl.d_ff),
    }
    fn, nbytes = calls[args.stage]
    for _ in range(max(0, args.warmup - 3)):
        fn()
    t = time_replays(fn, flush, torch.cuda.current_stream(dev), dev, args.steps)
    st, where, info = sm.switch_get_device_error(ws)
    if st != 0:
        raise RuntimeError(f"device error {st} at {where} ({info}) in {args.stage}")
    pk, pk_kind = peaks()
    line = {"stage": args.stage, "workload": workload_desc(wl), "us": t * 1e6}
    if args.stage == "expert_ffn":
        line.update({"useful_flops": nbytes, "tflops": nbytes / t / 1e12,
                     "frac_burst": nbytes / t / 1e12 / pk["bf16_tflops"]})
    else:
        line.update({"bytes": nbytes, "gbs": nbytes / t / 1e9,
                     "frac_hbm": nbytes / t / 1e9 / pk["hbm_gbs"]})
    line.update({"peak_kind": pk_kind, "steps": args.steps, "warmup": max(3, args.warmup),
                 "l2": "flushed (256 MiB write) before every replay"})
    print(json.dumps(line), flush=True)


def layer_bounds(wl, T_kept, pk):
    """Roofline of the whole layer: useful FLOPs (router + kept tokens' expert
    GEMMs) at the bf16 burst peak against the layer's minimum bytes (x read
    three times -- router, row copy, residual -- every expert weight once, out
    written once) at the HBM peak."""
    T, d, F, N = wl.T, wl.d_model, wl.d_ff, wl.n_experts
    es = 2 if wl.dtype == "bf16" else 4
    flops = 2.0 * T * d * N + 4.0 * T_kept * d * F
    nbytes = 3 * T * d * es + 2 * N * d * F * es + T * d * es
    t_c = flops / (pk["bf16_tflops"] * 1e12)
    t_m = nbytes / (pk["hbm_gbs"] * 1e9)
    return {"useful_flops": flops, "min_bytes": nbytes, "t_compute_us": t_c * 1e6,
            "t_mem_us": t_m * 1e6, "bound": "tensor" if t_c >= t_m else "hbm",
            "t_min_us": max(t_c, t_m) * 1e6}


def workload_row(wl, C, t_step_ms, t_ffn_s, T_kept, pk):
    """One row of the per-workload table: layer tokens/s and the expert GEMMs'
    throughput against the bf16 peak, with the routing statistics."""
    T, d, F, N = wl.T, wl.d_model, wl.d_ff, wl.n_experts
    b = layer_bounds(wl, T_kept, pk)
    ffn_flops = 4.0 * T_kept * d * F
    tfl = ffn_flops / t_ffn_s / 1e12
    return {"T": T, "d_model": d, "d_ff": F, "n_experts": N,
            "capacity_factor": wl.capacity_factor, "capacity": C,
            "ms_per_step": t_step_ms, "tokens_per_s": T / (t_step_ms * 1e-3),
            "layer_tflops": b["useful_flops"] / (t_step_ms * 1e-3) / 1e12,
            "layer_roofline_frac": b["t_min_us"] / (t_step_ms * 1e3),
            "t_compute_us": b["t_compute_us"], "t_mem_us": b["t_mem_us"], "bound": b["bound"],
            "expert_ffn_us": t_ffn_s * 1e6, "expert_ffn_tflops": tfl,
            "expert_ffn_frac_burst": tfl / pk["bf16_tflops"],
            "expert_ffn_frac_sustained": tfl / pk["bf16_tflops_sustained"],
            "T_kept": T_kept, "drop_rate": 1.0 - T_kept / T,
            "padding": 1.0 - T_kept / (N * C)}


def extra_workloads(args, world, headline):
    if args.workloads is None:
        names = "all" if world == 1 else ""
    else:
        names = args.workloads
    if names == "all":
        names = ",".join(n for n, w in WORKLOADS.items() if w.dtype == "bf16")
    if names == "none":
        return []
    unknown = [n for n in names.split(",") if n and n not in WORKLOADS]
    if unknown:
        raise SystemExit(f"unknown workloads: {unknown}")
    return [n for n in names.split(",") if n and n != headline]


def time_replays(fn, flush, stream, dev, reps):
    """Mean device time of `reps` replays of a CUDA graph of fn, each after an
    L2 flush, each bracketed by CUDA events on the launching stream."""
    import torch
    g = make_graph(fn)
    g()
    ts = []
    for _ in range(reps):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ts.append(e0.elapsed_time(e1) * 1e-3)
    return statistics.mean(ts)


def time_workload(sm, wl, dev, stream, flush, pk, steps):
    """The layer forward and the staged expert FFN of one more workload, timed
    like the headline (graph replay, L2 flushed before each step)."""
    import torch
    inp = host_inputs(wl)

    def to_dev(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    T, d, F, N = wl.T, wl.d_model, wl.d_ff, wl.n_experts
    x, w_r, b_r, w1, w2 = (to_dev(a) for a in (inp.x, inp.w_r, inp.b_r, inp.w1, inp.w2))
    del inp
    C = sm.switch_capacity(T, N, wl.capacity_factor)
    cfg = sm.config(T, d, F, N, wl.capacity_factor, dtype=wl.dtype, alpha=wl.alpha)
    ws = sm.workspace(cfg, device=dev)
    out = torch.empty_like(x)
    i32 = dict(dtype=torch.int32, device=dev)
    idx, counts = torch.empty(T, **i32), torch.empty(N, **i32)
    gate = torch.empty(T, dtype=torch.float32, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    t_step = time_replays(lambda: sm.switch_layer_forward(cfg, x, w_r, b_r, w1, w2, out, idx,
                                                          gate, counts, loss, ws),
                          flush, stream, dev, steps)
    rank, slot = torch.empty(T, **i32), torch.empty(N * C, **i32)
    drop = torch.empty(T, dtype=torch.uint8, device=dev)
    x_disp = torch.empty(N * C, d, dtype=x.dtype, device=dev)
    y = torch.empty(N * C, d, dtype=x.dtype, device=dev)
    sm.switch_dispatch(cfg, idx, None, rank, drop, counts, slot, x, x_disp, ws)
    cfg_rows = sm.config(T, d, F, N, wl.capacity_factor, dtype=wl.dtype, alpha=wl.alpha,
                         flags=sm.FLAG_ROWS_DISPATCHED)
    t_ffn = time_replays(lambda: sm.switch_expert_ffn(cfg_rows, x_disp, None, counts, w1, w2,
                                                      y, ws), flush, stream, dev, 10)
    st, where, info = sm.switch_get_device_error(ws)
    if st != 0:
        raise RuntimeError(f"device error {st} at {where} ({info}) timing {wl.name}")
    cnt = counts.cpu().numpy().astype(np.int64)
    T_kept = int(np.minimum(cnt, C).sum())
    row = workload_row(wl, C, t_step * 1e3, t_ffn, T_kept, pk)
    row["steps"] = steps
    del x, w_r, b_r, w1, w2, ws, out, x_disp, y
    torch.cuda.empty_cache()
    return row


def make_graph(fn, warm=3):
    """Capture fn (a sequence of launches on the current stream) in a CUDA
    graph after a few warm-up calls on the capture stream; returns replay."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(warm):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g.replay


def max_over_ranks(value, device, world):
    """The largest per-rank value (rank timings are aggregated by their max)."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank, steps, world, max_total_ms):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * steps * world / (max_total_ms / 1e3)


def launches_per_step(cfg, wl):
    """Kernels switch_layer_forward launches with the default flags on this
    workload: router (weight split + tensor-core router, or SIMT router +
    tile ranks), the scan (which also forms the loss), finalize (for bf16
    with the row copy, which also writes the dropped tokens' rows), GEMM1,
    GEMM2 (with the combine); fp32 adds the dropped-token copy."""
    return 2 + 1 + 1 + 2 + (0 if wl.dtype == "bf16" else 1)


def kernel_rooflines(sm, cfg, wl, C, x, w_r, b_r, w1, w2, ws, flush, stream, dev, pk, pk_kind,
                     reps=10):
    """Staged calls timed alone (L2 flushed before each), with their
    algorithmic bytes / FLOPs."""
    import torch
    T, d, F, N = wl.T, wl.d_model, wl.d_ff, wl.n_experts
    i32 = dict(dtype=torch.int32, device=dev)
    idx = torch.empty(T, **i32)
    gate = torch.empty(T, dtype=torch.float32, device=dev)
    probs = torch.empty(T, N, dtype=torch.float32, device=dev)
    rank = torch.empty(T, **i32)
    drop = torch.empty(T, dtype=torch.uint8, device=dev)
    counts = torch.empty(N, **i32)
    slot = torch.empty(N * C, **i32)
    x_disp = torch.empty(N * C, d, dtype=x.dtype, device=dev)
    y = torch.empty(N * C, d, dtype=x.dtype, device=dev)
    out = torch.empty_like(x)
    loss = torch.empty(1, dtype=torch.float32, device=dev)

    def timed(fn):
        fn = make_graph(fn)
        fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ts.append(e0.elapsed_time(e1) * 1e-3)
        return statistics.mean(ts)

    es = x.element_size()
    t_router = timed(lambda: sm.switch_router(cfg, x, w_r, b_r, idx, gate, None, ws))
    t_router_p = timed(lambda: sm.switch_router(cfg, x, w_r, b_r, idx, gate, probs, ws))
    t_disp = timed(lambda: sm.switch_dispatch(cfg, idx, None, rank, drop, counts, slot, None,
                                              None, ws))
    t_disp_g = timed(lambda: sm.switch_dispatch(cfg, idx, None, rank, drop, counts, slot, x,
                                                x_disp, ws))
    cnt = counts.cpu().numpy().astype(np.int64)
    T_kept = int(np.minimum(cnt, C).sum())
    # GEMM1 + GEMM2 alone: the rows dispatch_gather laid out, fed straight in
    cfg_rows = sm.config(T, d, F, N, wl.capacity_factor, dtype=wl.dtype, alpha=wl.alpha,
                         flags=sm.FLAG_ROWS_DISPATCHED)
    t_ffn = timed(lambda: sm.switch_expert_ffn(cfg_rows, x_disp, None, counts, w1, w2, y, ws))
    t_comb = timed(lambda: sm.switch_combine(cfg, x, idx, rank, drop, gate, y, out))
    # the top-2 routing variant of the whole layer (capacity over 2T)
    t_top2 = None
    T_kept2 = 0
    if N >= 2:
        cfg2 = sm.config(T, d, F, N, wl.capacity_factor, dtype=wl.dtype, alpha=wl.alpha,
                         flags=sm.FLAG_TOP2)
        ws2 = sm.workspace(cfg2, device=dev)
        idx2 = torch.empty(2 * T, **i32)
        gate2 = torch.empty(2 * T, dtype=torch.float32, device=dev)
        counts2 = torch.empty(N, **i32)
        t_top2 = timed(lambda: sm.switch_layer_forward(cfg2, x, w_r, b_r, w1, w2, out, idx2,
                                                       gate2, counts2, loss, ws2))
        st2, where2, info2 = sm.switch_get_device_error(ws2)
        if st2 != 0:
            raise RuntimeError(f"device error {st2} at {where2} ({info2}) in the top-2 layer")
        C2 = sm.switch_capacity(2 * T, N, wl.capacity_factor)
        T_kept2 = int(np.minimum(counts2.cpu().numpy().astype(np.int64), C2).sum())
        del ws2
    # the backward pass of the whole layer (recomputes routing, dispatch and H)
    t_bwd = t_bwd_saved = t_train = t_bwd2 = None
    if wl.dtype == "bf16":
        wsb = sm.backward_workspace(cfg, device=dev)
        dout = torch.empty_like(x).normal_()
        dx = torch.empty_like(x)
        dw_r = torch.empty_like(w_r)
        db_r = torch.empty(N, dtype=torch.float32, device=dev)
        dw1 = torch.empty_like(w1)
        dw2 = torch.empty_like(w2)
        t_bwd = timed(lambda: sm.switch_layer_backward(cfg, x, w_r, b_r, w1, w2, dout, 1.0, dx,
                                                       dw_r, db_r, dw1, dw2, None, wsb))
        stb, whereb, infob = sm.switch_get_device_error(wsb)
        if stb != 0:
            raise RuntimeError(f"device error {stb} at {whereb} ({infob}) in the backward pass")
        del wsb
        # training mode: the forward keeps its activations, the backward reads
        # them (no recompute); and one whole training step of the layer
        cfg_t = sm.config(T, d, F, N, wl.capacity_factor, dtype=wl.dtype, alpha=wl.alpha,
                          flags=sm.FLAG_TRAINING)
        wst = sm.backward_workspace(cfg_t, device=dev)

        def fwd_t():
            sm.switch_layer_forward(cfg_t, x, w_r, b_r, w1, w2, out, idx, gate, counts, loss, wst)

        def bwd_t():
            sm.switch_layer_backward(cfg_t, x, w_r, b_r, w1, w2, dout, 1.0, dx, dw_r, db_r, dw1,
                                     dw2, None, wst)

        fwd_t()
        t_bwd_saved = timed(bwd_t)
        t_train = timed(lambda: (fwd_t(), bwd_t()))
        stb, whereb, infob = sm.switch_get_device_error(wst)
        if stb != 0:
            raise RuntimeError(f"device error {stb} at {whereb} ({infob}) in the training step")
        del wst
        # the top-2 backward (recomputes the top-2 routing, dispatch and H)
        if N >= 2:
            wsb2 = sm.backward_workspace(cfg2, device=dev)
            t_bwd2 = timed(lambda: sm.switch_layer_backward(cfg2, x, w_r, b_r, w1, w2, dout, 1.0,
                                                            dx, dw_r, db_r, dw1, dw2, None,
                                                            wsb2))
            stb, whereb, infob = sm.switch_get_device_error(wsb2)
            if stb != 0:
                raise RuntimeError(f"device error {stb} at {whereb} ({infob}) in the top-2 "
                                   "backward pass")
            del wsb2
        del dout, dx, dw1, dw2
    t_aux = timed(lambda: sm.switch_aux_loss(cfg, counts, probs, loss, None, None, ws))
    st, where, info = sm.switch_get_device_error(ws)
    if st != 0:
        raise RuntimeError(f"device error {st} at {where} ({info}) in kernel timing")
    hbm = pk["hbm_gbs"]

    def bw(name, t, nbytes):
        gbs = nbytes / t / 1e9
        return {"us": t * 1e6, "bytes": nbytes, "gbs": gbs, "frac_hbm": gbs / hbm,
                "frac_8tbs": gbs / 8000.0}

    flops = 4.0 * T_kept * d * F
    res = {
        "router": bw("router", t_router, T * d * es + N * d * 4 + T * 8),
        "router_with_probs": bw("router", t_router_p, T * d * es + N * d * 4 + T * 8 + T * N * 4),
        "dispatch_metadata": {"us": t_disp * 1e6,
                              "bytes": T * 4 + T * 5 + N * 4 + N * C * 4},
        "dispatch_gather": bw("dispatch", t_disp_g,
                              T * 9 + N * 4 + N * C * 4 + T_kept * d * es + N * C * d * es),
        "expert_ffn": {"us": t_ffn * 1e6, "useful_flops": flops, "tflops": flops / t_ffn / 1e12,
                       "frac_burst": flops / t_ffn / 1e12 / pk["bf16_tflops"],
                       "frac_sustained": flops / t_ffn / 1e12 / pk["bf16_tflops_sustained"],
                       "weight_bytes": 2 * N * d * F * es, "traffic": None},
        "combine": bw("combine", t_comb, 2 * T * d * es + T_kept * d * es + T * 13),
        "aux_loss_from_probs": bw("aux", t_aux, T * N * 4 + N * 4),
        "layer_top2": None if t_top2 is None else {
            "us": t_top2 * 1e6, "tokens_per_s": T / t_top2,
            "capacity": sm.switch_capacity(2 * T, N, wl.capacity_factor)},
        "layer_backward": None if t_bwd is None else {
            "us": t_bwd * 1e6, "tokens_per_s": T / t_bwd,
            # algorithmic: dH, dW2, dW1, dX (2 T_kept d F each) + dW_r and dh W_r
            "useful_flops": 8.0 * T_kept * d * F + 4.0 * T * N * d,
            "recompute_flops": 2.0 * T_kept * d * F + 2.0 * T * N * d,
            "tflops": (8.0 * T_kept * d * F + 4.0 * T * N * d) / t_bwd / 1e12,
            "tflops_with_recompute": (10.0 * T_kept * d * F + 6.0 * T * N * d) / t_bwd / 1e12,
            "frac_burst_with_recompute": (10.0 * T_kept * d * F + 6.0 * T * N * d) / t_bwd / 1e12
                                         / pk["bf16_tflops"]},
        "layer_backward_saved": None if t_bwd_saved is None else {
            "us": t_bwd_saved * 1e6, "tokens_per_s": T / t_bwd_saved,
            "tflops": (8.0 * T_kept * d * F + 4.0 * T * N * d) / t_bwd_saved / 1e12,
            "frac_burst": (8.0 * T_kept * d * F + 4.0 * T * N * d) / t_bwd_saved / 1e12
                          / pk["bf16_tflops"],
            "note": "SWITCH_FLAG_TRAINING: activations kept by the forward, no recompute"},
        "layer_backward_top2": None if t_bwd2 is None else {
            "us": t_bwd2 * 1e6, "tokens_per_s": T / t_bwd2, "kept_assignments": T_kept2,
            "useful_flops": 8.0 * T_kept2 * d * F + 4.0 * T * N * d,
            "tflops_with_recompute": (10.0 * T_kept2 * d * F + 6.0 * T * N * d) / t_bwd2 / 1e12,
            "note": "SWITCH_FLAG_TOP2, routing, dispatch and H recomputed"},
        "training_step": None if t_train is None else {
            "us": t_train * 1e6, "tokens_per_s": T / t_train,
            "tflops": (12.0 * T_kept * d * F + 6.0 * T * N * d) / t_train / 1e12,
            "note": "switch_layer_forward + switch_layer_backward, SWITCH_FLAG_TRAINING"},
        "peaks": {"hbm_gbs": hbm, "bf16_tflops": pk["bf16_tflops"], "kind": pk_kind},
        "_T_kept": T_kept,
    }
    return res


if __name__ == "__main__":
    main()
