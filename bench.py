"""Benchmark of the MoE-layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

One step is one moe_forward over one batch of the workload (router GEMM,
top-k + gates, dispatch layout with the deduplicated send layout, permute,
grouped SwiGLU GEMMs, combine).  Default workload: configuration 2 of the
MoE layer set (T=16384 tokens, d=256, E=64 SwiGLU experts of width 64,
top-4, bf16, EP=8 contiguous), the fine-grained expert layer.

Timing: inputs resident in HBM; L2 is flushed (a 256 MB write) before each
step, outside the step's CUDA events; the K steps sit between a barrier and
a device synchronisation on both sides; with N > 1 ranks (torchrun, one per
GPU) each rank runs its own replica of the workload on its own tokens (the
layer shards by tokens with no exchange), and the slowest rank's time
counts.  Prints one JSON line on rank 0.

`--impl reference` times the CPU oracle (the only reference this method
has) on a bounded sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import routing_dispatch_experts_b200 as moe  # noqa: E402
from routing_dispatch_experts_b200 import workloads as W  # noqa: E402

METRIC = "MoE-layer fwd routed tokens/s"
L2_FLUSH_BYTES = 256 << 20
SLEEP_CYCLES = 200_000  # ~0.1 ms of device-side sleep before each timed iteration
# kernels of one moe_forward: bf16 = fused router, layout scatter, (permute
# when x is larger than 96 MB), gate/up GEMM, down GEMM, combine; fp32 =
# router, top-k, layout histogram, layout scatter, permute, gate/up, down,
# combine


def fused_ffn(w: W.Workload) -> bool:
    """moe_forward runs the expert FFN as one kernel (H on chip) for these."""
    return w.dtype == "bf16" and w.f in (64, 128) and w.d in (128, 256)


def launches_per_step(w: W.Workload) -> int:
    if w.dtype != "bf16":
        return 8
    permute = 1 if w.T * w.d * 2 > (96 << 20) else 0
    # route, scatter, [permute], gate/up [+ down], combine
    return (4 if fused_ffn(w) else 5) + permute
MEASURED_PEAKS = os.path.join(ROOT, "MEASURED_PEAKS.json")


def peaks():
    try:
        p = json.load(open(MEASURED_PEAKS))
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sus=p["bf16_tflops_sustained"],
                    sm_max_mhz=p.get("sm_max_mhz", 1965.0), src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, sm_max_mhz=1965.0, src="fallback")


# DRAM bytes (read + write) per launch of the dominant kernel, from one ncu
# capture of that kernel as committed (cold cache, the profiles directory
# holds the summary); None where no capture of the current kernel exists
NCU_TRAFFIC = {
    (2, "gate_up"): 14_992_128 + 89_088,  # ffn_fused_kernel<64, 256, gather>
}


# ------------------------------------------------------------ algorithmic work
def work(w: W.Workload, T: int):
    """Algorithmic bytes / FLOPs of each forward stage for T tokens: what the
    method must move or compute, not what a particular kernel happens to
    move.  Stages as moe_forward_timed names them."""
    b = 2 if w.dtype == "bf16" else 4
    R = T * w.k
    out = {
        # x read, W_r read, logits + idx + gate written
        "route": dict(bytes=T * w.d * b + w.E * w.d * b + T * w.E * 4 + 2 * R * 4,
                      flops=2 * T * w.d * w.E),
        # idx read; row_token, slot_row, send_token, slot_send_row written
        "layout": dict(bytes=R * 4 + 4 * R * 4, flops=0),
        # x read once, x_perm written, row indices read
        "permute": dict(bytes=T * w.d * b + R * w.d * b + R * 4, flops=0),
        # rows of x (or x_perm) read, W_g / W_u read, h written
        "gate_up": dict(bytes=R * w.d * b + 2 * w.E * w.d * w.f * b + R * w.f * b,
                        flops=4 * R * w.d * w.f),
        # h read, W_d read, y_perm written
        "down": dict(bytes=R * w.f * b + w.E * w.f * w.d * b + R * w.d * b,
                     flops=2 * R * w.d * w.f),
        # y_perm read, gates / slot rows read, y written
        "combine": dict(bytes=R * w.d * b + T * w.d * b + 2 * R * 4, flops=0),
    }
    if fused_ffn(w):
        # one kernel for the whole expert FFN, timed as the gate/up stage:
        # rows of x read, W_g / W_u / W_d read, y_perm written (h stays on chip)
        out["gate_up"] = dict(bytes=R * w.d * b + 3 * w.E * w.d * w.f * b + R * w.d * b,
                              flops=6 * R * w.d * w.f)
        out["down"] = dict(bytes=0, flops=0)
    return out


# ------------------------------------------------------------------- helpers
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled in the background."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.p = None
        self.out = []

    def start(self):
        try:
            self.p = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            out, _ = self.p.communicate(timeout=5)
        except Exception:
            self.p.kill()
            out = ""
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [v.strip() for v in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus):
    if n_gpus <= 1 and "RANK" not in os.environ:
        return 0, 1, 0
    import datetime
    import torch.distributed as dist
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", local))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """The largest of every rank's v (a timing is the slowest rank's)."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def config_of(w: W.Workload, world: int) -> dict:
    """The workload a bench line measures (the same for both arms)."""
    return {"workload": f"MoE layer config {w.cfg} ({w.name}): {w.describe()}",
            "T": w.T, "d": w.d, "E": w.E, "f": w.f, "k": w.k, "ep": w.eps[0],
            "routed_rows_per_step": w.T * w.k,
            "l2": "flushed before every step (256 MB write, outside the step events)",
            "parallelism": f"replicas x{world} (tokens sharded, no exchange)"}


def replica_seed(base: int, rank: int) -> int:
    """Every replica draws its own tokens (the layer shards by tokens)."""
    return base + rank


def job_value(T: int, world: int, ms: float) -> float:
    """Whole-job routed tokens/s: all ranks' tokens over the slowest rank's
    step time (weak scaling: T tokens per rank)."""
    return T * world / (ms * 1e-3)


# ----------------------------------------------------------------- our arm
def run_ours(args, rank, world, local):
    w = W.WORKLOADS[args.config]
    T = w.T
    ep = w.eps[0]
    seed = replica_seed(args.seed, rank)
    dev = torch.device("cuda", local)
    x = W.make_x(w, seed, T)
    wr = W.make_router(w, args.seed)
    bias = W.make_bias(w, args.seed)
    wg, wu, wd = W.make_experts(w, args.seed)
    shape = moe.Shape(T=T, d=w.d, E=w.E, k=w.k, f=w.f, ep=ep, dtype=w.torch_dtype)
    dx = x.to(dev)
    dbias = None if bias is None else bias.to(dev)
    packed = moe.pack_weights(shape, wr.to(dev), wg.to(dev), wu.to(dev), wd.to(dev))
    del wg, wu, wd
    ws = moe.workspace(shape, forward=True, device=dev)
    buf = moe.ForwardBuffers(shape, device=dev)
    y = torch.empty((T, w.d), dtype=w.torch_dtype, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    rmap = None if (w.placements[0] == "contiguous") else W.permutation_placement(w.E, ep, args.seed)

    def step():
        moe.forward(shape, dx, packed, dbias, ws, expert_rank=rmap, y=y, buffers=buf)

    def graph_of(fn):
        # the whole call sequence in one CUDA graph: one launch per step
        fn()
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            fn()
        torch.cuda.synchronize(dev)
        return g

    side = torch.cuda.Stream(dev)
    clocks = ClockSampler(local)
    clocks.start()
    step_graph = graph_of(step)
    # warm-up (at least W steps, and long enough for the clock sampler to see load)
    t_end = time.time() + (0.0 if args.profile else 1.0)
    i = 0
    while i < args.warmup or time.time() < t_end:
        flush.fill_(i & 0xFF)
        step_graph.replay()
        i += 1
        if i % 64 == 0:
            torch.cuda.synchronize(dev)
    torch.cuda.synchronize(dev)
    moe.check_device_status(ws)

    def timed(run, n, gap=True):
        """Per-iteration CUDA-event durations of run(); before each, L2 is
        flushed and a short device-side sleep lets the host queue the
        iteration, so no host launch gap falls inside the events."""
        e = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(n)]
        for i in range(n):
            flush.fill_(i & 0xFF)
            if gap:
                torch.cuda._sleep(SLEEP_CYCLES)
            e[i][0].record(stream)
            run()
            e[i][1].record(stream)
        torch.cuda.synchronize(dev)
        return [a.elapsed_time(b) for a, b in e]

    # ---- timed region: K steps, L2 flushed before each
    barrier(world)
    torch.cuda.synchronize(dev)
    step_ms = timed(step_graph.replay, args.steps)
    barrier(world)
    ms = max_over_ranks(sum(step_ms) / len(step_ms), world)
    moe.check_device_status(ws)
    # the same steps issued eagerly (one moe_forward call each, no graph)
    eager_ms = sum(timed(step, args.steps)) / args.steps

    # ---- per-stage device times inside the forward (moe_forward_timed:
    # events recorded between the stages on the launching stream), same L2
    # flush and host lead as the timed steps
    nst = len(moe.FORWARD_STAGES)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)]
    for e in evs:
        e.record(stream)
    reps = max(args.steps, 20)
    acc = [0.0] * nst
    for i in range(reps):
        flush.fill_(i & 0xFF)
        torch.cuda._sleep(SLEEP_CYCLES)
        moe.forward_timed(shape, dx, packed, dbias, ws, evs, expert_rank=rmap, y=y, buffers=buf)
        torch.cuda.synchronize(dev)
        for j in range(nst):
            acc[j] += evs[j].elapsed_time(evs[j + 1])
    calls = {name: acc[j] / reps for j, name in enumerate(moe.FORWARD_STAGES)}
    moe.check_device_status(ws)
    clk = clocks.stop()
    if args.profile:
        return {"profile": True, "ms_per_step": ms, "stage_ms": calls}

    # ---- end to end through the public API with host buffers: every step
    # copies its own x host -> device (pinned) and its y device -> host.
    # Steps are pipelined the way a serving loop runs them: device x / y are
    # double-buffered and the two copy directions run on their own streams,
    # so step i's copies overlap the forwards of steps i-1 and i+1 (the
    # forwards themselves stay in order on one stream).
    x_host = x.pin_memory()
    dx2 = [dx, torch.empty_like(dx)]
    y2 = [y, torch.empty_like(y)]
    y_host = [torch.empty((T, w.d), dtype=w.torch_dtype).pin_memory() for _ in range(2)]
    graphs = [step_graph,
              graph_of(lambda: moe.forward(shape, dx2[1], packed, dbias, ws, expert_rank=rmap,
                                           y=y2[1], buffers=buf))]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def run_e2e(n):
        fwd_done = [None, None]  # the last forward that read dx2[b] / wrote y2[b]
        out_done = [None, None]  # the last copy-out of y2[b]
        for i in range(n):
            b = i & 1
            with torch.cuda.stream(s_in):
                if fwd_done[b] is not None:
                    s_in.wait_event(fwd_done[b])
                dx2[b].copy_(x_host, non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
            stream.wait_event(ev_in)
            if out_done[b] is not None:
                stream.wait_event(out_done[b])
            graphs[b].replay()
            ev_fw = torch.cuda.Event()
            ev_fw.record(stream)
            fwd_done[b] = ev_fw
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_fw)
                y_host[b].copy_(y2[b], non_blocking=True)
                ev_out = torch.cuda.Event()
                ev_out.record(s_out)
                out_done[b] = ev_out

    e2e_ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    run_e2e(4)
    torch.cuda.synchronize(dev)
    barrier(world)
    e2e_ev[0].record(s_in)
    run_e2e(args.steps)
    e2e_ev[1].record(s_out)
    torch.cuda.synchronize(dev)
    barrier(world)
    e2e_ms = max_over_ranks(e2e_ev[0].elapsed_time(e2e_ev[1]) / args.steps, world)
    # the pipelined loop returned the same y as the timed forward
    if not torch.equal(y_host[(args.steps - 1) & 1], y.cpu()):
        raise RuntimeError("end-to-end loop produced a different y")

    wk = work(w, T)
    dom = max(calls, key=calls.get)
    pk = peaks()
    d = wk[dom]
    # steps that ran at the power-capped clock (the sampler saw sw_power_cap
    # during the timed region, or the step is a millisecond or more) take the
    # sustained GEMM peak as denominator, the others the burst one
    sustained = ms >= 1.0 or bool(clk and "sw_power_cap" in clk.get("reasons", []))
    tpeak = pk["bf16_sus"] if sustained else pk["bf16"]
    if w.dtype != "bf16" and d["flops"] > 0:
        # fp32 expert GEMMs run on the CUDA cores' FMA pipes: SMs x 128 fp32
        # lanes x 2 FLOP per clock at the maximum SM clock
        props = torch.cuda.get_device_properties(dev)
        fma_peak = props.multi_processor_count * 128 * 2 * pk["sm_max_mhz"] * 1e6 / 1e12
        bound, achieved, peak, unit = "alu", d["flops"] / (calls[dom] * 1e-3) / 1e12, fma_peak, "TFLOP/s"
        psrc = (f"derived: {props.multi_processor_count} SMs x 128 fp32 lanes x 2 FLOP x "
                f"{pk['sm_max_mhz']:.0f} MHz")
    elif d["flops"] > 0 and d["flops"] / d["bytes"] > tpeak * 1e12 / (pk["hbm"] * 1e9):
        bound, achieved, peak, unit = "tensor", d["flops"] / (calls[dom] * 1e-3) / 1e12, tpeak, "TFLOP/s"
        psrc = pk["src"] + (" bf16 sustained" if sustained else " bf16 burst")
    else:
        bound, achieved, peak, unit = "hbm", d["bytes"] / (calls[dom] * 1e-3) / 1e9, pk["hbm"], "GB/s"
        psrc = pk["src"] + " hbm copy"
    result = {
        "metric": METRIC,
        "value": job_value(T, world, ms),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": config_of(w, world),
        "e2e": {"value": job_value(T, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": x.numel() * x.element_size(),
                "d2h_bytes_per_step": y.numel() * y.element_size(),
                "pipelining": "device x / y double-buffered; host->device and device->host "
                              "copies on their own streams overlap the neighbouring steps"},
        "gpu_launches": launches_per_step(w) * args.steps,
        "ms_per_step_eager": eager_ms,
        "step": f"one moe_forward ({launches_per_step(w)} kernels) replayed from a CUDA graph",
        "stage_ms": {k: round(v, 5) for k, v in calls.items()},
        "roofline": {"kernel": dom, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak, "peak_source": psrc,
                     "traffic": NCU_TRAFFIC.get((args.config, dom)),
                     "algorithmic": d},
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.profile:
        result["cpu_baseline"] = cpu_baseline(w, args)
    return result


# ------------------------------------------------- CPU oracle (reference arm)
def cpu_baseline(w: W.Workload, args, budget_s: float = 12.0):
    """The oracle, as it stands, on a bounded seeded sample of the workload's
    tokens (routing, layout of the sample, experts, combine), scaled to
    tokens/s.  Runs on the host cores."""
    import oracle
    oracle.build()
    x = W.make_x(w, args.seed, w.T)
    wr = W.make_router(w, args.seed)
    bias = W.make_bias(w, args.seed)
    wg, wu, wd = W.make_experts(w, args.seed)

    def run(n):
        toks = W.sample_tokens(w.T, n, seed=args.seed + 5)
        t0 = time.perf_counter()
        r = oracle.forward(x, wr, bias, wg, wu, wd, w.k, tokens=toks)
        oracle.dispatch_layout(r["idx"], w.E, w.eps[0])
        return time.perf_counter() - t0

    n = 64
    dt = run(n)
    while dt < budget_s / 4 and n < w.T:
        n = min(w.T, int(n * max(2.0, budget_s / 2 / max(dt, 1e-3))))
        dt = run(n)
    return {"value": n / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} of {w.T} tokens (seeded), full router + top-k + layout + experts + combine in float64"}


def run_reference(args, rank, world):
    w = W.WORKLOADS[args.config]
    if rank != 0:
        return None
    cb = cpu_baseline(w, args, budget_s=max(5.0, 2.0 * args.steps))
    return {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": w.T / cb["value"] * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, world),
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=2, choices=sorted(W.WORKLOADS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="short run for a profiler: no clock warm-up, e2e or CPU baseline")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", 0))
        world = int(os.environ.get("WORLD_SIZE", 1))
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    rank, world, local = dist_setup(args.gpus)
    res = run_ours(args, rank, world, local)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
