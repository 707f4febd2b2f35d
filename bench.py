"""Benchmark of the MoE-layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

One step is one moe_forward over one batch of the workload (router GEMM,
top-k + gates, dispatch layout with the deduplicated send layout, permute,
grouped SwiGLU GEMMs, combine).  Default workload: configuration 5 of the
MoE layer set, the largest that fits one GPU (T=32768 tokens, d=4096,
E=128 SwiGLU experts of width 1536, top-8, bf16, Zipf(1.1) logit bias,
EP=16 contiguous); `--config N` selects the others.

Timing: inputs resident in HBM; L2 is flushed (a 256 MB write) before each
step, outside the step's CUDA events; the K steps sit between a barrier and
a device synchronisation on both sides; with N > 1 ranks (torchrun, one per
GPU) each rank runs its own replica of the workload on its own tokens (the
layer shards by tokens with no exchange), and the slowest rank's time
counts.  Prints one JSON line on rank 0.

`--impl reference` times the CPU oracle (the only reference this method
has) on a bounded sample of the same workload, on the host cores.

`--kernel NAME` runs one entry point alone (see run_kernel) for profiler
captures and per-kernel timing.
"""
from __future__ import annotations

import argparse
import dataclasses
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
# the largest workload that fits one GPU (T=32768, d=4096, E=128, f=1536, top-8)
DEFAULT_CONFIG = 5
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
    # gemm_tc_kernel<256, SwiGLU, gather>: a quarter-size capture (4096 of
    # 16384 tokens, 16 of 64 experts, same rows per expert) scaled by 4
    (3, "gate_up"): 4 * (157_522_688 + 11_830_272),
    # the same kernel on the top-6 workload's quarter case, scaled by 4
    (4, "gate_up"): 4 * (165_850_880 + 37_479_168),
    # grouped_f32_kernel<SwiGLU> at the tiny workload's full size
    (1, "gate_up"): 16_829_440,
    # gemm_tc_kernel<256, SwiGLU> (one CTA per tile, the forward's gate/up
    # engine on this workload): a quarter-size capture (32 of 128 experts,
    # same rows per expert) scaled by 4
    (5, "gate_up"): 4 * (1_424_801_792 + 197_288_192),
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
    if w.dtype == "bf16" and T * w.d * b <= (96 << 20):
        # the gate/up GEMM (or fused FFN) gathers the rows of x itself: no
        # permute kernel runs, and its bytes are the GEMM's row reads
        out["permute"] = dict(bytes=0, flops=0)
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


def exchange_splits(idx, rank_map, P: int, dedup: bool):
    """Rows one rank sends each of the P ranks for its routing idx [T, k]
    under an expert -> rank map: one row per assignment (dedup False, the
    per-expert dispatch B of 'Expert Coupling', Fig. 7) or one row per
    (token, destination rank) (dedup True, D)."""
    import numpy as np
    owner = np.asarray(rank_map, dtype=np.int64)[np.asarray(idx, dtype=np.int64)]
    if not dedup:
        return np.bincount(owner.ravel(), minlength=P)[:P].astype(np.int64)
    hit = np.zeros((owner.shape[0], P), dtype=bool)
    np.put_along_axis(hit, owner, True, axis=1)
    return hit.sum(0).astype(np.int64)


def time_exchange(send_splits, rank: int, world: int, row_elems: int, dtype, dev, reps: int = 5):
    """The all-to-all of one dispatch plan across the ranks (row payloads
    only): every rank's send splits are all-gathered, then the rows move
    with dist.all_to_all_single; median of `reps` timed calls (CUDA events
    on the GPU), the slowest rank's.  Returns (ms, rows this rank puts on
    the wire, i.e. to other ranks)."""
    import statistics as st
    import torch.distributed as dist
    mine = torch.tensor([int(v) for v in send_splits], dtype=torch.int64, device=dev)
    allc = torch.empty(world * world, dtype=torch.int64, device=dev)
    dist.all_gather_into_tensor(allc, mine)
    C = allc.view(world, world).cpu().tolist()
    send = [int(C[rank][r]) for r in range(world)]
    recv = [int(C[q][rank]) for q in range(world)]
    inp = torch.empty((sum(send), row_elems), dtype=dtype, device=dev)
    out = torch.empty((sum(recv), row_elems), dtype=dtype, device=dev)
    cuda = dev.type == "cuda"
    for _ in range(2):
        dist.all_to_all_single(out, inp, output_split_sizes=recv, input_split_sizes=send)
    times = []
    for _ in range(reps):
        dist.barrier()
        if cuda:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            e0.record()
            dist.all_to_all_single(out, inp, output_split_sizes=recv, input_split_sizes=send)
            e1.record()
            torch.cuda.synchronize(dev)
            times.append(e0.elapsed_time(e1))
        else:
            t0 = time.perf_counter()
            dist.all_to_all_single(out, inp, output_split_sizes=recv, input_split_sizes=send)
            times.append((time.perf_counter() - t0) * 1e3)
    ms = max_over_ranks(st.median(times), world)
    return ms, sum(send) - send[rank]


def ep_exchange(idx, contiguous_map, correlated_map, rank: int, world: int, d: int, dtype, dev):
    """Fig. 7 of 'Expert Coupling' on the ranks of this job (P = world):
    the dispatch all-to-all of every rank's measured batch one row per
    assignment (B), deduplicated under contiguous placement (D) and under
    the correlated placement (D+P)."""
    out = {"ranks": world, "row_bytes": d * torch.tensor([], dtype=dtype).element_size(),
           "tokens_per_rank": int(idx.shape[0])}
    for name, m, dedup in (("B", contiguous_map, False), ("D", contiguous_map, True),
                           ("D+P", correlated_map, True)):
        ms, wire = time_exchange(exchange_splits(idx, m, world, dedup), rank, world, d, dtype, dev)
        wire_max = int(max_over_ranks(float(wire), world))
        out[name] = {"ms": round(ms, 4), "wire_rows_max_rank": wire_max,
                     "wire_GB_s_max_rank": round(wire_max * out["row_bytes"] / (ms * 1e-3) / 1e9, 1)}
    out["timing"] = ("dist.all_to_all_single of the row payloads (NCCL), CUDA events, median of 5, "
                     "slowest rank; not part of the timed step")
    return out


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
    cpu_leg = rank == 0 and world == 1 and not args.no_cpu_baseline and not args.profile
    # the CPU baseline reuses the host copies of the inputs (drawing the large
    # workload's experts again would take minutes)
    host_inputs = (x, wr, bias, wg, wu, wd) if cpu_leg else None
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
    # router observability of the measured batch (outside the timed region):
    # tokens whose top-k margin is below the near-tie bound, where routing
    # may flip between runs or implementations
    rstats, _ = moe.router_stats(shape, buf.logits, buf.topk_idx, threshold=1e-5)
    # the deduplicated send plan of the measured batch ('Expert Coupling',
    # Table I: GPUs per token, rows removed by deduplication)
    dstats = moe.stats_dict(buf.layout["stats"])
    # rows on the wire of the measured batch under each EP degree the
    # workload names: one row per assignment (B), deduplicated under the
    # contiguous placement (D) and under the correlated placement fitted on
    # a calibration batch (D+P) ('Expert Coupling', Fig. 7; Table III's
    # co-selection counts and the greedy fit, both on the GPU)
    placement_rows = {}
    if shape.ep > 1 and not args.profile:
        cal_T = min(T, 4096)
        cshape = dataclasses.replace(shape, T=cal_T)
        cws = moe.workspace(cshape, device=dev)
        cal = W.make_x(w, args.seed, cal_T, stream="calib").to(dev)
        _, cidx, _ = moe.route(cshape, cal, packed, dbias, cws)
        co = moe.coselection_counts(cshape, cidx, cws)
        for P_ in w.eps:
            s_ = dataclasses.replace(shape, ep=P_)
            ws_ = moe.workspace(s_, device=dev)
            for name, m_ in (("D_contiguous", W.contiguous_placement(w.E, P_)),
                             ("D+P_correlated", moe.fit_placement(w.E, P_, co))):
                lay_ = moe.dispatch_layout(s_, buf.topk_idx, ws_, expert_rank=m_)
                placement_rows[f"ep{P_}_{name}"] = moe.stats_dict(lay_["stats"])["rows_sent"]
                moe.check_device_status(ws_)
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
    # the stage is timed inside a step of milliseconds, not a seconds-long
    # loop, so the burst GEMM peak is the denominator; the fraction of the
    # sustained (power-capped) peak is printed beside it
    tpeak = pk["bf16"]
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
        psrc = pk["src"] + " bf16 burst"
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
    if bound == "tensor":
        result["roofline"]["frac_of_sustained"] = achieved / pk["bf16_sus"]
    if ep > 1:
        R = T * w.k
        result["dispatch"] = {
            "ep": ep, "placement": w.placements[0],
            "rows_per_expert_dispatch": R, "rows_deduplicated": dstats["rows_sent"],
            "rows_removed": dstats["dup_removed"], "rows_removed_frac": dstats["dup_removed"] / R,
            "gpus_per_token": dstats["rows_sent"] / T,
            "tokens_on_one_rank": dstats["tokens_single_rank"],
            "home_rank_assignment_frac": dstats["home_rank_rows"] / R,
            "computed_by": "moe_forward's dispatch layout (device statistics)",
            "rows_sent_by_placement": dict(B_per_assignment=R, **placement_rows),
            "placement_fit": "greedy correlated fit of co-selection counts of a 4096-token "
                             "calibration batch (moe_coselection_counts, moe_fit_placement)"}
    if world > 1 and w.E % world == 0:
        # the exchange the dedup send plan is for, on this job's ranks: the
        # same calibration batch and router on every rank give the same
        # correlated placement everywhere
        cal_T = min(T, 4096)
        cshape = moe.Shape(T=cal_T, d=w.d, E=w.E, k=w.k, f=w.f, ep=world, dtype=w.torch_dtype)
        cws = moe.workspace(cshape, device=dev)
        cal = W.make_x(w, args.seed, cal_T, stream="calib").to(dev)
        _, cidx, _ = moe.route(cshape, cal, packed, dbias, cws)
        fit = moe.fit_placement(w.E, world, moe.coselection_counts(cshape, cidx, cws))
        result["ep_exchange"] = ep_exchange(buf.topk_idx.cpu().numpy(),
                                            W.contiguous_placement(w.E, world), fit, rank, world,
                                            w.d, w.torch_dtype, dev)
    result["routing"] = {"near_tie_tokens": rstats["near_tie_tokens"],
                         "near_tie_share": rstats["near_tie_tokens"] / max(T, 1),
                         "near_tie_threshold": 1e-5,
                         "computed_by": "moe_router_stats on the timed forward's logits"}
    result["stage_roofline"] = stage_rooflines(wk, calls, pk)
    if cpu_leg:
        result["cpu_baseline"] = cpu_baseline(w, args, inputs=host_inputs,
                                              gpu_idx=buf.topk_idx.cpu().numpy())
        result["routing_check"] = result["cpu_baseline"].pop("routing_check")
    return result


def stage_rooflines(wk, calls, pk):
    """Every stage's fraction of its own roofline: HBM copy bandwidth for the
    data-movement stages, the burst bf16 GEMM peak (and the sustained one)
    for the expert GEMMs; stages that a path fuses into another are left
    out."""
    out = {}
    for name, ms in calls.items():
        d = wk[name]
        if ms <= 0 or (d["bytes"] == 0 and d["flops"] == 0):
            continue
        gbs = d["bytes"] / (ms * 1e-3) / 1e9
        e = {"ms": round(ms, 5), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm"], 4)}
        if d["flops"] and d["flops"] / d["bytes"] > pk["bf16"] * 1e12 / (pk["hbm"] * 1e9):
            tf = d["flops"] / (ms * 1e-3) / 1e12
            e.update({"TFLOP/s": round(tf, 1), "frac_bf16_burst": round(tf / pk["bf16"], 4),
                      "frac_bf16_sustained": round(tf / pk["bf16_sus"], 4)})
        out[name] = e
    return out


# ------------------------------------------------- CPU oracle (reference arm)
def cpu_baseline(w: W.Workload, args, budget_s: float = 12.0, inputs=None, gpu_idx=None):
    """The oracle, as it stands, on a bounded seeded sample of the workload's
    tokens (router, top-k and gates of the sample, its dispatch layout, its
    experts and combine, all in float64), with the sample's rate taken as
    the batch's tokens/s: tokens are independent once routed, so the
    sample's rate extrapolates to the whole batch.  Runs on the host cores.
    With `gpu_idx` (the GPU's routing of the whole batch) it also counts the
    sampled tokens whose expert sets differ from the oracle's, and how many
    of those are not near-ties (margin below 1e-5)."""
    import oracle
    oracle.build()
    if inputs is None:
        x = W.make_x(w, args.seed, w.T)
        wr = W.make_router(w, args.seed)
        bias = W.make_bias(w, args.seed)
        wg, wu, wd = W.make_experts(w, args.seed)
    else:
        x, wr, bias, wg, wu, wd = inputs

    def run(n):
        toks = W.sample_tokens(w.T, n, seed=args.seed + 5)
        t0 = time.perf_counter()
        r = oracle.forward(x, wr, bias, wg, wu, wd, w.k, tokens=toks)
        oracle.dispatch_layout(r["idx"], w.E, w.eps[0])
        return time.perf_counter() - t0, toks, r

    n = 64
    dt, toks, r = run(n)
    while dt < budget_s / 4 and n < w.T:
        n = min(w.T, int(n * max(2.0, budget_s / 2 / max(dt, 1e-3))))
        dt, toks, r = run(n)
    what = "router, top-k, layout, experts and combine in float64"
    sample = (f"all {w.T} tokens: {what}" if n == w.T else
              f"{n} of {w.T} tokens (seeded): {what}; tokens/s of the sample, extrapolated "
              f"to the batch (tokens are independent once routed)")
    out = {"value": n / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
           "sample": sample, "extrapolated": n < w.T}
    if gpu_idx is not None:
        import numpy as np
        gi = gpu_idx[toks.numpy()]
        bad = np.where((np.sort(gi, 1) != np.sort(r["idx"], 1)).any(1))[0]
        m = oracle.margin(r["logits"], w.k)
        out["routing_check"] = {"tokens": n, "mismatches": int(len(bad)),
                                "mismatches_not_near_tie": int((m[bad] >= 1e-5).sum()),
                                "near_tie_threshold": 1e-5,
                                "oracle_near_ties_in_sample": int((m < 1e-5).sum())}
    return out


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


# ------------------------------------------------- one kernel, for profilers
KERNELS = ("route", "topk", "layout", "permute", "permute_by_token", "grouped",
           "grouped_gather", "combine", "forward", "forward_routed", "forward_combine_in_down",
           "stats", "capacity",
           "coselection", "ep_pack",
           "ep_dispatch_peer", "ep_expert", "ep_home", "ep_signal")


def run_kernel(args):
    """One entry point of the library alone on a workload's seeded inputs,
    for profiler captures and per-kernel timing:

      route            moe_route (bf16: the fused router; fp32: router + top-k)
      topk             moe_route in given-logits mode (top-k + gates only)
      layout           moe_dispatch_layout (histogram + lookback, scatter)
      permute          moe_permute (row order)
      permute_by_token moe_permute_by_token (token order)
      grouped          moe_grouped_swiglu (gate/up GEMM + SwiGLU, down GEMM)
      grouped_gather   moe_grouped_swiglu_gather
      combine          moe_combine
      forward          moe_forward
      forward_routed   moe_forward_routed on the router's own routing (a
                       recorded routing table replayed: layout, experts and
                       combine, no router)
      forward_combine_in_down
                       moe_debug_forward_options with the combine summed in
                       the down GEMM's epilogue (the opt-in path)
      stats            moe_router_stats (margin, near-tie count)
      capacity         moe_capacity_keep (capacity factor 1.25)
      coselection      moe_coselection_counts (W[e,e'])
      ep_pack          moe_ep_pack (this rank's deduplicated send rows, ep = the
                       workload's EP degree)
      ep_dispatch_peer moe_ep_dispatch_peer (the same rows stored into one
                       receive buffer per destination rank, here all on this
                       GPU: the pack's stores where NVLink would carry them)
      ep_expert        moe_ep_expert_forward of rank 0 on the send rows this
                       batch sends it (layout over its experts, expert FFN,
                       partial combine)
      ep_home          moe_ep_home_combine (one returned row per send row)
      ep_signal        moe_ep_signal_wait of a single rank (its own flag)

    Routing comes from the workload's own router on its own x; expert
    weights are seeded N(0, 1/d) stand-ins drawn on the device (values do
    not change what the kernels move or compute), and kernels that never
    read them get f = 64 stand-ins.  `--tokens` / `--experts` shrink the
    case for captures (fewer tokens; fewer experts with the same EP degree).
    `--launches N` makes N launches and synchronises (a profiler picks
    among them); `--time REPS` times CUDA graphs of 10 x (256 MB L2 flush +
    launch) minus graphs of the 10 flushes alone and prints the median
    microseconds per launch."""
    import ctypes
    w = W.WORKLOADS[args.config]
    T = args.tokens or w.T
    E = args.experts or w.E
    ep = min(w.eps[0], E)
    dev = torch.device("cuda", 0)
    needs_experts = args.kernel in ("grouped", "grouped_gather", "forward", "forward_routed",
                                    "forward_combine_in_down", "ep_expert")
    f = w.f if needs_experts else 64
    shape = moe.Shape(T=T, d=w.d, E=E, k=w.k, f=f, ep=ep, dtype=w.torch_dtype)
    wc = dataclasses.replace(w, E=E) if E != w.E else w
    x = W.make_x(w, args.seed, T).to(dev)
    bias = W.make_bias(wc, args.seed)
    bias = None if bias is None else bias.to(dev)
    g = torch.Generator(device=dev).manual_seed(args.seed + 1)
    std = 1.0 / math.sqrt(w.d)

    def stand_in(*sz):
        return (torch.randn(*sz, generator=g, device=dev) * std).to(w.torch_dtype)

    packed = moe.pack_weights(shape, W.make_router(wc, args.seed).to(dev), stand_in(E, w.d, f),
                              stand_in(E, w.d, f), stand_in(E, f, w.d))
    ws = moe.workspace(shape, forward=args.kernel.startswith("forward"), device=dev)
    logits, idx, gate = moe.route(shape, x, packed, bias, ws)
    lay = moe.dispatch_layout(shape, idx, ws)
    torch.cuda.synchronize()
    moe.check_device_status(ws)
    R = shape.R
    L, sc, P = moe.lib(), shape.c, moe._p
    x_perm = moe.permute(shape, x, lay["row_token"]) if args.kernel.startswith("grouped") \
        or args.kernel == "combine" else None
    h = torch.empty((R, f), dtype=w.torch_dtype, device=dev) if needs_experts else None
    y_perm = torch.empty((R, w.d), dtype=w.torch_dtype, device=dev) if needs_experts else x_perm
    out = torch.empty((R, w.d), dtype=w.torch_dtype, device=dev) if "permute" in args.kernel \
        else torch.empty((T, w.d), dtype=w.torch_dtype, device=dev)
    idx2 = torch.empty_like(idx)
    gate2 = torch.empty_like(gate)
    counts = torch.zeros(5, dtype=torch.int64, device=dev)
    cosel = torch.empty((E, E), dtype=torch.int64, device=dev)
    send_rows = int(lay["rank_offsets"][-1]) if ep > 1 else 0
    if args.kernel in ("ep_pack", "ep_home", "ep_dispatch_peer", "ep_expert"):
        send = moe.ep_pack(shape, x, idx, gate, lay, send_rows) if ep > 1 else None
        y_back = send[0] if send is not None else None
    if args.kernel == "ep_dispatch_peer":
        if ep < 2:
            raise SystemExit("ep_dispatch_peer needs a workload with EP >= 2")
        rc = [int(v) for v in lay["rank_counts"].tolist()]
        recv = [(torch.empty((n, w.d), dtype=w.torch_dtype, device=dev),
                 torch.empty((n, w.k), dtype=torch.int32, device=dev),
                 torch.empty((n, w.k), dtype=torch.float32, device=dev)) for n in rc]
        dests = (moe.moe_ep_peer_dest * ep)(*[moe.moe_ep_peer_dest(P(a), P(b), P(c), 0, n)
                                              for (a, b, c), n in zip(recv, rc)])
    if args.kernel == "ep_expert":
        if ep < 2:
            raise SystemExit("ep_expert needs a workload with EP >= 2")
        n0 = int(lay["rank_offsets"][1])
        rshape = dataclasses.replace(shape, T=n0)
        rsc = rshape.c
        El = E // ep
        lshape = moe.Shape(T=n0, d=w.d, E=El, k=min(w.k, El), f=f, dtype=w.torch_dtype)
        packed_local = moe.pack_weights(lshape, None, stand_in(El, w.d, f), stand_in(El, w.d, f),
                                        stand_in(El, f, w.d))
        rws = moe.ep_expert_workspace(rshape, device=dev)
        y_ret = torch.empty((n0, w.d), dtype=w.torch_dtype, device=dev)
        recv = (send[0][:n0], send[1][:n0].contiguous(), send[2][:n0].contiguous())
    if args.kernel == "ep_signal":
        flags1 = torch.zeros(1, dtype=torch.int64, device=dev)
        fl_arr = (ctypes.c_void_p * 1)(P(flags1))
        epoch = [0]
    clay = moe._c_layout(moe._layout_tensors(shape, dev))
    clay_ep = moe._c_layout(lay)
    rmap = None

    def launch(stream=None):
        st = moe._stream(stream)
        k = args.kernel
        if k == "route":
            r = L.moe_route(ctypes.byref(sc), P(x), P(packed), P(bias), P(logits), P(idx2),
                            P(gate2), P(ws), ws.numel(), st)
        elif k == "topk":
            r = L.moe_route(ctypes.byref(sc), None, None, P(bias), P(logits), P(idx2), P(gate2),
                            P(ws), ws.numel(), st)
        elif k == "layout":
            r = L.moe_dispatch_layout(ctypes.byref(sc), P(idx), rmap, ctypes.byref(clay), P(ws),
                                      ws.numel(), st)
        elif k == "permute":
            r = L.moe_permute(ctypes.byref(sc), P(x), P(lay["row_token"]), P(out), st)
        elif k == "permute_by_token":
            r = L.moe_permute_by_token(ctypes.byref(sc), P(x), P(lay["slot_row"]), P(out), st)
        elif k == "grouped":
            r = L.moe_debug_grouped_swiglu_engine(ctypes.byref(sc), P(x_perm), None,
                                                  P(lay["expert_offsets"]), P(packed), P(h),
                                                  P(y_perm), P(ws), ws.numel(), args.engine, st)
        elif k == "grouped_gather":
            r = L.moe_debug_grouped_swiglu_engine(ctypes.byref(sc), P(x), P(lay["row_token"]),
                                                  P(lay["expert_offsets"]), P(packed), P(h),
                                                  P(y_perm), P(ws), ws.numel(), args.engine, st)
        elif k == "combine":
            r = L.moe_combine(ctypes.byref(sc), P(y_perm), P(lay["slot_row"]), P(gate), P(out), st)
        elif k == "stats":
            r = L.moe_router_stats(ctypes.byref(sc), P(logits), None, P(idx), None, 1e-5, None,
                                   P(counts), st)
        elif k == "coselection":
            r = L.moe_coselection_counts(ctypes.byref(sc), P(idx), P(cosel), P(ws), ws.numel(), st)
        elif k == "ep_pack":
            r = L.moe_ep_pack(ctypes.byref(sc), P(x), P(idx), P(gate), None, ctypes.byref(clay_ep),
                              P(send[0]), P(send[1]), P(send[2]), send_rows, st)
        elif k == "ep_dispatch_peer":
            r = L.moe_ep_dispatch_peer(ctypes.byref(sc), P(x), P(idx), P(gate), None,
                                       ctypes.byref(clay_ep), dests, st)
        elif k == "ep_expert":
            r = L.moe_ep_expert_forward(ctypes.byref(rsc), P(recv[0]), P(recv[1]), P(recv[2]),
                                        P(packed_local), P(y_ret), P(rws), rws.numel(), st)
        elif k == "ep_signal":
            epoch[0] += 1
            r = L.moe_ep_signal_wait(fl_arr, 0, 1, epoch[0], P(ws), st)
        elif k == "ep_home":
            r = L.moe_ep_home_combine(ctypes.byref(sc), P(y_back), P(lay["slot_send_row"]),
                                      send_rows, P(out), st)
        elif k == "capacity":
            r = L.moe_capacity_keep(ctypes.byref(sc), P(idx), P(gate), 1.25, P(idx2), P(gate2),
                                    None, P(ws), ws.numel(), st)
        elif k == "forward_routed":
            r = L.moe_forward_routed(ctypes.byref(sc), P(x), P(packed), P(idx), P(gate), rmap,
                                     P(out), None, P(ws), ws.numel(), st)
        elif k == "forward_combine_in_down":
            r = L.moe_debug_forward_options(ctypes.byref(sc), P(x), P(packed), P(bias), rmap,
                                            P(out), None, P(ws), ws.numel(),
                                            moe.FWD_COMBINE_IN_DOWN, st)
        else:
            r = L.moe_forward(ctypes.byref(sc), P(x), P(packed), P(bias), rmap, P(out), None,
                              P(ws), ws.numel(), st)
        moe._check(r, k)

    for _ in range(args.launches):
        launch()
    torch.cuda.synchronize()
    moe.check_device_status(ws)
    print(f"config {args.config} {args.kernel}: T={T} E={E} f={f} ep={ep}, "
          f"{args.launches} launches ok", flush=True)
    if not args.time:
        return
    reps = 10
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    side = torch.cuda.Stream(dev)

    def capture(with_kernel):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=side):
            for i in range(reps):
                flush.fill_(i & 255)
                if with_kernel:
                    launch(side)
        return gr

    g1, g0 = capture(True), capture(False)

    def run(gr):
        gr.replay()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        gr.replay()
        e1.record()
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) * 1e3

    d = [(run(g1) - run(g0)) / reps for _ in range(args.time)]
    moe.check_device_status(ws)
    us = statistics.median(d)
    print(json.dumps({"kernel": args.kernel, "engine": args.engine, "config": args.config, "T": T, "E": E,
                      "us_median": us, "us_min": min(d), "us_max": max(d), "reps": args.time}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=DEFAULT_CONFIG, choices=sorted(W.WORKLOADS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="short run for a profiler: no clock warm-up, e2e or CPU baseline")
    ap.add_argument("--kernel", choices=KERNELS,
                    help="run one entry point alone (profiler captures, per-kernel timing)")
    ap.add_argument("--tokens", type=int, default=0, help="--kernel: token count (default: the workload's)")
    ap.add_argument("--experts", type=int, default=0, help="--kernel: expert count (default: the workload's)")
    ap.add_argument("--launches", type=int, default=5, help="--kernel: launches before exit")
    ap.add_argument("--time", type=int, default=0, metavar="REPS", help="--kernel: timing repetitions")
    ap.add_argument("--engine", type=int, default=0, choices=(0, 1, 2, 3, 4),
                    help="--kernel grouped*: GEMM engine (0 library's choice, 1 one CTA per "
                         "tile, 2 CTA pairs, 3 pairs for the down GEMM, 4 for gate/up)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.kernel:
        run_kernel(args)
        return
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
