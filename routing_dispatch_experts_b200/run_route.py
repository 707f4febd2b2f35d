"""Run the router alone (moe_route) on a workload's seeded inputs, for
profilers and timing.

    python -m routing_dispatch_experts_b200.run_route --config 5 --launches 5
    python -m routing_dispatch_experts_b200.run_route --config 5 --time 9

The router reads x, W_r and the bias only; the expert weights it is packed
with are f = 64 stand-ins (random, never read), so the device holds x, W_r
and the outputs plus a few hundred MB.  `--launches N` makes N launches and
synchronises (an ncu capture selects among them); `--time REPS` times graphs
of 10 x (256 MB L2 flush + moe_route) minus graphs of the 10 flushes alone,
and prints the median microseconds per launch and the algorithmic bytes
(x, W_r read; logits, indices and gates written) per microsecond."""
import argparse
import ctypes
import statistics

import torch

import routing_dispatch_experts_b200 as moe
from routing_dispatch_experts_b200 import workloads as W


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", type=int, default=5, choices=sorted(W.WORKLOADS))
    ap.add_argument("--launches", type=int, default=5)
    ap.add_argument("--time", type=int, default=0, metavar="REPS")
    a = ap.parse_args()
    w = W.WORKLOADS[a.config]
    dev = torch.device("cuda", 0)
    f = 64
    shape = moe.Shape(T=w.T, d=w.d, E=w.E, k=w.k, f=f, ep=w.eps[0], dtype=w.torch_dtype)
    x = W.make_x(w, 0, w.T).to(dev)
    bias = W.make_bias(w, 0)
    bias = None if bias is None else bias.to(dev)
    g = torch.Generator(device=dev).manual_seed(1)
    ew = lambda *s: (torch.randn(*s, generator=g, device=dev) * 0.02).to(w.torch_dtype)
    packed = moe.pack_weights(shape, W.make_router(w, 0).to(dev), ew(w.E, w.d, f),
                              ew(w.E, w.d, f), ew(w.E, f, w.d))
    ws = moe.workspace(shape, device=dev)
    logits = torch.empty((w.T, w.E), dtype=torch.float32, device=dev)
    idx = torch.empty((w.T, w.k), dtype=torch.int32, device=dev)
    gate = torch.empty((w.T, w.k), dtype=torch.float32, device=dev)
    L, sc = moe.lib(), shape.c

    def launch(stream=None):
        moe._check(L.moe_route(ctypes.byref(sc), moe._p(x), moe._p(packed), moe._p(bias),
                               moe._p(logits), moe._p(idx), moe._p(gate), moe._p(ws),
                               ws.numel(), moe._stream(stream)), "moe_route")

    for _ in range(a.launches):
        launch()
    torch.cuda.synchronize()
    moe.check_device_status(ws)
    print(f"config {a.config}: {a.launches} router launches ok")
    if not a.time:
        return
    R = 10
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    side = torch.cuda.Stream()

    def capture(with_route):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=side):
            for i in range(R):
                flush.fill_(i & 255)
                if with_route:
                    launch(side)
        return gr

    g1, g0 = capture(True), capture(False)

    def run(gr):
        gr.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        gr.replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e3

    d = [(run(g1) - run(g0)) / R for _ in range(a.time)]
    moe.check_device_status(ws)
    us = statistics.median(d)
    nbytes = (w.T * w.d + w.E * w.d) * x.element_size() + w.T * w.E * 4 + 2 * w.T * w.k * 4
    print(f"config {a.config}: router {us:.2f} us per launch (median of {a.time}; "
          f"{min(d):.2f}-{max(d):.2f}), {nbytes / us / 1e3:.0f} GB/s algorithmic")


if __name__ == "__main__":
    main()
