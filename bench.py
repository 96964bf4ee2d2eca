"""Benchmark of the hard-routed sparse MoE layer forward on B200.

One step = one whole-layer forward (router logits, softmax/top-k, row sort,
grouped gate|up + SwiGLU, grouped down, combine) over one batch of seeded
synthetic input already resident in HBM, through the C ABI (moe_forward,
captured once in a CUDA graph and replayed).

Default workload: the 2,048-token prefill chunk (T=2048, d=2048, E=512,
top-10, F=512, 4-bit affine group-64 experts, bf16 activations). The decode
layer at T=1 and T=32 is timed in the same run and reported under
"decode".

Prints one JSON line (rank 0). Multi-GPU (torchrun): every rank runs an
independent replica on its own tokens (no collective on the data path);
value = all ranks' tokens / max-over-ranks device time.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the CPU fp64 oracle on host cores
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (read + write) of one gate|up launch on the prefill workload,
# from an ncu capture of that kernel (the stage call's grouped_tc_kernel<2, 0>
# as of the commit that trims its raw-ring bookkeeping: 675.49 MB read +
# 20.75 MB written); to be retaken whenever that kernel changes
GATE_UP_TRAFFIC = {"prefill": 696238336}
L2_FLUSH_BYTES = 256 << 20


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"moe_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
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
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ accounting

def expert_bytes(ex) -> int:
    return ex.nbytes_per_expert()


def gate_up_bytes(ex) -> int:
    tot = ex.w_gu[0].numel() * ex.w_gu.element_size()
    for t in (ex.s_gu, ex.b_gu):
        if t is not None:
            tot += t[0].numel() * t.element_size()
    return tot


def kernels_per_forward(T, k, regime_tc: bool, fused_decode: bool = False) -> int:
    if fused_decode:
        return 1                      # the whole layer in one cooperative kernel
    R = T * k
    sort = 1 if R <= 1024 else 3
    conv = 1                          # x -> fp16 (gathered for the tensor cores)
    return 2 + sort + conv + 2 + 1    # router + top-k, sort, x16, gate|up, down, combine


# ------------------------------------------------------------------ ranks

def max_over_ranks(vals, device):
    """Each value's maximum over all ranks (the slowest rank's time) when a
    process group is up; the values unchanged in a single process."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return [float(v) for v in vals]
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def replicas_tokens_per_s(world: int, T: int, ms: float) -> float:
    """Whole-job throughput of `world` independent replicas of T tokens each,
    timed by the slowest rank: every rank's tokens over that time."""
    return world * T / (ms * 1e-3)


# ------------------------------------------------------------------ timing

def time_device(fn, steps, warmup, flush):
    """Per-step CUDA-event time (ms) of fn() on the current stream. Before
    every step, outside the timed events, the L2 is flushed: a 256 MB buffer
    is written, then a second 256 MB buffer is read, so the dirty lines the
    write leaves are written back before the step starts and the step begins
    with a cold, clean L2."""
    wbuf, rbuf = flush
    for _ in range(warmup):
        fn()
    s = torch.cuda.current_stream()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    sink = torch.empty((), dtype=torch.float32, device=wbuf.device)
    torch.cuda.synchronize()
    for i in range(steps):
        wbuf.add_(1)
        torch.sum(rbuf, dim=0, out=sink)
        starts[i].record(s)
        fn()
        ends[i].record(s)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in zip(starts, ends)]


def time_layer(moe, layer, k, steps, warmup, flush, pk):
    """One workload's whole-layer forward, graph-replayed and timed like the
    headline step (L2 flushed before every step): ms per step, tokens/s, and
    the layer's algorithmic bytes (the experts with at least one routed row,
    read once, + x + y) and flops (6 R d F) as fractions of the peaks."""
    wl = layer.wl
    ws = moe.forward_workspace(layer.x, layer.experts, k)
    y = torch.empty(wl.T, wl.d, dtype=layer.x.dtype, device=layer.x.device)
    fwd = lambda: moe.forward(layer.x, layer.w_router, layer.router_bias, layer.experts, k,
                              ws=ws, out=y)
    fwd()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fwd()
    torch.cuda.synchronize()
    ms = statistics.mean(time_device(g.replay, steps, warmup, flush))
    L = moe.forward_layout(wl.T, wl.d, wl.E, k, wl.F, layer.x.dtype, wl.wfmt)
    counts = ws[L.counts:L.counts + wl.E * 4].view(torch.int32).cpu().numpy()
    active = int((counts > 0).sum())
    nbytes = active * expert_bytes(layer.experts) + 2 * wl.T * wl.d * layer.x.element_size()
    flops = 6.0 * wl.T * k * wl.d * wl.F
    del g
    return {"T": wl.T, "k": k, "ms": ms, "us_per_layer": ms * 1e3,
            "tokens_per_s": wl.T / (ms * 1e-3), "active_experts": active,
            "regime": {1: "gemv", 2: "tcgen05"}.get(L.regime, "?"),
            "bytes": nbytes, "flops": flops,
            "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
            "tensor_frac": flops / (ms * 1e-3) / 1e12 / pk["bf16_tflops"]}


def time_e2e_pipelined(moe, layer, ex, k, ws, x_host, y_host, steps, warmup):
    """Per-step time (ms) of a serving loop through the public call: every
    step copies its own input x from pinned host memory, runs the whole-layer
    forward and copies its result y back to pinned host memory. Two device
    buffer sets and three streams (host->device, compute, device->host) let
    step i+1's input and step i-1's result cross PCIe while step i computes;
    each copy waits only for what it needs (its buffer free, its forward
    done). CUDA events on the copy streams bracket the K timed steps, from
    the first input copy to the last result copy; the L2 is not flushed (the
    weights, 0.9 GB on the prefill workload, exceed it)."""
    wl = layer.wl
    dev = layer.x.device
    xs = [torch.empty_like(layer.x) for _ in range(2)]
    ys = [torch.empty(wl.T, wl.d, dtype=layer.x.dtype, device=dev) for _ in range(2)]
    comp = torch.cuda.current_stream()
    h2d, d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    graphs = []
    for b in range(2):
        moe.forward(xs[b], layer.w_router, layer.router_bias, ex, k, ws=ws, out=ys[b])
        gb = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gb):
            moe.forward(xs[b], layer.w_router, layer.router_bias, ex, k, ws=ws, out=ys[b])
        graphs.append(gb)
    torch.cuda.synchronize()
    in_done = [torch.cuda.Event() for _ in range(2)]
    fwd_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def step(i):
        b = i % 2
        if i >= 2:
            h2d.wait_event(fwd_done[b])        # step i-2's forward has read xs[b]
        with torch.cuda.stream(h2d):
            xs[b].copy_(x_host, non_blocking=True)
        in_done[b].record(h2d)
        comp.wait_event(in_done[b])
        if i >= 2:
            comp.wait_event(out_done[b])       # step i-2's result has left ys[b]
        graphs[b].replay()
        fwd_done[b].record(comp)
        d2h.wait_event(fwd_done[b])
        with torch.cuda.stream(d2h):
            y_host.copy_(ys[b], non_blocking=True)
        out_done[b].record(d2h)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(h2d)
    for i in range(steps):
        step(i)
    t1.record(d2h)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    del graphs
    return ms


def run_ours(args, rank, world, local_rank):
    import sparse_mixture_experts_top_b200 as moe
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    pk, pk_kind = peaks()
    wl = mi.WORKLOADS[args.workload]
    layer = mi.make_layer(wl, seed=args.seed + 1000 * rank, device=dev)
    ex = layer.experts
    k, T = wl.k, wl.T
    ws = moe.forward_workspace(layer.x, ex, k)
    y = torch.empty(T, wl.d, dtype=layer.x.dtype, device=dev)
    flush = (torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev),
             torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev))
    L = moe.forward_layout(T, wl.d, wl.E, k, wl.F, layer.x.dtype, wl.wfmt)

    def fwd():
        moe.forward(layer.x, layer.w_router, layer.router_bias, ex, k, ws=ws, out=y)

    fwd()
    torch.cuda.synchronize()
    # CUDA graph of one forward
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fwd()
    torch.cuda.synchronize()

    if world > 1:
        torch.distributed.barrier()
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    ms = time_device(g.replay, args.steps, args.warmup, flush)
    clocks = sampler.stop()
    ms_eager = time_device(fwd, args.steps, 1, flush)
    if world > 1:
        torch.distributed.barrier()

    # dominant kernel: the gate|up (SwiGLU) stage, timed alone through its C call
    st = moe.SortTables(*(
        ws[off:off + n * 4].view(dt) for off, n, dt in (
            (L.order, T * k, torch.uint32), (L.inv_order, T * k, torch.uint32),
            (L.row_map, T * k, torch.uint32), (L.counts, wl.E, torch.int32),
            (L.row_off, wl.E + 1, torch.int32), (L.tile_off, wl.E + 1, torch.int32))), L.BM)
    h = ws[L.h:L.h + T * k * wl.F * 2].view(torch.float16).view(T * k, wl.F)
    x16 = ws[L.x16:L.total]
    regime = L.regime
    exs = moe.experts_struct(ex)

    def swiglu():
        moe.lib.moe_grouped_swiglu(
            moe._ptr(layer.x), moe._dt(layer.x), moe._ptr(st.row_map), moe._ptr(st.row_off),
            moe._ptr(st.tile_off), L.BM, T, k, __import__("ctypes").byref(exs),
            moe._ptr(h), moe._ptr(x16), x16.numel(), regime, moe._stream())

    fwd()
    ms_swiglu = time_device(swiglu, args.steps, args.warmup, flush)
    counts = st.counts.cpu().numpy()
    active = int((counts > 0).sum())
    gu_bytes = active * gate_up_bytes(ex) + T * wl.d * 2 + T * k * wl.F * 2
    sw_s = statistics.mean(ms_swiglu) * 1e-3
    achieved_gbs = gu_bytes / sw_s / 1e9
    gu_flops = 2.0 * T * k * wl.d * 2 * wl.F
    tflops = gu_flops / sw_s / 1e12

    # end-to-end through the C ABI with host buffers: pinned x -> device,
    # forward, y -> pinned host, every step inside the timed region; serially
    # (one step after another), and as a serving loop that overlaps the copies
    # of neighbouring steps with the forward
    x_host = layer.x.cpu().pin_memory()
    y_host = torch.empty(T, wl.d, dtype=layer.x.dtype).pin_memory()

    def e2e():
        layer.x.copy_(x_host, non_blocking=True)
        g.replay()
        y_host.copy_(y, non_blocking=True)

    ms_e2e_serial = time_device(e2e, args.steps, args.warmup, flush)
    ms_e2e = time_e2e_pipelined(moe, layer, ex, k, ws, x_host, y_host, args.steps, args.warmup)

    # the other workloads, each as one graph-replayed forward timed the same
    # way: decode at T = 1 and T = 32, the acceptance shape (sparse top-2 and
    # dense soft routing, k = E) and the large skewed layer
    extra = {}
    names = [] if args.no_decode else ["decode_t1", "decode_t32"]
    if not args.no_dense:
        names.append("acceptance")
    if not args.no_skewed:
        names.append("skewed")
    for name in names:
        other = mi.make_layer(name, seed=args.seed + 1000 * rank, device=dev)
        ks = [other.wl.k] + ([other.wl.E] if name == "acceptance" else [])
        for kk in ks:
            key = name if kk == other.wl.k else name + "_dense"
            extra[key] = time_layer(moe, other, kk, max(args.steps, 20), args.warmup, flush, pk)
        del other
        torch.cuda.empty_cache()
    decode = {n: extra[n] for n in ("decode_t1", "decode_t32") if n in extra}
    dense = {}
    if "acceptance" in extra:
        wlA = mi.WORKLOADS["acceptance"]
        sp, dn = extra["acceptance"]["ms"], extra["acceptance_dense"]["ms"]
        dense = {"workload": f"acceptance: T={wlA.T} d={wlA.d} E={wlA.E} F={wlA.F} bf16 experts",
                 "sparse_k": wlA.k, "sparse_ms": sp, "dense_ms": dn, "speedup": dn / sp,
                 "target": 1.5}

    step_ms = statistics.mean(ms)
    res = {"ms": step_ms, "ms_eager": statistics.mean(ms_eager), "ms_e2e": ms_e2e,
           "ms_e2e_serial": statistics.mean(ms_e2e_serial),
           "ms_swiglu": statistics.mean(ms_swiglu), "achieved_gbs": achieved_gbs,
           "tflops_swiglu": tflops, "gu_bytes": gu_bytes, "clocks": clocks, "decode": decode, "sparse_vs_dense": dense,
           "acceptance": extra.get("acceptance"), "skewed": extra.get("skewed"),
           "active": active, "regime": regime, "BM": L.BM, "pk": pk, "pk_kind": pk_kind,
           "layer_bytes": active * expert_bytes(ex) + 2 * T * wl.d * 2,
           "layer_flops": 6.0 * T * k * wl.d * wl.F}
    return res, layer


def cpu_baseline(layer, budget_s=12.0):
    """The oracle as it stands, on this host's cores, on a bounded sample of
    the workload's tokens (the layer is token-independent, so tokens/s of a
    sample is the workload's rate)."""
    import oracle
    wl = layer.wl
    x = layer.x.cpu()
    wr = layer.w_router.cpu()
    b = None if layer.router_bias is None else layer.router_bias.cpu()
    ex = layer.experts.to("cpu")
    nth = oracle.default_threads()
    n = min(4, wl.T)
    total_t, total_tok = 0.0, 0
    while True:
        lo = total_tok % wl.T
        xs = x[lo: lo + n]
        t0 = time.perf_counter()
        oracle.forward(xs, wr, b, ex, wl.k, nthreads=nth)
        dt = time.perf_counter() - t0
        total_t += dt
        total_tok += xs.shape[0]
        if total_t >= budget_s or total_tok >= wl.T:
            break
        rate = xs.shape[0] / max(dt, 1e-3)
        n = int(max(1, min(wl.T - total_tok, rate * (budget_s - total_t))))
    return {"value": total_tok / total_t, "unit": "tokens/s", "cores": nth, "kind": "oracle",
            "sample": f"{total_tok} of {wl.T} tokens of the {wl.name} workload (whole layer per "
                      f"token, fp64, {nth} threads), {total_t:.1f} s"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="prefill", choices=sorted(mi.WORKLOADS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-skewed", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    wl = mi.WORKLOADS[args.workload]
    metric = "MoE-layer tokens/s"
    config = {"workload": f"{wl.name}: T={wl.T} d={wl.d} E={wl.E} top-{wl.k} F={wl.F} "
                          f"{wl.wfmt} experts, {wl.act} activations"
                          + (f", router bias {wl.bias}" if wl.bias != "none" else ""),
              "T": wl.T, "d": wl.d, "E": wl.E, "k": wl.k, "F": wl.F, "weights": wl.wfmt,
              "l2": "flushed before every timed step, outside the events: 256 MB written, then "
                    "256 MB read so the write-back finishes before the step"}

    if args.impl == "reference":
        if rank != 0:
            return
        layer = mi.make_layer(wl, seed=args.seed, device="cpu")
        cb = cpu_baseline(layer, budget_s=min(60.0, max(5.0, 1.0 * args.steps)))
        # ms_per_step: one step of the whole workload at the sample's rate
        line = {"impl": "reference", "metric": metric, "value": cb["value"], "unit": "tokens/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": wl.T / cb["value"] * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic", "config": config,
                "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if world > 1:
        torch.distributed.init_process_group(
            "nccl", timeout=__import__("datetime").timedelta(seconds=120),
            device_id=torch.device("cuda", local_rank))
    res, layer = run_ours(args, rank, world, local_rank)
    ms = res["ms"]
    ms_e2e = res["ms_e2e"]
    if world > 1:
        ms, ms_e2e = max_over_ranks([ms, ms_e2e], torch.device("cuda", local_rank))
    if rank == 0:
        pk = res["pk"]
        sw_s = res["ms_swiglu"] * 1e-3
        line = {
            "metric": metric, "value": replicas_tokens_per_s(world, wl.T, ms), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; shapes and distributions of the workload)",
            "config": dict(config, parallelism=f"replicas x{world}" if world > 1 else "single GPU",
                           regime={1: "gemv", 2: "tcgen05"}.get(res["regime"], "?"), BM=res["BM"],
                           active_experts=res["active"], cuda_graph=True),
            "roofline": {"kernel": "grouped gate|up + SwiGLU (moe_grouped_swiglu)",
                         "bound": "hbm", "achieved": res["achieved_gbs"],
                         "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": res["achieved_gbs"] / pk["hbm_gbs"],
                         "traffic": GATE_UP_TRAFFIC.get(args.workload),
                         "peak_source": res["pk_kind"],
                         "us_per_launch": res["ms_swiglu"] * 1e3,
                         "tensor_tflops": res["tflops_swiglu"],
                         "tensor_frac": res["tflops_swiglu"] / pk["bf16_tflops"]},
            "layer_roofline": {
                "bytes": res["layer_bytes"], "flops": res["layer_flops"],
                "hbm_frac": res["layer_bytes"] / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                "tensor_frac": res["layer_flops"] / (ms * 1e-3) / 1e12 / pk["bf16_tflops"]},
            "ms_per_step_eager": res["ms_eager"],
            "e2e": {"value": replicas_tokens_per_s(world, wl.T, ms_e2e), "unit": "tokens/s",
                    "h2d_bytes_per_step": wl.T * wl.d * 2, "d2h_bytes_per_step": wl.T * wl.d * 2,
                    "ms_per_step": ms_e2e,
                    "how": "serving loop: each step copies its x in from pinned host memory and "
                           "its y out to pinned host memory; copies of neighbouring steps overlap "
                           "the forward (two buffer sets, separate copy streams)",
                    "serial": {"value": replicas_tokens_per_s(world, wl.T, res["ms_e2e_serial"]),
                               "ms_per_step": res["ms_e2e_serial"],
                               "how": "copy in, forward, copy out, one step after another, L2 "
                                      "flushed before each step"}},
            "gpu_launches": kernels_per_forward(wl.T, wl.k, res["regime"] == 2) * args.steps,
            "clocks": res["clocks"],
            "decode": res["decode"],
            "acceptance": res["acceptance"],
            "skewed": res["skewed"],
            "sparse_vs_dense": res["sparse_vs_dense"],
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(layer)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
