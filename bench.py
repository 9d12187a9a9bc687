"""Benchmark: MoE-layer forward tokens/s on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill|decode|mid|skew|tiny]
                    [--impl ours|reference]

A step is one pass of the whole hot path over one batch of T tokens: router
(scores, biased top-6, joint gates, counts) -> dispatch -> routed experts
(tcgen05 grouped GEMMs) beside the shared experts (second stream) -> combine
-> bias update.  Inputs are seeded synthetic tensors of the workload's shape,
generated in HBM before timing; every input (x 0.94 GB, weights 15 GB at the
prefill size) is far larger than the 126 MB L2, so no L2 flush is needed.

With N > 1 (torchrun, one process per GPU) each rank runs the layer on its own
T tokens (data-parallel replicas of the same weights: weak scaling); the load
counts are summed over ranks with one NCCL all-reduce (256 int32) before the
bias update, so every replica keeps the same bias.

The default (prefill) run also measures the decode-scale layer (T 64, d 7168,
weight-streaming bound) after the prefill steps, on its own clock, and reports
it under "decode" in the same line (--no-decode skips it).

--impl reference times the CPU oracle (fp64, the layer's plain definition) on
the host cores on a bounded sample of the same workload; rank 0 only.
"""
from __future__ import annotations

import argparse
import copy
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402

METRIC = "MoE-layer fwd tokens/s on 1 B200; % BF16 tensor peak (prefill), % HBM BW (decode)"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0

# the decode record of the default run times this many decode steps per prefill step (a decode
# step is ~2 ms, a prefill step ~30 ms)
DECODE_STEPS_PER_STEP = 10

# DRAM bytes (read + write) of one GEMM1 + GEMM2 launch pair, from one single-pass ncu capture of the
# full-size layer with the current kernels (profiles/grouped_gemm_prefill_dram.md: 256 x 512 pair tiles,
# three stages); workloads without a capture of the current kernels report null
TRAFFIC_PER_LAUNCH_PAIR = {"prefill": 18729761792 + 2210518528 + 13690001152 + 7472903168}
# Weight-streaming launches read what their tokens touch, which drifts as the bias moves the loads, so the
# capture gives DRAM bytes over algorithmic bytes at the captured launches (profiles/launches_decode.md),
# applied to the timed launches' algorithmic bytes
TRAFFIC_RATIO = {"decode": 1.0}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "src": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": FALLBACK_BF16_TFLOPS_SUSTAINED, "src": "fallback"}


def config_of(w, world):
    return {"workload": w.name, "description": w.description, "T_per_gpu": w.T, "global_tokens": w.T * world,
            "d": w.d, "d_ff": w.f, "n_routed": w.n_routed, "n_shared": w.n_shared, "top_k": w.k,
            "activation": w.activation, "gate_scale": w.gate_scale, "parallelism": f"dp{world} (replicas, counts all-reduced)" if world > 1
            else "single GPU", "l2": "inputs larger than L2 (no flush)", "seed": w.seed}


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                try:
                    power.append(float(parts[3]))
                except ValueError:
                    pass
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_median": statistics.median(power) if power else None}


# ---------------------------------------------------------------------------
# our arm: the CUDA path through libmoe
# ---------------------------------------------------------------------------
def run_ours(args, w, rank, world, local_rank, want_cpu=False):
    import torch
    import torch.distributed as dist

    import sparse_moe_layer_joint_b200 as moe
    from sparse_moe_layer_joint_b200 import dp

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    t = mi.torch_workload(w, device=dev)
    if rank > 0:  # each replica gets its own tokens: rows rank*T .. of one global x stream
        mi.gpu_normal_bf16(t["x"].data_ptr(), t["x"].numel(), w.seed, mi.STREAM_X, rank * w.T * w.d, w.std_x,
                           stream.cuda_stream)
    layer = moe.MoELayer(moe.LayerShape(w.T, w.d, w.f, w.n_routed, w.n_shared, w.k), device=dev,
                         gather_rows=args.gather_rows, capacity_factor=args.capacity_factor,
                         activation=w.activation, route_scale=w.gate_scale, precision=args.precision,
                         fused_experts=not args.shared_stream)
    if args.precision == "nvfp4":
        layer.set_nvfp4_weights(t["w1"], t["w2"])
        torch.cuda.synchronize()
    bias0 = t["bias"].clone()
    ffn_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]

    def step(i=None, x=None):
        layer.forward(t["x"] if x is None else x, t["w_r"], t["w1"], t["w2"], t["bias"], t["logit_offset"],
                      ffn_events=None if i is None else ffn_ev[i])
        dp.bias_step(layer, t["bias"], w.gamma)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = moe.moe_get_status()
    if st != 0:
        raise RuntimeError(f"device status {st:#x} after warm-up")

    bias_at_start = t["bias"].clone()   # to replay the timed steps afterwards
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    ffn_ms = statistics.mean(a.elapsed_time(b) for a, b in ffn_ev)
    eager_ms = None
    if args.graph and world == 1:
        # the whole step (its 7-9 launches) captured once as a CUDA graph and replayed: for the
        # latency-bound sizes the host's launch cost, not the GPU, sets the eager step time
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        clocks = ClockSampler(local_rank)
        clocks.start()
        time.sleep(0.3)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        clk = clocks.stop()
        eager_ms, ms = ms, g0.elapsed_time(g1) / args.steps
        del graph

    # replay the timed steps (routing is deterministic) to learn which experts each
    # step touched: the expert GEMMs read only those experts' weights
    t["bias"].copy_(bias_at_start)
    local_counts = torch.empty((args.steps, w.n_routed), dtype=torch.int32, device=dev)
    served = []
    for i in range(args.steps):
        layer.forward(t["x"], t["w_r"], t["w1"], t["w2"], t["bias"], t["logit_offset"])
        local_counts[i].copy_(layer.counts)
        if layer.capacity is not None:
            served.append(w.T * w.k - layer.balance()["dropped"])
        dp.bias_step(layer, t["bias"], w.gamma)
    touched = (local_counts > 0).sum(dim=1).double().mean().item()
    routed_rows = statistics.mean(served) if served else w.T * w.k   # rows the expert GEMMs compute
    if args.log_balance and rank == 0:
        write_balance_log(args.log_balance, local_counts.cpu().numpy(), w.T, w.k, layer.capacity)

    # end to end through the public API: every step copies its x in from pinned host memory and
    # its output back to pinned host memory.  Like a serving loop, the copies of neighbouring steps
    # overlap the current step: x and out are double-buffered on the device, the H2D copies run on
    # one stream and the D2H copies on another, with events so that no buffer is overwritten
    # before it has been consumed.
    x_host = t["x"].cpu().pin_memory()
    out_host = [torch.empty((w.T, w.d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(t["x"]) for _ in range(2)]
    out_dev = [torch.empty_like(layer.out) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("x_ready", "x_free", "out_ready", "out_free")}
    for b in range(2):
        ev["x_free"][b].record(stream)
        ev["out_free"][b].record(stream)

    def e2e_step(i):
        b = i % 2
        s_in.wait_event(ev["x_free"][b])
        with torch.cuda.stream(s_in):
            x_dev[b].copy_(x_host, non_blocking=True)
        ev["x_ready"][b].record(s_in)
        stream.wait_event(ev["x_ready"][b])
        stream.wait_event(ev["out_free"][b])
        layer.forward(x_dev[b], t["w_r"], t["w1"], t["w2"], t["bias"], t["logit_offset"], out=out_dev[b])
        dp.bias_step(layer, t["bias"], w.gamma)
        ev["x_free"][b].record(stream)
        ev["out_ready"][b].record(stream)
        s_out.wait_event(ev["out_ready"][b])
        with torch.cuda.stream(s_out):
            out_host[b].copy_(out_dev[b], non_blocking=True)
        ev["out_free"][b].record(s_out)

    for i in range(2):
        e2e_step(i)
    barrier()
    torch.cuda.synchronize()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    s_in.wait_stream(stream)
    for i in range(args.steps):
        e2e_step(i)
    stream.wait_stream(s_out)   # the last output is on the host before the clock stops
    e3.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e2.elapsed_time(e3) / args.steps
    st = moe.moe_get_status()
    if st != 0:
        raise RuntimeError(f"device status {st:#x} after timing")

    vals = torch.tensor([ms, e2e_ms, ffn_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(vals, op=dist.ReduceOp.MAX)
    ms, e2e_ms, ffn_ms = vals.tolist()

    # the dominant kernels: the experts' grouped GEMMs (both launches of one
    # moe_experts_ffn call).  Algorithmic work per step: FLOPs = 2 GEMMs x 2 * rows * d * d_ff
    # over the T*k routed and T*n_shared shared (token, expert) rows; bytes = weights of the
    # touched routed experts and the shared experts + A rows read + hidden written and read
    # + outputs written (bf16)
    pk = peaks()
    if args.precision == "nvfp4":
        line = nvfp4_line(args, w, world, layer, ms, e2e_ms, ffn_ms, clk, touched, routed_rows, pk)
        if want_cpu:
            line["cpu_baseline"] = cpu_baseline_nvfp4(w)
        return line
    # the timed launch pair: all experts (routed and shared tiles in the same launches), or with
    # --shared-stream the routed experts' pair alone (the shared experts' pair runs on the other stream)
    n_sh = 0 if args.shared_stream else w.n_shared
    rows = routed_rows + w.T * n_sh
    mats = 3 if w.activation == "swiglu" else 2   # weight matrices per expert
    ffn_flops = 2 * mats * rows * w.d * w.f
    ffn_bytes = ((touched + n_sh) * mats * w.d * w.f * 2
                 + rows * w.d * 2 + rows * w.f * 2 * 2 + rows * w.d * 2)
    tflops = ffn_flops / (ffn_ms * 1e-3) / 1e12
    gbs = ffn_bytes / (ffn_ms * 1e-3) / 1e9
    kernel = (f"grouped_gemm_kernel x2 ({'routed experts' if args.shared_stream else 'all experts'}: "
              f"GEMM1+{'SwiGLU' if w.activation == 'swiglu' else 'GELU'}, GEMM2)")
    traffic = None
    if args.capacity_factor is None and not args.gather_rows and not args.shared_stream:
        if w.name in TRAFFIC_PER_LAUNCH_PAIR:
            traffic = TRAFFIC_PER_LAUNCH_PAIR[w.name]
        elif w.name in TRAFFIC_RATIO:
            traffic = round(TRAFFIC_RATIO[w.name] * ffn_bytes)
    # the expert launches are timed inside a step of tens of ms, not a seconds-long loop: the burst peak
    tensor_roof = {"kernel": kernel, "bound": "tensor", "achieved": round(tflops, 1),
                   "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                   "frac": round(tflops / pk["bf16_tflops"], 4),
                   "frac_of_sustained": round(tflops / pk["bf16_tflops_sustained"], 4),
                   "peak_source": f"{pk['src']} bf16 burst (MEASURED_PEAKS.json)" if pk["src"] == "measured"
                   else "fallback bf16 burst (1.59 PFLOP/s)", "traffic": traffic, "traffic_unit": "bytes per launch pair",
                   "algorithmic_bytes_per_launch_pair": round(ffn_bytes),
                   "flop_per_launch_pair": ffn_flops, "ms_per_launch_pair": round(ffn_ms, 4)}
    hbm_roof = {"kernel": kernel, "bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(gbs / pk["hbm_gbs"], 4),
                "peak_source": f"{pk['src']} HBM copy (MEASURED_PEAKS.json)" if pk["src"] == "measured"
                else "fallback HBM copy (6.65 TB/s)", "traffic": traffic,
                "bytes_per_launch_pair": round(ffn_bytes), "touched_routed_experts_mean": round(touched, 2),
                "ms_per_launch_pair": round(ffn_ms, 4)}
    weight_bound = w.name in ("decode", "mid", "inkling_decode")
    roofline = hbm_roof if weight_bound else tensor_roof
    layer_flops = w.flops() - 2.0 * mats * (w.T * w.k - routed_rows) * w.d * w.f
    roofline["layer_tflops"] = round(layer_flops / (ms * 1e-3) / 1e12, 1)
    line = {
        "metric": METRIC, "value": round(world * w.T / (ms * 1e-3), 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded Philox, random-init weights)",
        "config": dict(config_of(w, world), dispatch="rows gathered by GEMM1 (TMA gather4)" if args.gather_rows
                       else "rows copied by moe_permute",
                       shared_experts="own launches on a second stream" if args.shared_stream
                       else "tiles of the routed experts' launches",
                       **({"cuda_graph": True, "ms_per_step_without_graph": round(eager_ms, 4)}
                          if eager_ms is not None else {}),
                       **({"capacity_factor": args.capacity_factor, "capacity": layer.capacity,
                           "served_routed_rows_mean": round(routed_rows, 1)} if layer.capacity is not None else {})),
        "clocks": clk,
        "e2e": {"value": round(world * w.T / (e2e_ms * 1e-3), 1), "unit": UNIT,
                "h2d_bytes_per_step": w.T * w.d * 2, "d2h_bytes_per_step": w.T * w.d * 2,
                "ms_per_step": round(e2e_ms, 4),
                "note": "pinned host x in and out every step; copies of neighbouring steps overlap compute"},
        "gpu_launches": layer.launches_per_step() * args.steps,
        "roofline": roofline,
        "roofline_other": tensor_roof if weight_bound else hbm_roof,
    }
    del bias0
    if want_cpu:
        line["cpu_baseline"] = cpu_baseline(w, t)
    return line


def nvfp4_line(args, w, world, layer, ms, e2e_ms, ffn_ms, clk, touched, routed_rows, pk):
    """Bench line of the layer with NVFP4 routed experts; the roofline kernel is the pair of
    FP4 grouped GEMMs (routed rows only: the shared experts run in bf16 outside the window)."""
    rows = routed_rows
    mats = 3 if w.activation == "swiglu" else 2               # d x d_ff matrices per expert
    ffn_flops = 2 * mats * rows * w.d * w.f
    fp4_matrix = w.d * w.f // 2 + w.d * w.f // 16            # codes + block scales of one matrix
    ffn_bytes = (touched * mats * fp4_matrix                  # the touched routed experts' weights
                 + rows * (w.d // 2 + w.d // 16)              # A codes and scales
                 + 2 * rows * (w.f // 2 + w.f // 16)          # hidden codes and scales, written and read
                 + rows * w.d * 2)                            # y rows (bf16)
    tflops = ffn_flops / (ffn_ms * 1e-3) / 1e12
    gbs = ffn_bytes / (ffn_ms * 1e-3) / 1e9
    fp4_peak = 4.0 * pk["bf16_tflops_sustained"]              # nominal dense FP4 / BF16 = 9 / 2.25
    act = "SwiGLU" if w.activation == "swiglu" else "GELU"
    kernel = f"fp4_gemm_kernel x2 (routed experts: GEMM1+{act}+FP4 requantization, GEMM2)"
    tensor_roof = {"kernel": kernel, "bound": "tensor", "achieved": round(tflops, 1), "peak": round(fp4_peak, 1),
                   "unit": "TFLOP/s", "frac": round(tflops / fp4_peak, 4),
                   "peak_source": "measured bf16 sustained x 4 (nominal dense FP4/BF16 ratio)", "traffic": None,
                   "flop_per_launch_pair": ffn_flops, "ms_per_launch_pair": round(ffn_ms, 4)}
    hbm_roof = {"kernel": kernel, "bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(gbs / pk["hbm_gbs"], 4), "peak_source": f"{pk['src']} HBM copy (MEASURED_PEAKS.json)",
                "traffic": None, "bytes_per_launch_pair": round(ffn_bytes),
                "touched_routed_experts_mean": round(touched, 2), "ms_per_launch_pair": round(ffn_ms, 4)}
    weight_bound = w.T * w.k < 16 * w.n_routed
    roofline = hbm_roof if weight_bound else tensor_roof
    return {
        "metric": METRIC, "value": round(world * w.T / (ms * 1e-3), 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e2m1, e4m3 block-16 scales, fp32 acc) routed "
                                                      "experts; bf16 router and shared experts",
        "data": "synthetic (seeded Philox, random-init weights)",
        "config": dict(config_of(w, world), precision="nvfp4 routed experts (W4A4)"), "clocks": clk,
        "e2e": {"value": round(world * w.T / (e2e_ms * 1e-3), 1), "unit": UNIT,
                "h2d_bytes_per_step": w.T * w.d * 2, "d2h_bytes_per_step": w.T * w.d * 2,
                "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": layer.launches_per_step() * args.steps,
        "roofline": roofline, "roofline_other": tensor_roof if weight_bound else hbm_roof,
    }


# ---------------------------------------------------------------------------
# the Router Balance Lab loop ("Inkling, Dissected" §02g): routing only
# ---------------------------------------------------------------------------
LAB_METRIC = "Router Balance Lab routing step tokens/s on 1 B200 (router + capped dispatch + load stats + bias update)"


def run_lab(args):
    import torch

    import sparse_moe_layer_joint_b200 as moe

    w = mi.LAB
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    cap = moe.capacity_for(w.capacity_factor, w.T, w.k, w.n_routed)
    x_host = torch.from_numpy(mi.lab_x_all(w).view(np.int16)).view(torch.bfloat16)   # [steps, T, d]
    xs = x_host.to(dev)
    wr = torch.from_numpy(mi.lab_wr(w).view(np.int16)).view(torch.bfloat16).to(dev)
    b = torch.zeros(w.n_routed, dtype=torch.float32, device=dev)
    idx = torch.empty((w.T, w.k), dtype=torch.int32, device=dev)
    g = torch.empty((w.T, w.k), dtype=torch.float32, device=dev)
    c = torch.empty(w.n_routed, dtype=torch.int32, device=dev)
    off = torch.empty(w.n_routed + 1, dtype=torch.int32, device=dev)
    rt = torch.empty(w.T * w.k, dtype=torch.int32, device=dev)
    tr = torch.empty((w.T, w.k), dtype=torch.int32, device=dev)
    nb = moe.moe_permute_scratch_bytes(w.T, w.n_routed)
    scratch = torch.empty(nb, dtype=torch.uint8, device=dev)
    n_steps = w.steps
    stats = torch.empty((n_steps, 2), dtype=torch.int32, device=dev)

    def step(i, x=None):
        j = i % n_steps
        moe.moe_router_topk(xs[j] if x is None else x, wr, b, None, w.T, w.d, w.n_routed, 0, w.k, 1.0, idx, g, c)
        moe.moe_permute_capped(None, idx, c, w.T, w.d, w.n_routed, w.k, cap, off, None, rt, tr, scratch, nb)
        moe.moe_load_stats(c, w.n_routed, w.T, w.k, cap, stats[j])
        moe.moe_bias_update(c, w.n_routed, w.T, w.k, args.gamma, b)

    # the balance of one full run from b = 0 (the lab's 100 steps), outside the timing
    for i in range(n_steps):
        step(i)
    torch.cuda.synchronize()
    st = stats.cpu().numpy().astype(np.float64)
    kT = w.k * w.T
    if args.log_balance:
        with open(args.log_balance, "w") as fh:
            for i in range(n_steps):
                fh.write(json.dumps({"step": i, "max_load": int(st[i, 0]),
                                     "max_vio": round(float(st[i, 0] * w.n_routed / kT - 1), 6),
                                     "capacity": cap, "dropped": int(st[i, 1]),
                                     "drop_rate": round(float(st[i, 1] / kT), 8)}) + "\n")
    late = slice(n_steps // 2, None)
    balance = {"gamma": args.gamma, "capacity": cap,
               "max_vio_late_mean": round(float((st[late, 0] * w.n_routed / kT - 1).mean()), 4),
               "drop_rate_late_mean": round(float((st[late, 1] / kT).mean()), 5),
               "max_vio_first_step": round(float(st[0, 0] * w.n_routed / kT - 1), 4)}
    b.zero_()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    eager_ms = None
    if args.graph:
        # the lab's 100 steps (600 launches) captured once and replayed as one CUDA graph
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(n_steps):
                step(i)
        graph.replay()
        torch.cuda.synchronize()
        reps = max(1, args.steps // n_steps)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(reps):
            graph.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        eager_ms, ms = ms, g0.elapsed_time(g1) / (reps * n_steps)
        del graph
    # end to end: each step copies its tokens in from pinned host memory and reads its two load
    # statistics back (the step's result a caller would log)
    x_pin = x_host.pin_memory()
    x_dev = torch.empty((w.T, w.d), dtype=torch.bfloat16, device=dev)
    st_host = torch.empty((2,), dtype=torch.int32).pin_memory()
    torch.cuda.synchronize()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for i in range(args.steps):
        x_dev.copy_(x_pin[i % n_steps], non_blocking=True)
        step(i, x_dev)
        st_host.copy_(stats[i % n_steps], non_blocking=True)
    e3.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e2.elapsed_time(e3) / args.steps
    if moe.moe_get_status() != 0:
        raise RuntimeError("device status after the lab run")
    # algorithmic bytes of one step: x and W_r read, top-k/gates written, top-k read twice by the
    # dispatch, its indices written (everything else is a few KB)
    step_bytes = (w.T * w.d * 2 + w.n_routed * w.d * 2 + w.T * w.k * (4 + 4) + 2 * w.T * w.k * 4
                  + w.T * w.k * 4 * 2)
    pk = peaks()
    gbs = step_bytes / (ms * 1e-3) / 1e9
    return {
        "metric": LAB_METRIC, "value": round(w.T / (ms * 1e-3), 1), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Philox: Zipf-lumpy jittered tokens, frozen random router)",
        "config": dict(lab_config(), **({"cuda_graph": True, "ms_per_step_without_graph": round(eager_ms, 5)}
                                        if eager_ms is not None else {})),
        "clocks": clk,
        "e2e": {"value": round(w.T / (e2e_ms * 1e-3), 1), "unit": UNIT, "h2d_bytes_per_step": w.T * w.d * 2,
                "d2h_bytes_per_step": 8, "ms_per_step": round(e2e_ms, 5)},
        "gpu_launches": 6 * args.steps,
        "roofline": {"kernel": "whole routing step (6 launches)", "bound": "hbm", "achieved": round(gbs, 2),
                     "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 6), "traffic": None,
                     "note": "a 2048-token step moves ~0.4 MB: launch latency, not bandwidth, bounds it"},
        "balance": balance,
    }


def write_balance_log(path, counts, T, k, capacity):
    """One JSON line per step: the largest load, MaxVio (largest load over the ideal k*T/E, minus one)
    and, with a capacity, the assignments dropped and their share of the k*T slots."""
    with open(path, "w") as fh:
        for step, L in enumerate(np.asarray(counts, dtype=np.int64)):
            rec = {"step": step, "max_load": int(L.max()), "max_vio": round(float(L.max() * len(L) / (k * T) - 1), 6),
                   "mean_load": round(float(L.mean()), 3)}
            if capacity is not None:
                dropped = int(np.maximum(L - capacity, 0).sum())
                rec.update(capacity=int(capacity), dropped=dropped, drop_rate=round(dropped / (k * T), 8))
            fh.write(json.dumps(rec) + "\n")


def lab_config():
    w = mi.LAB
    return {"workload": "lab", "description": w.description, "T": w.T, "d": w.d, "n_routed": w.n_routed,
            "top_k": w.k, "capacity_factor": w.capacity_factor, "steps_per_run": w.steps,
            "l2": "not flushed: the whole lab (13 MB of tokens) is L2-resident; latency-bound"}


def lab_cpu(args, steps):
    import oracle

    w = mi.LAB
    t0 = time.perf_counter()
    r = oracle.lab_run(w, args.gamma, steps=steps)
    dt = time.perf_counter() - t0
    return dt, r


# ---------------------------------------------------------------------------
# the CPU oracle on a bounded sample
# ---------------------------------------------------------------------------
def oracle_sample(w, n_tokens, seed_offset=0):
    """Prepare a bounded sample: n_tokens tokens of the workload and the host
    weights of every expert they use (generated before any timing)."""
    import oracle

    tokens = (np.arange(n_tokens) * 7919 + seed_offset) % w.T
    b = mi.host_bias(w)
    off = mi.host_logit_offset(w)
    r = oracle.route_workload(w, b, tokens, off)
    experts = sorted(set(int(e) for e in np.unique(r["contrib"])))
    weights = {"w1": {e: mi.host_w1(w, e) for e in experts}, "w2": {e: mi.host_w2(w, e) for e in experts}}
    return tokens, b, off, weights


def oracle_forward_timed(w, tokens, b, off, weights):
    import oracle

    t0 = time.perf_counter()
    oracle.forward_tokens(w, tokens, b, off, weights=weights)
    return time.perf_counter() - t0


def cpu_baseline(w, t=None, n_sample=32):
    """The oracle as it stands, on the host cores, priced for the whole batch: the fp64 routing
    (logits over 258 experts, biased top-k, joint gates) of every token of the batch, then the whole
    layer (routing, the 8 expert MLPs of each token, combine) on a seeded sample of tokens.  Tokens
    are independent, so the sample's time per token plus the routing time per token prices the
    batch.  ``t``: the workload's device tensors; the sample's expert weights are copied from them
    before timing (the device and host generators give the same bits), which avoids regenerating
    hundreds of weight matrices on the host."""
    import oracle

    b = mi.host_bias(w)
    off = mi.host_logit_offset(w)
    x_all = None
    if t is not None:
        import torch

        x_all = t["x"].view(torch.int16).cpu().numpy().view(np.uint16)
    t0 = time.perf_counter()
    oracle.route_workload(w, b, logit_offset=off, x=x_all)
    t_route = time.perf_counter() - t0
    n_sample = min(n_sample, w.T)
    tokens = (np.arange(n_sample) * 7919) % w.T
    r = oracle.route_workload(w, b, tokens, off)
    experts = sorted(set(int(e) for e in np.unique(r["contrib"])))
    if t is not None:
        import torch

        def bits(a):
            return a.view(torch.int16).cpu().numpy().view(np.uint16)
        weights = {"w1": {e: bits(t["w1"][e]) for e in experts}, "w2": {e: bits(t["w2"][e]) for e in experts}}
    else:
        weights = {"w1": {e: mi.host_w1(w, e) for e in experts}, "w2": {e: mi.host_w2(w, e) for e in experts}}
    t_layer = oracle_forward_timed(w, tokens, b, off, weights)
    per_token = t_route / w.T + t_layer / n_sample
    return {"value": round(1.0 / per_token, 4), "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"routing of all {w.T} tokens of the {w.name} workload (fp64 logits over 258 experts, top-{w.k}, "
                      f"joint gates; {t_route:.2f} s on all cores) + the whole layer on a {n_sample}-token sample "
                      f"(routing, 8 expert MLPs per token, combine; {t_layer:.2f} s, one thread per row of an "
                      f"expert's group); value = 1 / (route s / {w.T} + layer s / {n_sample}); expert weights "
                      "prepared before timing"}


def cpu_baseline_nvfp4(w, n_tokens=2):
    """The NVFP4 oracle (routed experts on FP4 operands, fp64 sums) on a bounded sample; the
    touched experts' weights are generated and quantized before timing."""
    from oracle import nvfp4

    tokens = (np.arange(n_tokens) * 7919) % w.T
    b = mi.host_bias(w)
    cache = {}
    nvfp4.forward_tokens(w, tokens, b, cache=cache)       # fills the cache (untimed)
    t0 = time.perf_counter()
    nvfp4.forward_tokens(w, tokens, b, cache=cache)
    dt = time.perf_counter() - t0
    return {"value": round(len(tokens) / dt, 4), "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{len(tokens)} tokens of the {w.name} workload through the NVFP4 oracle (FP4 activation "
                      f"quantization, fp64 sums over dequantized operands), wall {dt:.2f} s; weights quantized "
                      "before timing"}


def run_reference(args, w):
    """The oracle on the host cores, one token a step (a bounded sample of the same workload): the fp64
    layer, or with --precision nvfp4 the NVFP4 oracle (expert weights quantized before timing)."""
    if args.precision == "nvfp4":
        from oracle import nvfp4

        tokens = (np.arange(2) * 7919) % w.T
        b = mi.host_bias(w)
        cache = {}
        nvfp4.forward_tokens(w, tokens, b, cache=cache)  # quantizes the touched experts (untimed)

        def one(tok):
            t0 = time.perf_counter()
            nvfp4.forward_tokens(w, tok, b, cache=cache)
            return time.perf_counter() - t0
        what = "the NVFP4 oracle (FP4 activation quantization, fp64 sums over dequantized operands)"
    else:
        tokens, b, off, weights = oracle_sample(w, 2)

        def one(tok):
            return oracle_forward_timed(w, tok, b, off, weights)
        what = "the fp64 oracle (router + 8 expert MLPs + combine)"
    per_step = 1
    for i in range(args.warmup):
        one(tokens[i % len(tokens):i % len(tokens) + per_step])
    total = 0.0
    for i in range(args.steps):
        j = i % len(tokens)
        total += one(tokens[j:j + per_step])
    ms = total / args.steps * 1e3
    v = round(per_step / (ms * 1e-3), 4)
    config = dict(config_of(w, 1), dispatch="rows gathered by GEMM1 (TMA gather4)" if args.gather_rows
                  else "rows copied by moe_permute")
    if args.precision == "nvfp4":
        config["precision"] = "nvfp4 routed experts (W4A4)"
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded Philox, random-init weights)",
        "config": config,
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
                         "sample": f"each step: {per_step} token of the {w.name} workload through {what}, "
                                   "weights generated before timing"},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_kernel_case(args):
    """The grouped expert GEMMs alone, on a prefill-shaped slice small enough to
    profile (32 experts x 1536 rows, d 7168, d_ff 2048: 3.5 GB on the device,
    inputs larger than L2).  Prints one diagnostic JSON line (not a bench line)."""
    import torch

    import sparse_moe_layer_joint_b200 as moe

    G, per, d, f = 32, 1536, 7168, 2048
    if args.kernel_case == "nvfp4_decode":
        G, per = 64, 2  # decode-shaped: a couple of rows per expert, the weights streamed once
    n = G * per
    dev = torch.device("cuda", 0)
    s = torch.cuda.current_stream(dev).cuda_stream
    if args.kernel_case != "router":
        rows = torch.empty((n, d), dtype=torch.bfloat16, device=dev)
        w1 = torch.empty((G, f, d), dtype=torch.bfloat16, device=dev)
        w2 = torch.empty((G, d, f), dtype=torch.bfloat16, device=dev)
        mi.gpu_normal_bf16(rows.data_ptr(), rows.numel(), 0, mi.STREAM_TEST_ROWS, 0, 1.0, s)
        mi.gpu_normal_bf16(w1.data_ptr(), w1.numel(), 0, mi.STREAM_W1, 0, d ** -0.5, s)
        mi.gpu_normal_bf16(w2.data_ptr(), w2.numel(), 0, mi.STREAM_W2, 0, f ** -0.5, s)
        offsets = torch.arange(0, n + 1, per, dtype=torch.int32, device=dev)
        h = torch.empty((n, f), dtype=torch.bfloat16, device=dev)
        y = torch.empty((n, d), dtype=torch.bfloat16, device=dev)

    if args.kernel_case == "router":
        # the router alone on the chosen workload's tokens (diagnostic / profiling case)
        w = mi.WORKLOADS[args.workload]
        t = mi.torch_workload(w, with_weights=False)
        layer = moe.MoELayer(moe.LayerShape(w.T, w.d, w.f, w.n_routed, w.n_shared, w.k))

        def call():
            moe.moe_router_topk(t["x"], t["w_r"], t["bias"], t["logit_offset"], w.T, w.d, w.n_routed, w.n_shared,
                                w.k, 1.0, layer.topk_idx, layer.gates, layer.counts)
    elif args.kernel_case == "grouped_ffn":
        def call():
            moe.moe_grouped_ffn(rows, offsets, G, n, 0, w1, w2, d, f, moe.MOE_ACT_GELU_TANH, h, y)
    elif args.kernel_case in ("nvfp4_ffn", "nvfp4_decode"):
        # the same slice with NVFP4 operands: rows quantized once by the FP4 dispatch (one expert
        # per row, groups of 1536 = 12 x 128 rows, so no padding), then GEMM1 + GELU + FP4 and GEMM2
        u8 = torch.uint8
        w1q = torch.empty((G, f, d // 2), dtype=u8, device=dev)
        w1sf = torch.empty((G, f * d // 16), dtype=u8, device=dev)
        g1 = torch.empty(G, dtype=torch.float32, device=dev)
        w2q = torch.empty((G, d, f // 2), dtype=u8, device=dev)
        w2sf = torch.empty((G, d * f // 16), dtype=u8, device=dev)
        g2 = torch.empty(G, dtype=torch.float32, device=dev)
        moe.moe_nvfp4_quantize_weights(w1, G, f, d, w1q, w1sf, g1)
        moe.moe_nvfp4_quantize_weights(w2, G, d, f, w2q, w2sf, g2)
        rows_cap = moe.moe_nvfp4_rows_capacity(n, G, 1)
        xq = torch.empty((rows_cap, d // 2), dtype=u8, device=dev)
        xsf = torch.empty((rows_cap * d // 16,), dtype=u8, device=dev)
        hq = torch.empty((rows_cap, f // 2), dtype=u8, device=dev)
        hsf = torch.empty((rows_cap * f // 16,), dtype=u8, device=dev)
        topk = (torch.arange(n, device=dev, dtype=torch.int32) // per).reshape(n, 1)
        trow = torch.arange(n, device=dev, dtype=torch.int32).reshape(n, 1)
        trp = torch.empty_like(trow)
        offp = torch.empty(G + 1, dtype=torch.int32, device=dev)
        moe.moe_nvfp4_dispatch(rows, topk, trow, offsets, n, d, G, 1, xq, xsf, trp, offp)

        real = offsets if args.kernel_case == "nvfp4_decode" else None  # load only the real A rows

        def call():
            moe.moe_nvfp4_grouped_gemm(xq, xsf, offp, G, rows_cap, w1q, w1sf, g1, f, d, moe.MOE_NVFP4_EPI_GELU_FP4,
                                       hq, hsf, None, real, n if real is not None else 0)
            moe.moe_nvfp4_grouped_gemm(hq, hsf, offp, G, rows_cap, w2q, w2sf, g2, d, f, moe.MOE_NVFP4_EPI_BF16,
                                       None, None, y, offsets, n)
    else:
        # comparison only (not the product path): the same two GEMMs per expert through cuBLAS
        xr, hr, yr = rows.view(G, per, d), h.view(G, per, f), y.view(G, per, d)

        def call():
            torch.bmm(xr, w1.transpose(1, 2), out=hr)
            torch.bmm(hr, w2.transpose(1, 2), out=yr)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    h0 = time.perf_counter()
    for _ in range(args.steps):
        call()
    host_us = (time.perf_counter() - h0) / args.steps * 1e6
    e1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    if args.kernel_case == "router":
        print(json.dumps({"kernel_case": "router", "workload": args.workload, "us_per_call": round(ms * 1e3, 2),
                          "host_us_per_call": round(host_us, 2),
                          "clocks": clk, "status": moe.moe_get_status()}), flush=True)
        return
    flops = 2 * 2.0 * n * d * f
    wbytes = G * 2 * d * f * (0.5 + 1 / 16 if args.kernel_case.startswith("nvfp4") else 2)
    print(json.dumps({"kernel_case": args.kernel_case, "experts": G, "rows_per_expert": per, "d": d, "d_ff": f,
                      "ms_per_call": round(ms, 4), "tflops": round(flops / (ms * 1e-3) / 1e12, 1),
                      "weight_gbs": round(wbytes / (ms * 1e-3) / 1e9, 1),
                      "clocks": clk, "status": moe.moe_get_status()}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="prefill", choices=sorted(mi.WORKLOADS) + ["lab"])
    ap.add_argument("--capacity-factor", type=float, default=None,
                    help="hard expert capacity, as a multiple of the ideal load k*T/n_routed (overflow dropped)")
    ap.add_argument("--gamma", type=float, default=0.01, help="bias step of the lab workload")
    ap.add_argument("--log-balance", default=None, metavar="PATH",
                    help="write one JSON line per step (largest load, MaxVio, drops) to PATH")
    ap.add_argument("--graph", action="store_true",
                    help="time the step as one replayed CUDA graph (one GPU; for the launch-bound sizes)")
    ap.add_argument("--precision", choices=["bf16", "nvfp4"], default="bf16",
                    help="nvfp4: the routed experts in NVFP4 (W4A4); router and shared experts stay bf16")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="prefill workload: skip the decode-scale record measured in the same run")
    ap.add_argument("--shared-stream", action="store_true",
                    help="shared experts as their own GEMM launches on a second stream (beside the router and "
                         "dispatch) instead of tiles of the routed experts' launches")
    ap.add_argument("--decode-first", action="store_true",
                    help="prefill workload: measure the decode-scale record before the prefill steps")
    ap.add_argument("--gather-rows", action="store_true",
                    help="GEMM1 gathers the routed rows from x (TMA tile::gather4) instead of reading rows copied "
                         "by dispatch")
    ap.add_argument("--kernel-case", choices=["grouped_ffn", "grouped_ffn_cublas", "nvfp4_ffn", "nvfp4_decode",
                                              "router"],
                    default=None,
                    help="time one kernel alone on a small profiling case instead of the layer")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.workload == "lab":
        if rank == 0:
            if args.impl == "reference":
                k = max(1, min(args.steps, 20))
                dt, _ = lab_cpu(args, k)
                v = round(mi.LAB.T * k / dt, 1)
                print(json.dumps({
                    "impl": "reference", "metric": LAB_METRIC, "value": v, "unit": UNIT, "n_gpus": 1,
                    "steps": k, "warmup": 0, "ms_per_step": round(dt / k * 1e3, 3), "higher_is_better": True,
                    "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                    "data": "synthetic (seeded Philox: Zipf-lumpy jittered tokens, frozen random router)",
                    "config": lab_config(),
                    "cpu_baseline": {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
                                     "sample": f"{k} lab steps through the fp64 oracle"},
                    "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}), flush=True)
            else:
                if world > 1:
                    raise SystemExit("the lab workload runs on one GPU")
                line = run_lab(args)
                if not args.no_cpu_baseline:
                    dt, _ = lab_cpu(args, 20)
                    line["cpu_baseline"] = {"value": round(mi.LAB.T * 20 / dt, 1), "unit": UNIT, "cores": 1,
                                            "kind": "oracle", "sample": f"20 lab steps through the fp64 oracle, "
                                                                         f"wall {dt:.2f} s"}
                print(json.dumps(line), flush=True)
        return
    w = mi.WORKLOADS[args.workload]

    if args.kernel_case is not None:
        run_kernel_case(args)
        return

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w)), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        want_decode = (args.workload == "prefill" and not args.no_decode and args.precision == "bf16"
                       and not args.graph and args.capacity_factor is None and not args.gather_rows)

        def decode_record():
            # the decode-scale layer (T 64, d 7168), weight-streaming bound, measured in the same run
            # on its own clock: each step reads the touched experts' weights from HBM
            dargs = copy.copy(args)
            dargs.steps = args.steps * DECODE_STEPS_PER_STEP
            dargs.log_balance = None
            dargs.graph = world == 1  # a 2 ms step of 7 launches: replayed as one CUDA graph
            dec = run_ours(dargs, mi.WORKLOADS["decode"], rank, world, local_rank)
            return {k: dec[k] for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                                        "config", "clocks", "e2e", "gpu_launches", "roofline")}

        dec = decode_record() if want_decode and args.decode_first else None
        line = run_ours(args, w, rank, world, local_rank,
                        want_cpu=rank == 0 and world == 1 and not args.no_cpu_baseline)
        if want_decode:
            line["decode"] = dec if dec is not None else decode_record()
            line["decode"]["measured"] = "before the prefill steps" if args.decode_first else "after the prefill steps"
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
