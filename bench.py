#!/usr/bin/env python
"""Benchmark of the MoE + multi-LoRA layer on B200: tokens/s of the whole hot path.

One step = one pass of the whole path over one batch resident in HBM:
  moe_lora_route   router logits x W_r^T, softmax top-k + renormalised weights,
                   stable (expert, adapter) sort into segments (one launch at decode)
  moe_lora_forward gather + gate_up LoRA shrink, tcgen05 gate_up GEMM running the LoRA
                   expand as extra MMA K steps and SiLU-and-mul in its epilogue, down
                   LoRA shrink, tcgen05 down GEMM with the expand and the routing weight,
                   fixed-order combine

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--M M]
    python bench.py --impl reference ...      (the fp64 CPU oracle, same metric)

Default workload: MoE decode, bf16 experts, E=64, top-8, H=2048, I=1408, 8 adapters
of rank 16 on gate_up and down, M=64 tokens per step.  For N > 1 (torchrun) every
rank runs an independent replica (weak scaling, no collective on the data path);
timing is the max over ranks.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import synth  # noqa: E402

METRIC = "MoE+multi-LoRA layer tokens/s; achieved HBM GB/s or TC util vs B200 peak"
DEFAULT_WORKLOAD = synth.MOE_DECODE_BF16.name
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024

# ncu-measured DRAM traffic (read + write bytes per launch) of the gate_up GEMM on the
# default workload, with the hash of the kernel source it was taken on; reported as
# null when the source has changed since.  Filled from profiles/.
NCU_TRAFFIC = {"gemm_tc.cu": "6ca23e0dc6e3bec3", "bytes_per_launch": 746.644224e6 + 5.415680e6,
               "workload": synth.MOE_DECODE_BF16.name, "M": 64}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--M", type=int, default=64)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--batches", type=int, default=4, help="distinct token batches cycled over the steps")
    ap.add_argument("--e2e-steps", type=int, default=0, help="0: same as --steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the base-only and same-adapter variants of the MoE step")
    ap.add_argument("--no-graph", action="store_true",
                    help="time plain API calls instead of replaying a CUDA graph of them")
    return ap.parse_args()


# ----------------------------------------------------------------------------- helpers

def dist_setup():
    """One process per GPU from torchrun's environment: NCCL on GPUs; gloo on a host
    without CUDA (the reference arm, and the multi-rank tests on CPU)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """The slowest rank's time: every multi-GPU number is the max over ranks."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def step_percentiles(run_step, n_steps: int) -> dict:
    """Device time of each of up to 200 further steps, run after the timed region (not part
    of `value`): median and 10th / 90th percentiles in ms."""
    try:
        n = max(1, min(n_steps, 200))
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
        evs[0].record()
        for i in range(n):
            run_step(i)
            evs[i + 1].record()
        torch.cuda.synchronize()
        d = sorted(evs[i].elapsed_time(evs[i + 1]) for i in range(n))
        q = lambda f: d[min(n - 1, int(round(f * (n - 1))))]  # noqa: E731
        return {"p10_ms": q(0.1), "p50_ms": q(0.5), "p90_ms": q(0.9), "steps": n}
    except Exception as e:  # a side measurement never costs the line
        return {"error": f"{type(e).__name__}: {str(e)[:120]}"}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms while running."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.uuid = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            pass
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [[c.strip() for c in ln.split(",")] for ln in out.strip().splitlines() if ln.count(",") >= 8]
        if self.uuid:
            mine = [r for r in rows if self.uuid.replace("GPU-", "") in r[0]]
            rows = mine or rows
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(sm)}


def src_hash(name: str) -> str:
    with open(os.path.join(ROOT, "moe_lora_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def routing_stats(rt: dict, shape: synth.MoEShape):
    """Touched experts and (adapter, expert) pairs of one routed batch (host side)."""
    so = rt["seg_offsets"].cpu().numpy().astype(np.int64)
    cnt = np.diff(so).reshape(shape.E, shape.L + 1)
    experts = int(np.count_nonzero(cnt.sum(1)))
    pairs = int(np.count_nonzero(cnt[:, : shape.L]))
    return experts, pairs


def expand_in_gemm(shape, M) -> bool:
    """The library's placement rule for the LoRA expand (inside the GEMM above 64 rows
    per expert, else the LoRA kernel's fp32 delta)."""
    return M * shape.k > 64 * shape.E


def gateup_alg_bytes(shape, M, experts, pairs):
    """Bytes the gate_up GEMM must move once: touched expert gate_up weights, the
    gathered x rows (bf16, or two e4m3 planes and their scales), its LoRA input (the
    fp32 delta, or the z rows and touched B_gu slices when it runs the expand), and the
    act it writes."""
    wb = 1 if shape.wdtype == "e4m3" else 2
    mk = M * shape.k
    xb = mk * (2 * shape.H + 8) if shape.wdtype == "e4m3" else mk * shape.H * 2
    if shape.L == 0:
        lora = 0
    elif expand_in_gemm(shape, M):
        lora = mk * shape.r * 2 + pairs * shape.r * 2 * shape.I * 2
    else:
        lora = mk * 2 * shape.I * 4
    return experts * 2 * shape.I * shape.H * wb + xb + lora + mk * shape.I * 2


def gateup_alg_flops(shape, M):
    """gate_up base GEMM plus its fused LoRA expand."""
    mk = M * shape.k
    return 2 * mk * 2 * shape.I * shape.H + 2 * mk * shape.r * 2 * shape.I


def layer_alg_bytes(shape, M, experts, pairs):
    """Bytes the whole layer must move once (intermediates excluded): touched expert
    weights, touched adapter slices, router weight, x, adapter ids and y."""
    wb = 1 if shape.wdtype == "e4m3" else 2
    per_expert = (2 * shape.I * shape.H + shape.H * shape.I) * wb
    per_pair = shape.r * (shape.H + 2 * shape.I + shape.I + shape.H) * 2
    return (experts * per_expert + pairs * per_pair + shape.E * shape.H * 2
            + M * shape.H * 2 * 2 + M * 4)


def layer_flops(shape, M):
    mk = M * shape.k
    return (2 * mk * (shape.H * 2 * shape.I + shape.I * shape.H)
            + 2 * mk * shape.r * (2 * shape.H + 3 * shape.I) + 2 * M * shape.H * shape.E)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- oracle timing

def oracle_tokens_per_s(shape, M, cpu_weights, seconds: float, max_calls: int | None = None,
                        tokens_per_call: int | None = None):
    """The fp64 oracle (route from x, sort, forward) on batch 0, repeated until `seconds`
    of CPU time have passed (or `max_calls`); returns (tokens/s, calls, tokens/call)."""
    from oracle import formats
    from oracle import moe_lora_ref as ref
    from tests.gpu_cases import CpuWeightsOracle
    OW = CpuWeightsOracle(shape, cpu_weights)
    x, ad = synth.moe_tokens(shape, M)
    x64 = formats.to_f64(synth.bits(x), "bf16")
    ad64 = ad.numpy().astype(np.int64)
    wr, bias = OW.router()
    n = M if tokens_per_call is None else max(1, min(M, tokens_per_call))
    sel = np.arange(n)
    # weights of the experts this batch touches are decoded once, like a model load
    lg = ref.router_logits(x64, wr, bias)
    ids, _ = ref.route_topk(lg, shape.k)
    for e in np.unique(ids[sel]):
        OW.expert(int(e))
    calls, t0 = 0, time.perf_counter()
    while True:
        lg = ref.router_logits(x64[sel], wr, bias)
        ids, w = ref.route_topk(lg, shape.k)
        ref.sort_pairs(ids, ad64[sel], shape.E, shape.L)
        ref.moe_lora_forward(x64[sel], ids, w, ad64[sel], shape.I, OW.expert, OW.adapter)
        calls += 1
        el = time.perf_counter() - t0
        if el >= seconds or (max_calls is not None and calls >= max_calls):
            break
    return n * calls / el, calls, n, el


def reference_arm(args, world, rank):
    """--impl reference: the oracle on the host cores, same metric/unit/config."""
    if rank != 0:
        return
    shape = synth.WORKLOADS[args.workload]
    if not isinstance(shape, synth.MoEShape):
        dense_oracle_tokens_per_s(shape, seconds=0.0, max_calls=max(1, args.warmup))
        tps, calls, n, el = dense_oracle_tokens_per_s(shape, seconds=1e9, max_calls=args.steps)
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": tps, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / calls, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": shape.name, "T": shape.T, "h_in": shape.h_in, "h_out": shape.h_out,
                       "L": shape.L, "r": shape.r},
            "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": f"{n} tokens per step, {calls} steps, {el:.1f} s"},
            "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
        return
    M = args.M
    cpu = synth.moe_weights(shape, device="cpu")
    # size one step so that warmup + steps take about two minutes of CPU time
    tps, _, _, _ = oracle_tokens_per_s(shape, M, cpu, seconds=2.0, max_calls=1, tokens_per_call=1)
    per_tok = 1.0 / tps
    budget = 120.0
    tok = int(max(1, min(M, budget / max(1, args.steps + args.warmup) / per_tok)))
    oracle_tokens_per_s(shape, M, cpu, seconds=0.0, max_calls=max(1, args.warmup), tokens_per_call=tok)
    tps, calls, n, el = oracle_tokens_per_s(shape, M, cpu, seconds=1e9, max_calls=args.steps, tokens_per_call=tok)
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": tps, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / calls, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": shape.name, "M": M, "E": shape.E, "k": shape.k, "H": shape.H, "I": shape.I,
                   "L": shape.L, "r": shape.r, "wdtype": shape.wdtype},
        "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{n} token(s) of batch 0 per step, {calls} steps, {el:.1f} s"},
        "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


# ----------------------------------------------------------------------------- dense SGMV arm

def dense_oracle_tokens_per_s(shape: synth.DenseShape, seconds: float, max_calls: int | None = None):
    """The fp64 oracle of one dense multi-LoRA projection on the bench's token batch,
    repeated until `seconds` of CPU time (or `max_calls`); weights decoded once, like a
    model load.  Returns (tokens/s, calls, tokens/call, elapsed s)."""
    from oracle import formats
    from oracle import moe_lora_ref as ref
    x, _, offs, segs = synth.dense_tokens(shape)
    w = synth.dense_weights(shape)
    f = lambda t: formats.to_f64(synth.bits(t), shape.dtype)  # noqa: E731
    x64, w64, a64, b64 = f(x), f(w["w"]), f(w["a"]), f(w["b"])
    so, sa = offs.numpy(), segs.numpy()
    calls, t0 = 0, time.perf_counter()
    while True:
        ref.dense_lora_forward(x64, w64, a64, b64, so, sa)
        calls += 1
        el = time.perf_counter() - t0
        if el >= seconds or (max_calls is not None and calls >= max_calls):
            break
    return shape.T * calls / el, calls, shape.T, el


def run_dense(args, shape: synth.DenseShape, world, rank, local):
    """One dense projection with segmented multi-LoRA (dense_lora_forward).  Its weight
    fits in L2, so the steps cycle over enough copies of the weights and adapters that
    the copy a step reads was evicted by the steps before it (inputs larger than L2)."""
    import moe_lora_b200 as ml
    dev = torch.device("cuda", local)
    T = shape.T
    x, tok_a, offs, segs = synth.dense_tokens(shape)
    w0 = synth.dense_weights(shape, device=dev)
    x, offs, segs = x.to(dev), offs.to(dev), segs.to(dev)
    eb = 2 if shape.dtype == "bf16" else 4
    copy_bytes = sum(t.numel() for t in w0.values()) * eb
    n_copies = int(min(512, -(-3 * L2_BYTES // copy_bytes) + 1))
    copies = [w0] + [{kk: v.clone() for kk, v in w0.items()} for _ in range(n_copies - 1)]
    ws = ml.new_workspace(ml.workspace_size(ml.OP_DENSE, T, shape.h_in, shape.h_out, 1, 1, shape.L, shape.r), dev)
    y = torch.empty((T, shape.h_out), dtype=x.dtype, device=dev)

    def step(i, xin=x):
        w = copies[i % n_copies]
        ml.dense_lora_forward(xin, w["w"], w["a"], w["b"], offs, segs, y=y, workspace=ws)

    for i in range(max(args.warmup, n_copies)):
        step(i)
    torch.cuda.synchronize()
    ml.check_status(ws)

    n0 = ml.launch_count()
    for i in range(args.steps):
        step(i)
    torch.cuda.synchronize()
    launches = ml.launch_count() - n0

    # ---- per-kernel device times: one step per weight copy captured as a CUDA graph
    #      with event nodes around every launch, replayed; the last replay is read
    if not args.no_graph:
        gs = torch.cuda.Stream()
        gs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(gs):
            step(0)
        torch.cuda.current_stream().wait_stream(gs)
        torch.cuda.synchronize()
        ml.profile_enable(n_copies * 4 + 16)
        pgraphs = []
        for c in range(n_copies):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(c)
            pgraphs.append(g)
        for _ in range(3):
            for g in pgraphs:
                g.replay()
        torch.cuda.synchronize()
        prof_steps = n_copies
    else:
        ml.profile_enable(args.steps * 4 + 16)
        for i in range(args.steps):
            step(i)
        torch.cuda.synchronize()
        prof_steps = args.steps
    gemm_ms, gemm_n = ml.profile_read("gemm_dense" if shape.dtype == "bf16" else "dense_f32")
    per_kernel = {k: ml.profile_read(k)[0] / prof_steps for k in ("lora", "shrink", "gemm_dense", "dense_f32")}
    ml.profile_enable(0)
    if not args.no_graph:
        del pgraphs

    # ---- one CUDA graph per weight copy
    graphs = []
    if not args.no_graph:
        for c in range(n_copies):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(c)
            graphs.append(g)
        for i in range(max(args.warmup, n_copies)):
            graphs[i % n_copies].replay()
        torch.cuda.synchronize()

    def run_step(i):
        if graphs:
            graphs[i % n_copies].replay()
        else:
            step(i)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.25)
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for i in range(args.steps):
        run_step(i)
    ev1.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms_max = max_over_ranks(ev0.elapsed_time(ev1), world)
    value = world * T * args.steps / (ms_max / 1e3)
    per_step = step_percentiles(run_step, args.steps)

    # ---- e2e: pinned host x -> device, dense_lora_forward, y -> pinned host, every step
    e2e_steps = args.e2e_steps or args.steps
    hx = x.cpu().pin_memory()
    hy = torch.empty((T, shape.h_out), dtype=x.dtype).pin_memory()
    dx = torch.empty_like(x)

    def e2e_step(i):
        dx.copy_(hx, non_blocking=True)
        step(i, dx)
        hy.copy_(y, non_blocking=True)

    e2e_graphs = []
    if not args.no_graph:
        for c in range(n_copies):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                e2e_step(c)
            e2e_graphs.append(g)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(e2e_steps):
        if e2e_graphs:
            e2e_graphs[i % n_copies].replay()
        else:
            e2e_step(i)
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    del graphs, e2e_graphs
    ml.check_status(ws)

    adapters = sorted(set(int(v) for v in tok_a.tolist() if v >= 0))
    lay_bytes = (shape.h_out * shape.h_in + len(adapters) * shape.r * (shape.h_in + shape.h_out)) * eb \
        + T * (shape.h_in + shape.h_out) * eb
    gemm_bytes = shape.h_out * shape.h_in * eb + T * shape.h_in * eb + T * shape.h_out * eb
    if shape.dtype == "bf16":  # the fused expand: z rows and the touched B slices
        gemm_bytes += T * shape.r * 2 + len(adapters) * shape.r * shape.h_out * 2
    peaks, peak_src = load_peaks()
    peak = float(peaks["hbm_gbs"])
    g_s = (gemm_ms / max(gemm_n, 1)) / 1e3
    step_s = ms_max / 1e3 / args.steps
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": shape.dtype, "data": "synthetic",
        "config": {"workload": shape.name, "T": T, "h_in": shape.h_in, "h_out": shape.h_out, "L": shape.L,
                   "r": shape.r, "adapters": shape.adapter_dist, "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2: steps cycle over {n_copies} copies of W, A and B "
                         f"({n_copies * copy_bytes / 1e6:.0f} MB)"},
        "roofline": {"bound": "hbm", "kernel": "gemm_tc (dense)" if shape.dtype == "bf16" else "dense_f32",
                     "achieved": gemm_bytes / g_s / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": gemm_bytes / g_s / 1e9 / peak, "peak_source": peak_src, "traffic": None,
                     "alg_bytes_per_launch": gemm_bytes, "avg_launch_us": g_s * 1e6},
        "layer": {"alg_bytes_per_step": lay_bytes, "achieved_GBps": lay_bytes / step_s / 1e9,
                  "frac_of_hbm_peak": lay_bytes / step_s / 1e9 / peak,
                  "kernel_ms_per_step": per_kernel,
                  "kernel_times": "CUDA events around each launch inside the replayed step graphs"
                  if not args.no_graph else "CUDA events around each launch of plain API calls"},
        "e2e": {"value": world * T * e2e_steps / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": T * shape.h_in * eb, "d2h_bytes_per_step": T * shape.h_out * eb,
                "how": "graph replay of H2D copy, dense_lora_forward, D2H copy" if not args.no_graph
                else "plain API calls"},
        "timing": {"mode": "CUDA graph replay of the API call" if not args.no_graph else "plain API calls",
                   "per_step": per_step},
        "gpu_launches": launches, "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps, calls, n, el = dense_oracle_tokens_per_s(shape, args.cpu_seconds)
        line["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"fp64 oracle, {n} tokens per call, {calls} calls in {el:.1f} s; "
                                          "weights decoded to fp64 once before timing"}
    if rank == 0:
        print(json.dumps(line))


# ----------------------------------------------------------------------------- our arm

def main():
    args = parse()
    world, rank, local = dist_setup()
    if args.impl == "reference":
        reference_arm(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    import moe_lora_b200 as ml

    shape = synth.WORKLOADS[args.workload]
    if not isinstance(shape, synth.MoEShape):
        run_dense(args, shape, world, rank, local)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    dev = torch.device("cuda", local)
    M, k, L = args.M, shape.k, shape.L
    cpu = synth.moe_weights(shape, device="cpu")
    W = {kk: (v.to(dev) if isinstance(v, torch.Tensor) else v) for kk, v in cpu.items()}
    batches = []
    for b in range(args.batches):
        x, ad = synth.moe_tokens(shape, M, batch=b)
        batches.append((x.to(dev), ad.to(dev)))
    rws = ml.new_workspace(ml.workspace_size(ml.OP_ROUTE, M, shape.H, 0, shape.E, k, L, 0), dev)
    fop = ml.OP_FORWARD_E4M3 if shape.wdtype == "e4m3" else ml.OP_FORWARD_BF16
    fws = ml.new_workspace(ml.workspace_size(fop, M, shape.H, shape.I, shape.E, k, L, shape.r), dev)
    rbufs = {"topk_ids": torch.empty((M, k), dtype=torch.int32, device=dev),
             "topk_w": torch.empty((M, k), dtype=torch.float32, device=dev),
             "sorted_pairs": torch.empty((M * k,), dtype=torch.int32, device=dev),
             "seg_offsets": torch.empty((shape.E * (L + 1) + 1,), dtype=torch.int32, device=dev)}
    y = torch.empty((M, shape.H), dtype=torch.bfloat16, device=dev)

    def step(i):
        xb, ab = batches[i % len(batches)]
        rt = ml.route(ab, k, L, x=xb, w_router=W["w_router"], bias=W["bias"], out=rbufs, workspace=rws)
        ml.forward(xb, rt, W, k=k, L=L, y=y, workspace=fws)
        return rt

    # routing statistics of each batch (outside any timed region)
    stats = []
    for b in range(len(batches)):
        rt = step(b)
        torch.cuda.synchronize()
        stats.append(routing_stats(rt, shape))
    ml.check_status(fws)
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    # ---- plain API calls (host enqueue included), for reference
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = ml.launch_count()
    p0.record()
    for i in range(args.steps):
        step(i)
    p1.record()
    torch.cuda.synchronize()
    launches_per_step = (ml.launch_count() - n0) / args.steps
    plain_ms = p0.elapsed_time(p1)

    # ---- per-kernel device times: each batch's step captured as a CUDA graph with an
    #      event pair around every launch (event nodes), replayed; the last replay of
    #      every graph is read.  Without graphs: plain calls (host gaps included).
    names = ("route", "router_logits", "topk", "sort", "lora", "quant", "gemm_gateup", "gemm_down", "combine")
    if not args.no_graph:
        gs = torch.cuda.Stream()
        gs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(gs):
            for b in range(len(batches)):
                step(b)  # warm the stream before capture
        torch.cuda.current_stream().wait_stream(gs)
        torch.cuda.synchronize()
        ml.profile_enable(len(batches) * 16 + 64)
        pgraphs = []
        for b in range(len(batches)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(b)
            pgraphs.append(g)
        for _ in range(5):
            for g in pgraphs:
                g.replay()
        torch.cuda.synchronize()
        prof_steps = len(batches)
    else:
        ml.profile_enable(args.steps * 16 + 64)
        for i in range(args.steps):
            step(i)
        torch.cuda.synchronize()
        prof_steps = args.steps
    per_kernel = {kname: ml.profile_read(kname) for kname in names}
    ml.profile_enable(0)
    if not args.no_graph:
        del pgraphs
    gu_ms, gu_n = per_kernel["gemm_gateup"]
    launches = int(round(launches_per_step * args.steps))

    # ---- the step as a CUDA graph of the same API calls (one graph per token batch)
    graphs = []
    if not args.no_graph:
        gs = torch.cuda.Stream()
        gs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(gs):
            for b in range(len(batches)):
                step(b)  # warm the stream before capture
        torch.cuda.current_stream().wait_stream(gs)
        torch.cuda.synchronize()
        for b in range(len(batches)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(b)
            graphs.append(g)
        for i in range(args.warmup):
            graphs[i % len(graphs)].replay()
        torch.cuda.synchronize()

    def run_step(i):
        if graphs:
            graphs[i % len(graphs)].replay()
        else:
            step(i)

    # ---- timed region: K steps on device-resident inputs
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.25)
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for i in range(args.steps):
        run_step(i)
    ev1.record()
    torch.cuda.synchronize()
    barrier(world)
    ms = ev0.elapsed_time(ev1)
    clk = clocks.stop()
    ms_max = max_over_ranks(ms, world)
    value = world * M * args.steps / (ms_max / 1e3)
    per_step = step_percentiles(run_step, args.steps)

    # ---- secondary measurements: the same step with every adapter id -1 (base only, the
    #      LoRA work skipped by segment) and with one adapter for every token
    secondary = None
    if not args.no_secondary and not args.no_graph:
        def timed_variant(ids_fn):
            vb = [(xb, ids_fn(ab)) for xb, ab in batches]
            vgraphs = []
            for b, (xb, ab) in enumerate(vb):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    rt = ml.route(ab, k, L, x=xb, w_router=W["w_router"], bias=W["bias"], out=rbufs, workspace=rws)
                    ml.forward(xb, rt, W, k=k, L=L, y=y, workspace=fws)
                vgraphs.append(g)
            n = min(args.steps, 1000)
            for i in range(min(args.warmup, 20)):
                vgraphs[i % len(vgraphs)].replay()
            torch.cuda.synchronize()
            v0, v1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            v0.record()
            for i in range(n):
                vgraphs[i % len(vgraphs)].replay()
            v1.record()
            torch.cuda.synchronize()
            del vgraphs
            return v0.elapsed_time(v1) / n

        t_none = timed_variant(lambda ab: torch.full_like(ab, -1))
        t_same = timed_variant(lambda ab: torch.zeros_like(ab)) if L > 0 else None
        t_main = ms_max / args.steps
        secondary = {
            "lora_overhead_ms_per_step": t_main - t_none, "base_only_ms_per_step": t_none,
            "same_adapter_ms_per_step": t_same, "distinct_adapters_ms_per_step": t_main,
            "adapters": f"{shape.adapter_dist} over L={L}",
            "swap_ab": "not measured: only the swapped (weights in the 128-row MMA M slot) tile exists; "
                       "a non-swapped tile would put <= 64 tokens per expert in M = 128",
        }

    # ---- e2e: pinned host inputs -> device, route + forward, y -> pinned host, every step
    e2e_steps = args.e2e_steps or args.steps
    hx = [b[0].cpu().pin_memory() for b in batches]
    ha = [b[1].cpu().pin_memory() for b in batches]
    hy = torch.empty((M, shape.H), dtype=torch.bfloat16).pin_memory()
    dx = torch.empty_like(batches[0][0])
    da = torch.empty_like(batches[0][1])

    def e2e_step(j):
        dx.copy_(hx[j], non_blocking=True)
        da.copy_(ha[j], non_blocking=True)
        rt = ml.route(da, k, L, x=dx, w_router=W["w_router"], bias=W["bias"], out=rbufs, workspace=rws)
        ml.forward(dx, rt, W, k=k, L=L, y=y, workspace=fws)
        hy.copy_(y, non_blocking=True)

    e2e_graphs = []
    if not args.no_graph:
        for j in range(len(batches)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                e2e_step(j)
            e2e_graphs.append(g)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(e2e_steps):
        j = i % len(batches)
        if e2e_graphs:
            e2e_graphs[j].replay()
        else:
            e2e_step(j)
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = world * M * e2e_steps / (e2e_ms / 1e3)
    del graphs, e2e_graphs
    ml.check_status(fws)
    ml.check_status(rws)

    # ---- roofline of the dominant kernel (gate_up GEMM) and of the whole layer
    peaks, peak_src = load_peaks()
    n_b = len(batches)
    mean = lambda f: float(np.mean([f(*stats[i % n_b]) for i in range(args.steps)]))  # noqa: E731
    gu_bytes = mean(lambda e, p: gateup_alg_bytes(shape, M, e, p))
    lay_bytes = mean(lambda e, p: layer_alg_bytes(shape, M, e, p))
    gu_avg_s = (gu_ms / max(gu_n, 1)) / 1e3
    tensor_bound = M * k >= 128 * shape.E  # >= 128 rows per expert: the MMA, not HBM, bounds gate_up
    if tensor_bound:
        achieved = gateup_alg_flops(shape, M) / gu_avg_s / 1e12
        peak_t = float(peaks["bf16_tflops_sustained"]) * (2.0 if shape.wdtype == "e4m3" else 1.0)
    else:
        achieved = gu_bytes / gu_avg_s / 1e9
    peak = float(peaks["hbm_gbs"])
    traffic = (NCU_TRAFFIC["bytes_per_launch"] if NCU_TRAFFIC["gemm_tc.cu"] == src_hash("gemm_tc.cu")
               and NCU_TRAFFIC["workload"] == shape.name and NCU_TRAFFIC["M"] == M else None)
    step_s = ms_max / 1e3 / args.steps

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if shape.wdtype == "bf16" else "e4m3/bf16",
        "data": "synthetic",
        "config": {"workload": shape.name, "M": M, "tokens_per_step_per_gpu": M, "E": shape.E, "k": k,
                   "H": shape.H, "I": shape.I, "L": L, "r": shape.r, "wdtype": shape.wdtype,
                   "adapters": shape.adapter_dist, "parallelism": f"replicas x{world}",
                   "l2": f"no flush: {lay_bytes / 1e9:.2f} GB of weights per step > 126 MB L2; "
                         f"{n_b} rotating token batches"},
        "roofline": ({"bound": "hbm", "kernel": "gemm_tc (gate_up, tcgen05)", "achieved": achieved, "peak": peak,
                      "unit": "GB/s", "frac": achieved / peak, "peak_source": peak_src,
                      "traffic": traffic, "alg_bytes_per_launch": gu_bytes,
                      "avg_launch_us": gu_avg_s * 1e6} if not tensor_bound else
                     {"bound": "tensor", "kernel": "gemm_tc (gate_up, tcgen05)", "achieved": achieved,
                      "peak": peak_t, "unit": "TFLOP/s", "frac": achieved / peak_t,
                      "peak_source": f"{peak_src} bf16 sustained" + (" x2 (fp8 nominal ratio)"
                                                                    if shape.wdtype == "e4m3" else ""),
                      "traffic": traffic, "alg_flops_per_launch": gateup_alg_flops(shape, M),
                      "alg_bytes_per_launch": gu_bytes, "achieved_GBps": gu_bytes / gu_avg_s / 1e9,
                      "avg_launch_us": gu_avg_s * 1e6}),
        "layer": {"alg_bytes_per_step": lay_bytes, "achieved_GBps": lay_bytes / step_s / 1e9,
                  "frac_of_hbm_peak": lay_bytes / step_s / 1e9 / peak,
                  "TFLOPs": layer_flops(shape, M) / step_s / 1e12,
                  "kernel_ms_per_step": {kk: v[0] / prof_steps for kk, v in per_kernel.items()},
                  "kernel_times": "CUDA events around each launch inside the replayed step graphs"
                  if not args.no_graph else "CUDA events around each launch of plain API calls"},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": M * shape.H * 2 + M * 4,
                "d2h_bytes_per_step": M * shape.H * 2,
                "how": "graph replay of H2D copy, route, forward, D2H copy" if not args.no_graph else "plain API calls"},
        "timing": {"mode": "CUDA graph replay of the route + forward API calls" if not args.no_graph
                   else "plain API calls", "plain_api_ms_per_step": plain_ms / args.steps,
                   "per_step": per_step},
        "gpu_launches": launches,
        "clocks": clk,
    }
    if secondary is not None:
        line["secondary"] = secondary
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps, calls, n, el = oracle_tokens_per_s(shape, M, cpu, seconds=args.cpu_seconds)
        line["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"fp64 oracle on batch 0 ({n} tokens), {calls} calls in {el:.1f} s; "
                                          "touched expert weights decoded to fp64 once before timing"}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
