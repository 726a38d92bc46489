#!/usr/bin/env python
"""Benchmark of the MoE + multi-LoRA layer on B200: tokens/s of the whole hot path.

One step = one pass of the whole path over one batch resident in HBM:
  moe_lora_route   router logits x W_r^T, softmax top-k + renormalised weights,
                   stable (expert, adapter) sort into segments
  moe_lora_forward gather + LoRA shrink, tcgen05 gate_up GEMM (LoRA expand, SiLU-and-mul),
                   down LoRA, tcgen05 down GEMM (LoRA expand, routing weight), fixed-order
                   combine

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--M M]
    python bench.py --impl reference ...      (the fp64 CPU oracle, same metric)

Default workload: the MoE prefill layer, the largest configuration that fits one GPU:
4096 tokens, bf16 experts, E=128, top-8, H=4096, I=1536, 16 adapters of rank 64 on
gate_up and down (Zipf adapter ids, router bias skewing the expert load).  The same line
carries a `sweep` of the decode layers (bf16 E=64 at M = 1, 8, 32, 64; e4m3 experts
E=128 at M = 1, 4, 16, 64, and the same e4m3 layer at 4096 tokens: FP8 prefill) and the
dense decode projection, measured in the same process.  `e2e` is the same step through the
public API with pinned host buffers, run as a serving pipeline (each step's inputs copied in
and its y copied out on two copy streams while the neighbouring step computes, every copy
inside the timed region); `e2e.serial_value` is the same with copies and compute one after
another.  For N > 1 (torchrun) every rank runs an independent replica (weak scaling, no
collective on the data path); timing is the max over ranks.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import platform
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
DEFAULT_WORKLOAD = synth.MOE_PREFILL_BF16.name
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024
# decode layers measured in the same process as the headline line
# (the e4m3-expert layer also at 4096 tokens: FP8 prefill on the same weights)
SWEEP = ((synth.MOE_DECODE_BF16.name, (1, 8, 32, 64)), (synth.MOE_DECODE_FP8.name, (1, 4, 16, 64, 4096)),
         (synth.DENSE_DECODE_BF16.name, (64,)))

# ncu-measured DRAM traffic (read + write bytes per launch) of the gate_up GEMM, with the
# hash of the kernel source it was taken on and the case it was taken on; reported as
# null when the source has changed since or the case differs.  Filled from profiles/.
NCU_TRAFFIC = {"gemm_tc.cu": "2cdc3e920394a8e1", "bytes_per_launch": 3897368832.0 + 106269729.0,
               "workload": "moe_prefill_bf16_e128_h4096_i1536", "M": 4096}


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--M", type=int, default=0, help="tokens per step (0: the workload's largest)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--batches", type=int, default=4, help="distinct token batches cycled over the steps")
    ap.add_argument("--e2e-steps", type=int, default=0, help="0: same as --steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the base-only and same-adapter variants of the MoE step")
    ap.add_argument("--no-sweep", action="store_true", help="skip the decode sweep")
    ap.add_argument("--sweep-seconds", type=float, default=0.25, help="timed device seconds per sweep entry")
    ap.add_argument("--no-graph", action="store_true",
                    help="time plain API calls instead of replaying a CUDA graph of them")
    a = ap.parse_args(argv)
    if a.M <= 0:
        shape = synth.WORKLOADS[a.workload]
        a.M = shape.M_list[-1] if isinstance(shape, synth.MoEShape) else shape.T
    return a


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


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


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


def lora_place(shape, M) -> str:
    """The library's placement of the LoRA work of the grouped GEMMs (MOE_LORA_EXPAND
    overrides): "tc" above 64 rows per expert (the tensor-core LoRA kernel writes bf16
    deltas: gate_up's is added by the GEMM epilogue, down's by the combine), else "delta"
    (the SIMT LoRA kernel's fp32 deltas)."""
    v = os.environ.get("MOE_LORA_EXPAND")
    if v in ("delta", "tc"):
        return v
    return "tc" if M * shape.k > 64 * shape.E else "delta"


def gateup_alg_bytes(shape, M, experts, pairs):
    """Bytes the gate_up GEMM must move once: touched expert gate_up weights, the
    gathered x rows (bf16, or two e4m3 planes and their scales), its LoRA input (the
    fp32 or bf16 delta) and the act it writes."""
    wb = 1 if shape.wdtype == "e4m3" else 2
    mk = M * shape.k
    xb = mk * (2 * shape.H + 8) if shape.wdtype == "e4m3" else mk * shape.H * 2
    if shape.L == 0:
        lora = 0
    elif lora_place(shape, M) == "tc":
        lora = mk * 2 * shape.I * 2
    else:
        lora = mk * 2 * shape.I * 4
    return experts * 2 * shape.I * shape.H * wb + xb + lora + mk * shape.I * 2


def gateup_alg_flops(shape, M):
    """The gate_up base GEMM (its LoRA expand runs in the LoRA kernels)."""
    return 2 * M * shape.k * 2 * shape.I * shape.H


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


def gateup_tensor_bound(shape, M) -> bool:
    """>= 128 rows per expert on average: the MMA, not the weight stream, bounds gate_up."""
    return M * shape.k >= 128 * shape.E


def scaled_kernel_times(event_ms: dict, instrumented_step_ms: float, step_ms: float) -> dict:
    """Per-kernel device time per step, reconciled with the uninstrumented step: each
    kernel's share of the instrumented step (event pairs around every launch inside the
    replayed graphs) applied to the step time measured without events.  The event nodes
    serialise the graph and add a few microseconds each, so the raw event sums exceed the
    plain step; the shares do not depend on that overhead's absolute size."""
    if instrumented_step_ms <= 0:
        return {k: 0.0 for k in event_ms}
    return {k: v / instrumented_step_ms * step_ms for k, v in event_ms.items()}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cores_desc() -> dict:
    return {"cores": blas_threads(), "cpu_model": cpu_model(), "host_cpus": os.cpu_count()}


# ----------------------------------------------------------------------------- oracle timing

class StoredSlices:
    """Expert and adapter slices of one MoE workload at their stored precision (bf16 or
    e4m3 bits), drawn once from the seeded generator before timing; every get widens
    the slice to fp64 anew, so the oracle's timed region runs from the stored weights
    to y, conversion included (generation excluded)."""

    def __init__(self, shape: synth.MoEShape):
        self.s = shape
        self.e, self.a = {}, {}

    def prepare(self, ids: np.ndarray, adapter_ids: np.ndarray):
        import concurrent.futures as cf
        need_e = sorted({int(e) for e in ids.reshape(-1)} - set(self.e))
        need_a = sorted({(int(adapter_ids[t]), int(e)) for t in range(ids.shape[0]) for e in ids[t]
                         if adapter_ids[t] >= 0} - set(self.a))
        with cf.ThreadPoolExecutor(max_workers=max(1, min(16, os.cpu_count() or 1))) as ex:
            for e, v in zip(need_e, ex.map(lambda e: synth.moe_expert(self.s, e), need_e)):
                self.e[e] = (synth.bits(v[0]), synth.bits(v[1]), float(v[2]), float(v[3]))
            for ae, v in zip(need_a, ex.map(lambda ae: synth.moe_adapter(self.s, *ae), need_a)):
                self.a[ae] = tuple(synth.bits(t) for t in v)

    def expert(self, e):
        from oracle import formats
        gu, d, sg, sd = self.e[int(e)]
        return formats.to_f64(gu, self.s.wdtype), formats.to_f64(d, self.s.wdtype), sg, sd

    def adapter(self, a, e):
        from oracle import formats
        return tuple(formats.to_f64(t, "bf16") for t in self.a[(int(a), int(e))])


def oracle_tokens_per_s(shape, M, seconds: float, max_calls: int | None = None,
                        tokens_per_call: int | None = None, slices: StoredSlices | None = None):
    """The fp64 oracle (route from x, sort, forward) on the first tokens of batch 0,
    repeated until `seconds` of CPU time have passed (or `max_calls`); returns
    (tokens/s, calls, tokens/call, elapsed s).  The touched expert and adapter slices are
    drawn at stored precision before timing; their fp64 conversion is timed."""
    from oracle import formats
    from oracle import moe_lora_ref as ref
    x, ad = synth.moe_tokens(shape, M)
    x64 = formats.to_f64(synth.bits(x), "bf16")
    ad64 = ad.numpy().astype(np.int64)
    wr_t, bias_t = synth.moe_router(shape)
    wr = formats.to_f64(synth.bits(wr_t), "bf16")
    bias = None if bias_t is None else bias_t.numpy().astype(np.float64)
    n = M if tokens_per_call is None else max(1, min(M, tokens_per_call))
    sel = np.arange(n)
    sl = slices if slices is not None else StoredSlices(shape)
    ids, _ = ref.route_topk(ref.router_logits(x64[sel], wr, bias), shape.k)
    sl.prepare(ids, ad64[sel])
    calls, t0 = 0, time.perf_counter()
    while True:
        lg = ref.router_logits(x64[sel], wr, bias)
        ids, w = ref.route_topk(lg, shape.k)
        ref.sort_pairs(ids, ad64[sel], shape.E, shape.L)
        ref.moe_lora_forward(x64[sel], ids, w, ad64[sel], shape.I, sl.expert, sl.adapter)
        calls += 1
        el = time.perf_counter() - t0
        if el >= seconds or (max_calls is not None and calls >= max_calls):
            break
    return n * calls / el, calls, n, el


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


def reference_arm(args, world, rank):
    """--impl reference: the oracle on the host cores, same metric/unit/config."""
    if rank != 0:
        return
    shape = synth.WORKLOADS[args.workload]
    base = {"impl": "reference", "metric": METRIC, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic"}
    if not isinstance(shape, synth.MoEShape):
        dense_oracle_tokens_per_s(shape, seconds=0.0, max_calls=max(1, args.warmup))
        tps, calls, n, el = dense_oracle_tokens_per_s(shape, seconds=1e9, max_calls=args.steps)
        print(json.dumps({
            **base, "value": tps, "ms_per_step": 1e3 * el / calls,
            "config": {"workload": shape.name, "T": shape.T, "h_in": shape.h_in, "h_out": shape.h_out,
                       "L": shape.L, "r": shape.r},
            "cpu_baseline": {"value": tps, "unit": "tokens/s", **cores_desc(), "kind": "oracle",
                             "sample": f"{n} tokens per step, {calls} steps, {el:.1f} s"},
            "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
        return
    M = args.M
    sl = StoredSlices(shape)
    # size one step so that warmup + steps take about two minutes of CPU time
    tps, _, _, _ = oracle_tokens_per_s(shape, M, seconds=2.0, max_calls=1, tokens_per_call=1, slices=sl)
    per_tok = 1.0 / tps
    budget = 120.0
    tok = int(max(1, min(M, 64, budget / max(1, args.steps + args.warmup) / per_tok)))
    oracle_tokens_per_s(shape, M, seconds=0.0, max_calls=max(1, args.warmup), tokens_per_call=tok, slices=sl)
    tps, calls, n, el = oracle_tokens_per_s(shape, M, seconds=1e9, max_calls=args.steps, tokens_per_call=tok,
                                            slices=sl)
    line = {
        **base, "value": tps, "ms_per_step": 1e3 * el / calls,
        "config": {"workload": shape.name, "M": M, "E": shape.E, "k": shape.k, "H": shape.H, "I": shape.I,
                   "L": shape.L, "r": shape.r, "wdtype": shape.wdtype},
        "cpu_baseline": {"value": tps, "unit": "tokens/s", **cores_desc(), "kind": "oracle",
                         "sample": f"{n} token(s) of batch 0 per step, {calls} steps, {el:.1f} s"},
        "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


# ----------------------------------------------------------------------------- dense arm

def measure_dense(args, shape: synth.DenseShape, world, local, *, steps, warmup, full):
    """One dense projection with segmented multi-LoRA (dense_lora_forward).  Its weight
    fits in L2, so the steps cycle over enough copies of the weights and adapters that
    the copy a step reads was evicted by the steps before it (inputs larger than L2).
    Returns the measurement fields of a line (full: also e2e, percentiles and clocks)."""
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

    for i in range(max(warmup, n_copies)):
        step(i)
    torch.cuda.synchronize()
    ml.check_status(ws)
    n0 = ml.launch_count()
    for i in range(n_copies):
        step(i)
    torch.cuda.synchronize()
    launches_per_step = (ml.launch_count() - n0) / n_copies

    def capture(fn, profile=0):
        gs = torch.cuda.Stream()
        gs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(gs):
            fn(0)
        torch.cuda.current_stream().wait_stream(gs)
        torch.cuda.synchronize()
        if profile:  # event pairs only around the captured launches, not the warm-up
            ml.profile_enable(profile)
        out = []
        for c in range(n_copies):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn(c)
            out.append(g)
        return out

    # ---- per-kernel device times: event pairs around every launch inside the graphs
    names = ("lora", "shrink", "gemm_dense", "dense_f32")
    if not args.no_graph:
        pgraphs = capture(step, profile=n_copies * 4 + 16)
        for _ in range(3):
            for g in pgraphs:
                g.replay()
        torch.cuda.synchronize()
        per_kernel = {k: ml.profile_read(k) for k in names}
        i0, i1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        i0.record()
        for g in pgraphs:
            g.replay()
        i1.record()
        torch.cuda.synchronize()
        instr_ms = i0.elapsed_time(i1) / n_copies
        ml.profile_enable(0)
        del pgraphs
        prof_steps = n_copies
    else:
        ml.profile_enable(steps * 4 + 16)
        for i in range(steps):
            step(i)
        torch.cuda.synchronize()
        per_kernel = {k: ml.profile_read(k) for k in names}
        ml.profile_enable(0)
        prof_steps, instr_ms = steps, 0.0
    gemm_ms, gemm_n = per_kernel["gemm_dense" if shape.dtype == "bf16" else "dense_f32"]
    event_ms = {k: v[0] / prof_steps for k, v in per_kernel.items()}
    if args.no_graph:
        instr_ms = sum(event_ms.values())

    graphs = capture(step) if not args.no_graph else []
    for i in range(max(warmup, n_copies)):
        graphs[i % n_copies].replay() if graphs else step(i)
    torch.cuda.synchronize()

    def run_step(i):
        if graphs:
            graphs[i % n_copies].replay()
        else:
            step(i)

    clocks = ClockSampler(local) if full else None
    if clocks:
        clocks.start()
        time.sleep(0.25)
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for i in range(steps):
        run_step(i)
    ev1.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop() if clocks else None
    ms_max = max_over_ranks(ev0.elapsed_time(ev1), world)
    step_ms = ms_max / steps

    adapters = sorted(set(int(v) for v in tok_a.tolist() if v >= 0))
    lay_bytes = (shape.h_out * shape.h_in + len(adapters) * shape.r * (shape.h_in + shape.h_out)) * eb \
        + T * (shape.h_in + shape.h_out) * eb
    gemm_bytes = shape.h_out * shape.h_in * eb + T * shape.h_in * eb + T * shape.h_out * eb
    if shape.dtype == "bf16" and T > 64:  # expand inside the GEMM: z rows and the touched B slices
        gemm_bytes += T * shape.r * 2 + len(adapters) * shape.r * shape.h_out * 2
    elif shape.dtype == "bf16":  # fp32 delta of the LoRA kernel
        gemm_bytes += T * shape.h_out * 4
    peaks, peak_src = load_peaks()
    peak = float(peaks["hbm_gbs"])
    g_s = (gemm_ms / max(gemm_n, 1)) / 1e3
    out = {
        "value": world * T / (step_ms / 1e3), "ms_per_step": step_ms, "steps": steps,
        "roofline": {"bound": "hbm", "kernel": "gemm_tc (dense)" if shape.dtype == "bf16" else "dense_f32",
                     "achieved": gemm_bytes / g_s / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": gemm_bytes / g_s / 1e9 / peak, "peak_source": f"{peak_src} HBM copy",
                     "traffic": None, "alg_bytes_per_launch": gemm_bytes, "avg_launch_us": g_s * 1e6},
        "layer": {"alg_bytes_per_step": lay_bytes, "achieved_GBps": lay_bytes / (step_ms / 1e3) / 1e9,
                  "frac_of_hbm_peak": lay_bytes / (step_ms / 1e3) / 1e9 / peak,
                  "kernel_ms_per_step": scaled_kernel_times(event_ms, instr_ms, step_ms),
                  "instrumented_step_ms": instr_ms},
        "gpu_launches": int(round(launches_per_step * steps)),
        "l2": f"inputs larger than L2: steps cycle over {n_copies} copies of W, A and B "
              f"({n_copies * copy_bytes / 1e6:.0f} MB)",
    }
    if full:
        out["clocks"] = clk
        out["timing_per_step"] = step_percentiles(run_step, steps)
        e2e_steps = args.e2e_steps or steps
        hx = x.cpu().pin_memory()
        hy = torch.empty((T, shape.h_out), dtype=x.dtype).pin_memory()
        dx = torch.empty_like(x)

        def e2e_step(i):
            dx.copy_(hx, non_blocking=True)
            step(i, dx)
            hy.copy_(y, non_blocking=True)

        e2e_graphs = capture(e2e_step) if not args.no_graph else []
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(e2e_steps):
            e2e_graphs[i % n_copies].replay() if e2e_graphs else e2e_step(i)
        e1.record()
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
        del e2e_graphs
        out["e2e"] = {"value": world * T * e2e_steps / (e2e_ms / 1e3), "unit": "tokens/s",
                      "h2d_bytes_per_step": T * shape.h_in * eb, "d2h_bytes_per_step": T * shape.h_out * eb,
                      "how": "graph replay of H2D copy, dense_lora_forward, D2H copy" if not args.no_graph
                      else "plain API calls"}
    del graphs
    ml.check_status(ws)
    return out


# ----------------------------------------------------------------------------- MoE arm

def measure_moe(args, shape: synth.MoEShape, M: int, W: dict, world, local, *, steps, warmup, full):
    """Route + forward of one MoE layer at M tokens per step, timed as CUDA-graph replays
    of the two API calls over `args.batches` rotating token batches.  Returns the
    measurement fields of a line (full: also e2e, percentiles, clocks, secondary)."""
    import moe_lora_b200 as ml
    dev = torch.device("cuda", local)
    k, L = shape.k, shape.L
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

    def call(xb, ab):
        rt = ml.route(ab, k, L, x=xb, w_router=W["w_router"], bias=W["bias"], out=rbufs, workspace=rws)
        ml.forward(xb, rt, W, k=k, L=L, y=y, workspace=fws)
        return rt

    def step(i):
        return call(*batches[i % len(batches)])

    stats = []  # routing statistics of each batch (outside any timed region)
    for b in range(len(batches)):
        rt = step(b)
        torch.cuda.synchronize()
        stats.append(routing_stats(rt, shape))
    ml.check_status(fws)
    ml.check_status(rws)
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()

    n0 = ml.launch_count()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_plain = len(batches) if not full else max(len(batches), min(steps, 200))
    p0.record()
    for i in range(n_plain):
        step(i)
    p1.record()
    torch.cuda.synchronize()
    launches_per_step = (ml.launch_count() - n0) / n_plain
    plain_ms = p0.elapsed_time(p1) / n_plain

    def capture(fn, nb, profile=0):
        gs = torch.cuda.Stream()
        gs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(gs):
            for b in range(nb):
                fn(b)  # warm the stream before capture
        torch.cuda.current_stream().wait_stream(gs)
        torch.cuda.synchronize()
        if profile:  # event pairs only around the captured launches, not the warm-up
            ml.profile_enable(profile)
        out = []
        for b in range(nb):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn(b)
            out.append(g)
        return out

    # ---- per-kernel device times: each batch's step captured as a CUDA graph with an
    #      event pair around every launch (event nodes), replayed; the last replay of
    #      every graph is read, and the instrumented replay itself is timed
    names = ("route", "router_logits", "topk", "sort", "gather", "lora", "quant", "gemm_gateup", "lora_down",
             "gemm_down", "combine")
    nb = len(batches)
    if not args.no_graph:
        pgraphs = capture(step, nb, profile=nb * 24 + 64)
        for _ in range(5):
            for g in pgraphs:
                g.replay()
        torch.cuda.synchronize()
        per_kernel = {kname: ml.profile_read(kname) for kname in names}
        i0, i1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        i0.record()
        for g in pgraphs:
            g.replay()
        i1.record()
        torch.cuda.synchronize()
        instr_ms = i0.elapsed_time(i1) / nb
        ml.profile_enable(0)
        del pgraphs
        prof_steps = nb
    else:
        ml.profile_enable(steps * 24 + 64)
        for i in range(steps):
            step(i)
        torch.cuda.synchronize()
        per_kernel = {kname: ml.profile_read(kname) for kname in names}
        ml.profile_enable(0)
        prof_steps, instr_ms = steps, 0.0
    event_ms = {kk: v[0] / prof_steps for kk, v in per_kernel.items()}
    if args.no_graph:
        instr_ms = sum(event_ms.values())
    gu_ms, gu_n = per_kernel["gemm_gateup"]

    # ---- the step as a CUDA graph of the same API calls (one graph per token batch)
    graphs = capture(step, nb) if not args.no_graph else []
    for i in range(warmup):
        graphs[i % nb].replay() if graphs else step(i)
    torch.cuda.synchronize()

    def run_step(i):
        if graphs:
            graphs[i % nb].replay()
        else:
            step(i)

    # ---- timed region: K steps on device-resident inputs
    clocks = ClockSampler(local) if full else None
    if clocks:
        clocks.start()
        time.sleep(0.25)
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for i in range(steps):
        run_step(i)
    ev1.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop() if clocks else None
    ms_max = max_over_ranks(ev0.elapsed_time(ev1), world)
    step_ms = ms_max / steps

    # ---- roofline of the dominant kernel (gate_up GEMM) and of the whole layer
    peaks, peak_src = load_peaks()
    mean = lambda f: float(np.mean([f(*stats[i % nb]) for i in range(steps)]))  # noqa: E731
    gu_bytes = mean(lambda e, p: gateup_alg_bytes(shape, M, e, p))
    lay_bytes = mean(lambda e, p: layer_alg_bytes(shape, M, e, p))
    gu_avg_s = (gu_ms / max(gu_n, 1)) / 1e3
    peak = float(peaks["hbm_gbs"])
    traffic = (NCU_TRAFFIC["bytes_per_launch"] if NCU_TRAFFIC["gemm_tc.cu"] == src_hash("gemm_tc.cu")
               and NCU_TRAFFIC["workload"] == shape.name and NCU_TRAFFIC["M"] == M else None)
    if gateup_tensor_bound(shape, M):
        fp8 = shape.wdtype == "e4m3"
        peak_t = float(peaks["bf16_tflops_sustained"]) * (2.0 if fp8 else 1.0)
        achieved = gateup_alg_flops(shape, M) / gu_avg_s / 1e12
        roof = {"bound": "tensor", "kernel": "gemm_tc (gate_up, tcgen05)", "achieved": achieved, "peak": peak_t,
                "unit": "TFLOP/s", "frac": achieved / peak_t,
                "peak_source": f"{peak_src} bf16 sustained" + (" x2 (fp8 nominal ratio)" if fp8 else ""),
                "traffic": traffic, "alg_flops_per_launch": gateup_alg_flops(shape, M),
                "alg_bytes_per_launch": gu_bytes, "achieved_GBps": gu_bytes / gu_avg_s / 1e9,
                "avg_launch_us": gu_avg_s * 1e6}
    else:
        achieved = gu_bytes / gu_avg_s / 1e9
        roof = {"bound": "hbm", "kernel": "gemm_tc (gate_up, tcgen05)", "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": achieved / peak, "peak_source": f"{peak_src} HBM copy",
                "traffic": traffic, "alg_bytes_per_launch": gu_bytes, "avg_launch_us": gu_avg_s * 1e6}
    out = {
        "value": world * M / (step_ms / 1e3), "ms_per_step": step_ms, "steps": steps,
        "roofline": roof,
        "layer": {"alg_bytes_per_step": lay_bytes, "achieved_GBps": lay_bytes / (step_ms / 1e3) / 1e9,
                  "frac_of_hbm_peak": lay_bytes / (step_ms / 1e3) / 1e9 / peak,
                  "TFLOPs": layer_flops(shape, M) / (step_ms / 1e3) / 1e12,
                  "kernel_ms_per_step": scaled_kernel_times(event_ms, instr_ms, step_ms),
                  "instrumented_step_ms": instr_ms,
                  "touched_experts": float(np.mean([s[0] for s in stats])),
                  "touched_adapter_expert_pairs": float(np.mean([s[1] for s in stats]))},
        "gpu_launches": int(round(launches_per_step * steps)),
        "plain_api_ms_per_step": plain_ms,
        "l2": f"no flush: {lay_bytes / 1e9:.2f} GB of weights per step > 126 MB L2; {nb} rotating token batches",
    }
    if not full:
        del graphs
        return out
    out["clocks"] = clk
    out["timing_per_step"] = step_percentiles(run_step, steps)

    # ---- secondary measurements: the same step with every adapter id -1 (base only, the
    #      LoRA work skipped by segment) and with one adapter for every token
    if not args.no_secondary and not args.no_graph:
        def timed_variant(ids_fn):
            vb = [(xb, ids_fn(ab)) for xb, ab in batches]
            vgraphs = capture(lambda b: call(*vb[b]), nb)
            n = max(10, min(steps, 200))
            for i in range(min(warmup, 20)):
                vgraphs[i % nb].replay()
            torch.cuda.synchronize()
            v0, v1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            v0.record()
            for i in range(n):
                vgraphs[i % nb].replay()
            v1.record()
            torch.cuda.synchronize()
            del vgraphs
            return v0.elapsed_time(v1) / n

        t_none = timed_variant(lambda ab: torch.full_like(ab, -1))
        t_same = timed_variant(lambda ab: torch.zeros_like(ab)) if L > 0 else None
        out["secondary"] = {
            "lora_overhead_ms_per_step": step_ms - t_none, "base_only_ms_per_step": t_none,
            "same_adapter_ms_per_step": t_same, "distinct_adapters_ms_per_step": step_ms,
            "adapters": f"{shape.adapter_dist} over L={L}",
        }
        if M * k >= 256 * shape.E and shape.wdtype == "bf16":
            # the operand swap at prefill tiles: weights in M (one CTA per 128 x 256 tile, and
            # CTA pairs, the default) against tokens in M (128 tokens x 256 weight rows)
            def with_env(env, fn):
                old = {kk: os.environ.get(kk) for kk in env}
                os.environ.update(env)
                try:
                    return fn()
                finally:
                    for kk, vv in old.items():
                        if vv is None:
                            os.environ.pop(kk, None)
                        else:
                            os.environ[kk] = vv
            same = lambda ab: ab  # noqa: E731
            t_single = with_env({"MOE_LORA_PAIR": "0"}, lambda: timed_variant(same))
            t_unswapped = with_env({"MOE_LORA_SWAP": "0"}, lambda: timed_variant(same))
            out["secondary"]["swap_ab"] = {
                "weights_in_m_cta_pairs_ms_per_step": step_ms, "weights_in_m_one_cta_ms_per_step": t_single,
                "tokens_in_m_ms_per_step": t_unswapped,
                "tiles": "weights in M: 128 (one CTA) or 256 (pair) weight rows x 256 tokens; tokens in M: 128 "
                         "tokens x 256 weight rows; both GEMMs of the layer"}
        else:
            out["secondary"]["swap_ab"] = ("decode: only the swapped tile (weights in M) is built; a tile with "
                                           "tokens in M would leave most of the MMA's 128 rows empty")

    # ---- e2e: pinned host inputs -> device, route + forward, y -> pinned host, every step.
    #      Serving pipeline: the compute of step i on this stream, the input copy of step
    #      i + 1 and the output copy of step i - 1 on two copy streams (double-buffered
    #      device inputs and outputs), the first input copy and the last output copy inside
    #      the timed region; the same steps one after another are reported beside it
    e2e_steps = args.e2e_steps or steps
    hx = [b[0].cpu().pin_memory() for b in batches]
    ha = [b[1].cpu().pin_memory() for b in batches]
    hy = torch.empty((M, shape.H), dtype=torch.bfloat16).pin_memory()
    dxs = [torch.empty_like(batches[0][0]) for _ in range(2)]
    das = [torch.empty_like(batches[0][1]) for _ in range(2)]
    ys = [y, torch.empty_like(y)]
    for b in range(2):  # real inputs before the graphs' warm-up calls
        dxs[b].copy_(batches[b % nb][0])
        das[b].copy_(batches[b % nb][1])

    def e2e_compute(b):
        rt = ml.route(das[b], k, L, x=dxs[b], w_router=W["w_router"], bias=W["bias"], out=rbufs, workspace=rws)
        ml.forward(dxs[b], rt, W, k=k, L=L, y=ys[b], workspace=fws)

    def e2e_serial(j):
        dxs[0].copy_(hx[j], non_blocking=True)
        das[0].copy_(ha[j], non_blocking=True)
        e2e_compute(0)
        hy.copy_(ys[0], non_blocking=True)

    cgraphs = capture(lambda b: e2e_compute(b % 2), 2) if not args.no_graph else []
    sgraphs = capture(e2e_serial, nb) if not args.no_graph else []
    cs = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def h2d(i, b):
        with torch.cuda.stream(s_in):
            dxs[b].copy_(hx[i % nb], non_blocking=True)
            das[b].copy_(ha[i % nb], non_blocking=True)
            in_done[b].record(s_in)

    def pipelined(n):
        s_in.wait_stream(cs)
        s_out.wait_stream(cs)
        h2d(0, 0)
        for i in range(n):
            b = i % 2
            cs.wait_event(in_done[b])
            if i >= 2:
                cs.wait_event(out_done[b])  # ys[b] of step i - 2 has been copied out
            cgraphs[b].replay() if cgraphs else e2e_compute(b)
            comp_done[b].record(cs)
            if i + 1 < n:
                if i >= 1:
                    s_in.wait_event(comp_done[1 - b])  # step i - 1 is done with its inputs
                h2d(i + 1, 1 - b)
            s_out.wait_event(comp_done[b])
            with torch.cuda.stream(s_out):
                hy.copy_(ys[b], non_blocking=True)
                out_done[b].record(s_out)
        cs.wait_stream(s_out)
        cs.wait_stream(s_in)

    def timed(fn):
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        barrier(world)
        return max_over_ranks(e0.elapsed_time(e1), world)

    pipelined(min(4, e2e_steps))  # warm the copy streams
    e2e_ms = timed(lambda: pipelined(e2e_steps))
    serial_ms = timed(lambda: [sgraphs[i % nb].replay() if sgraphs else e2e_serial(i % nb) for i in range(e2e_steps)])
    del graphs, cgraphs, sgraphs
    ml.check_status(fws)
    ml.check_status(rws)
    out["e2e"] = {"value": world * M * e2e_steps / (e2e_ms / 1e3), "unit": "tokens/s",
                  "h2d_bytes_per_step": M * shape.H * 2 + M * 4, "d2h_bytes_per_step": M * shape.H * 2,
                  "how": ("serving pipeline: route + forward of step i (graph replay) while step i + 1's "
                          "inputs go in and step i - 1's y comes out on two copy streams; pinned host "
                          "buffers, every step's copies inside the timed region"),
                  "serial_value": world * M * e2e_steps / (serial_ms / 1e3),
                  "serial_how": "H2D copy, route, forward, D2H copy one after another (graph replay)"}
    return out


def sweep_steps(est_ms: float, seconds: float) -> int:
    return int(min(4000, max(20, seconds * 1e3 / max(est_ms, 1e-3))))


def bound_by(ent: dict, gemm: dict) -> str:
    """What holds a sweep step below the layer's copy-peak time: the GEMMs' share against
    the rest of the step, kernel by kernel (event-timed), and the launches per step."""
    ms = ent["ms_per_step"]
    kt = {k: v for k, v in ent["kernel_ms_per_step"].items() if v > 0}
    g = sum(v for k, v in kt.items() if k.startswith("gemm"))
    rest = sorted(((k, v) for k, v in kt.items() if not k.startswith("gemm")), key=lambda kv: -kv[1])
    lead = (f"the GEMMs take {g * 1e3:.1f} of {ms * 1e3:.1f} us (gate_up at {gemm['frac']:.2f} of the "
            f"{'tensor' if gemm['bound'] == 'tensor' else 'HBM copy'} peak)")
    tail = ", ".join(f"{k} {v * 1e3:.1f} us" for k, v in rest[:4])
    return (f"{lead}; the other kernels: {tail}; the layer's bytes at the copy peak take "
            f"{ent['layer_frac_of_hbm_peak'] * ms * 1e3:.1f} us; {ent['launches_per_step']:.0f} dependent launches "
            f"per step")


def run_sweep(args, world, local, skip: str) -> list:
    """The decode layers (and the dense decode projection) measured in the same process:
    tokens/s, the layer's fraction of the HBM copy peak and the gate_up GEMM's roofline,
    per workload and token count.  Weights are drawn on the device (seeded)."""
    dev = torch.device("cuda", local)
    res = []
    for name, Ms in SWEEP:
        shape = synth.WORKLOADS[name]
        if isinstance(shape, synth.DenseShape):
            if name == skip:
                continue
            est = measure_dense(args, shape, world, local, steps=20, warmup=3, full=False)
            n = sweep_steps(est["ms_per_step"], args.sweep_seconds)
            m = measure_dense(args, shape, world, local, steps=n, warmup=10, full=False)
            ent = {"workload": name, "M": shape.T, "tokens_per_s": m["value"], "ms_per_step": m["ms_per_step"],
                   "steps": n, "layer_frac_of_hbm_peak": m["layer"]["frac_of_hbm_peak"],
                   "gemm": {kk: m["roofline"][kk] for kk in ("bound", "achieved", "unit", "frac")},
                   "kernel_ms_per_step": m["layer"]["kernel_ms_per_step"], "gpu_launches": m["gpu_launches"],
                   "launches_per_step": m["gpu_launches"] / max(1, n)}
            if ent["layer_frac_of_hbm_peak"] < 0.70:
                ent["bound_by"] = bound_by(ent, ent["gemm"])
            res.append(ent)
            continue
        W = synth.moe_weights_device(shape, dev)
        for M in Ms:
            if name == skip and M == args.M:
                continue
            est = measure_moe(args, shape, M, W, world, local, steps=10, warmup=3, full=False)
            n = sweep_steps(est["ms_per_step"], args.sweep_seconds)
            m = measure_moe(args, shape, M, W, world, local, steps=n, warmup=10, full=False)
            ent = {"workload": name, "M": M, "tokens_per_s": m["value"], "ms_per_step": m["ms_per_step"],
                   "steps": n, "layer_frac_of_hbm_peak": m["layer"]["frac_of_hbm_peak"],
                   "gate_up": {kk: m["roofline"][kk] for kk in ("bound", "achieved", "unit", "frac")},
                   "kernel_ms_per_step": m["layer"]["kernel_ms_per_step"], "gpu_launches": m["gpu_launches"],
                   "launches_per_step": m["gpu_launches"] / max(1, n)}
            if ent["layer_frac_of_hbm_peak"] < 0.70:
                ent["bound_by"] = bound_by(ent, ent["gate_up"])
            res.append(ent)
        del W
        torch.cuda.empty_cache()
    return res


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
    import moe_lora_b200  # noqa: F401  (fails loudly without the CUDA library)

    shape = synth.WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    line = {"metric": METRIC, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "data": "synthetic"}
    if isinstance(shape, synth.MoEShape):
        M = args.M
        W = synth.moe_weights_device(shape, dev)
        m = measure_moe(args, shape, M, W, world, local, steps=args.steps, warmup=args.warmup, full=True)
        del W
        torch.cuda.empty_cache()
        line["dtype"] = "bf16" if shape.wdtype == "bf16" else "e4m3/bf16"
        line["config"] = {"workload": shape.name, "M": M, "tokens_per_step_per_gpu": M, "E": shape.E, "k": shape.k,
                          "H": shape.H, "I": shape.I, "L": shape.L, "r": shape.r, "wdtype": shape.wdtype,
                          "adapters": shape.adapter_dist, "router_bias": shape.bias,
                          "parallelism": f"replicas x{world}", "l2": m.pop("l2"),
                          "weights": "expert and adapter weights drawn on the device (seeded); router, bias, "
                                     "tokens and adapter ids from the seeded slice generator"}
    else:
        M = shape.T
        m = measure_dense(args, shape, world, local, steps=args.steps, warmup=args.warmup, full=True)
        line["dtype"] = shape.dtype
        line["config"] = {"workload": shape.name, "T": shape.T, "h_in": shape.h_in, "h_out": shape.h_out,
                          "L": shape.L, "r": shape.r, "adapters": shape.adapter_dist,
                          "parallelism": f"replicas x{world}", "l2": m.pop("l2")}
    clk = m.pop("clocks", None)
    per_step = m.pop("timing_per_step", None)
    plain = m.pop("plain_api_ms_per_step", None)
    line.update(m)
    line["steps"] = args.steps
    line["timing"] = {"mode": "CUDA graph replay of the API calls" if not args.no_graph else "plain API calls",
                      "plain_api_ms_per_step": plain, "per_step": per_step}
    line["clocks"] = clk
    if not args.no_sweep:
        line["sweep"] = run_sweep(args, world, local, skip=shape.name)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        if isinstance(shape, synth.MoEShape):
            # a bounded sample: the first tokens of batch 0, sized to about cpu_seconds
            sl = StoredSlices(shape)
            tps1, _, _, _ = oracle_tokens_per_s(shape, M, seconds=0.0, max_calls=1, tokens_per_call=1, slices=sl)
            tok = int(max(1, min(M, 64, args.cpu_seconds / 4.0 * tps1)))
            tps, calls, n, el = oracle_tokens_per_s(shape, M, seconds=args.cpu_seconds, tokens_per_call=tok,
                                                    slices=sl)
            sample = (f"fp64 oracle (route, sort, forward) on the first {n} tokens of batch 0, {calls} calls in "
                      f"{el:.1f} s; the fp64 conversion of the touched stored-precision slices is timed, "
                      "their generation is not")
        else:
            tps, calls, n, el = dense_oracle_tokens_per_s(shape, args.cpu_seconds)
            sample = (f"fp64 oracle, {n} tokens per call, {calls} calls in {el:.1f} s; "
                      "weights decoded to fp64 once before timing")
        line["cpu_baseline"] = {"value": tps, "unit": "tokens/s", **cores_desc(), "kind": "oracle",
                                "sample": sample}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
