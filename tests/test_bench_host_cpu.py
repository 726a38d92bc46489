"""Host-side logic of bench.py on CPU: routing statistics, the byte models behind the
roofline numbers (hand-counted on tiny shapes), the expand-placement rule and the
per-step percentiles."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from workloads import synth  # noqa: E402

TINY = synth.MoEShape("tiny", 900, E=2, k=1, H=8, I=4, L=1, r=2)


def test_routing_stats_counts_touched_experts_and_pairs():
    shape = synth.MoEShape("t", 901, E=3, k=1, H=8, I=4, L=2, r=2)
    # rows per key e * (L + 1) + a', a' = L for tokens without an adapter
    counts = [2, 0, 1,   # expert 0: adapter 0, none
              0, 0, 0,   # expert 1: untouched
              0, 3, 0]   # expert 2: adapter 1
    so = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int32)
    assert bench.routing_stats({"seg_offsets": so}, shape) == (2, 2)


def test_lora_placement_boundary(monkeypatch):
    monkeypatch.delenv("MOE_LORA_EXPAND", raising=False)
    s = synth.MOE_DECODE_BF16  # E = 64, k = 8: more than 64 rows per expert above M = 512
    assert bench.lora_place(s, 512) == "delta"
    assert bench.lora_place(s, 513) == "tc"
    monkeypatch.setenv("MOE_LORA_EXPAND", "tc")
    assert bench.lora_place(s, 1) == "tc"


def test_gateup_bytes_hand_counted(monkeypatch):
    monkeypatch.delenv("MOE_LORA_EXPAND", raising=False)
    # delta form (3 rows <= 64 per expert): weights 2*2I*H*2 = 256, x 3*H*2 = 48,
    # fp32 delta 3*2I*4 = 96, act 3*I*2 = 24
    assert bench.gateup_alg_bytes(TINY, 3, experts=2, pairs=1) == 256 + 48 + 96 + 24
    # e4m3 weights: 1 byte per weight, x as two planes plus two fp32 scales per row
    f8 = TINY.with_(wdtype="e4m3")
    assert bench.gateup_alg_bytes(f8, 3, experts=2, pairs=1) == 128 + 3 * (2 * 8 + 8) + 96 + 24
    # tensor-core LoRA kernel (100 rows on one expert): the bf16 delta 100*2I*2
    one = TINY.with_(E=1)
    assert bench.gateup_alg_bytes(one, 100, experts=1, pairs=1) == 128 + 1600 + 1600 + 800
    assert bench.gateup_alg_flops(one, 100) == 2 * 100 * 8 * 8


def test_layer_bytes_hand_counted():
    # experts 2 * (2I*H + H*I) * 2 = 384; one (adapter, expert) slice r*(H + 2I + I + H)*2 = 112;
    # router E*H*2 = 32; x and y 3*H*2*2 = 96; adapter ids 3*4 = 12
    assert bench.layer_alg_bytes(TINY, 3, experts=2, pairs=1) == 384 + 112 + 32 + 96 + 12


def test_step_percentiles_from_event_times(monkeypatch):
    clock = {"t": 0.0}

    class Ev:
        def __init__(self, enable_timing=True):
            self.v = None

        def record(self):
            self.v = clock["t"]

        def elapsed_time(self, other):
            return other.v - self.v

    durations = [float(d) for d in range(1, 101)]

    def run_step(i):
        clock["t"] += durations[i]

    monkeypatch.setattr(torch.cuda, "Event", Ev)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda: None)
    assert bench.step_percentiles(run_step, 100) == {"p10_ms": 11.0, "p50_ms": 51.0, "p90_ms": 90.0,
                                                     "steps": 100}


def test_step_percentiles_never_raises():
    def run_step(i):
        raise RuntimeError("no device")

    out = bench.step_percentiles(run_step, 5)
    assert set(out) == {"error"}
