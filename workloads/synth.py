"""Seeded synthetic inputs for the MoE + multi-LoRA layer and the dense SGMV layer.

This module only draws random numbers and stores them at the precision the
kernels read (fp32, bf16 or OCP e4m3 with one fp32 scale per tensor).  It holds
none of the method's arithmetic: no routing, no sort, no GEMM, no activation.
Both the GPU path (tests, bench, smoke) and the oracle side consume what it
returns; neither side's code lives here.

Every tensor is split into independently seeded slices (one expert, one
(adapter, expert) pair, the token batch), so a full-size workload can be built
on the device slice by slice and the oracle can regenerate only the slices it
touches.  The seed of a slice is

    numpy.random.default_rng([20261202, workload_id, tensor_tag, *index])

Distributions (variance, as N(mean, variance)):
  x ~ N(0, 1); router W_r ~ N(0, 1/H); expert W_gu ~ N(0, 1/H), W_d ~ N(0, 1/I);
  dense W ~ N(0, 1/h_in); LoRA A ~ N(0, 1/h_in of its projection), B ~ N(0, 1/r);
  router bias ~ N(0, 0.5) where the workload skews expert load.
  Adapter ids: uniform over L, or finite Zipf P(i) ~ (i+1)^-1.1 (id 0 most popular).
FP8 weights: drawn in fp32, scale = amax/448, code = RNE(w/scale) to e4m3fn.
"""
from __future__ import annotations

import concurrent.futures as _cf
import os
from dataclasses import dataclass, replace

import numpy as np
import torch

BASE_SEED = 20261202

# tensor tags (part of every slice seed)
T_X, T_ADAPTER, T_WR, T_BIAS, T_WGU, T_WD, T_AGU, T_BGU, T_AD, T_BD, T_LOGITS = range(1, 12)
T_DX, T_DW, T_DA, T_DB, T_DADAPTER = range(20, 25)


@dataclass(frozen=True)
class MoEShape:
    """One MoE + multi-LoRA layer: E experts, top-k, hidden H, expert intermediate I,
    L adapters of rank r on gate_up (H -> 2I) and down (I -> H)."""
    name: str
    wid: int
    E: int
    k: int
    H: int
    I: int
    L: int
    r: int
    wdtype: str = "bf16"          # "bf16" or "e4m3"
    bias: bool = False            # router bias skewing expert load
    adapter_dist: str = "uniform"  # "uniform" or "zipf"
    M_list: tuple = (64,)
    no_adapter_frac: float = 0.0  # share of tokens with adapter id -1 (base only)
    gu_split: bool = False        # separate gate and up adapters (A [2][r][H], B [2][r][I])

    def with_(self, **kw) -> "MoEShape":
        return replace(self, **kw)


@dataclass(frozen=True)
class DenseShape:
    """One dense projection h_in -> h_out with L adapters of rank r (SGMV)."""
    name: str
    wid: int
    T: int
    h_in: int
    h_out: int
    L: int
    r: int
    dtype: str = "f32"            # "f32" or "bf16"
    adapter_dist: str = "uniform"
    no_adapter_frac: float = 0.0

    def with_(self, **kw) -> "DenseShape":
        return replace(self, **kw)


# The five workloads of the hot path, named by what they are.
SGMV_F32 = DenseShape("sgmv_f32_t64_h512", 0, T=64, h_in=512, h_out=512, L=4, r=16,
                      dtype="f32", adapter_dist="uniform")
DENSE_DECODE_BF16 = DenseShape("dense_decode_bf16_t64_4096x11008", 1, T=64, h_in=4096,
                               h_out=11008, L=32, r=16, dtype="bf16", adapter_dist="zipf")
MOE_DECODE_BF16 = MoEShape("moe_decode_bf16_e64_h2048_i1408", 2, E=64, k=8, H=2048, I=1408,
                           L=8, r=16, wdtype="bf16", bias=False, adapter_dist="uniform",
                           M_list=(1, 8, 32, 64))
MOE_PREFILL_BF16 = MoEShape("moe_prefill_bf16_e128_h4096_i1536", 3, E=128, k=8, H=4096,
                            I=1536, L=16, r=64, wdtype="bf16", bias=True, adapter_dist="zipf",
                            M_list=(4096,))
MOE_DECODE_FP8 = MoEShape("moe_decode_fp8_e128_h7168_i2048", 4, E=128, k=8, H=7168, I=2048,
                          L=32, r=32, wdtype="e4m3", bias=True, adapter_dist="zipf",
                          M_list=(1, 4, 16, 64))

# A profiling-size cut of the prefill layer: a quarter of the experts and tokens, so 256
# pairs per expert (the full layer's tile shapes) with about 2 GB of weights on the device.
MOE_PREFILL_BF16_SMALL = MOE_PREFILL_BF16.with_(name="moe_prefill_bf16_e32_h4096_i1536", wid=5, E=32,
                                                M_list=(1024,))

WORKLOADS = {w.name: w for w in (SGMV_F32, DENSE_DECODE_BF16, MOE_DECODE_BF16,
                                 MOE_PREFILL_BF16, MOE_DECODE_FP8, MOE_PREFILL_BF16_SMALL)}


def rng(*key: int) -> np.random.Generator:
    return np.random.default_rng([BASE_SEED, *[int(v) for v in key]])


def normal_f32(g: np.random.Generator, shape, var: float) -> np.ndarray:
    a = g.standard_normal(shape, dtype=np.float32)
    a *= np.float32(np.sqrt(var))
    return a


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """fp32 -> bf16 with round-to-nearest-even (torch's cast)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def quant_e4m3(a: np.ndarray) -> tuple[torch.Tensor, float]:
    """Per-tensor e4m3 quantisation: scale = amax/448, code = RNE(w/scale)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    amax = float(t.abs().max())
    scale = np.float32(amax / 448.0) if amax > 0 else np.float32(1.0)
    q = (t / torch.tensor(scale, dtype=torch.float32)).to(torch.float8_e4m3fn)
    return q, float(scale)


def adapter_probs(L: int, dist: str) -> np.ndarray:
    if dist == "uniform":
        return np.full(L, 1.0 / L)
    if dist == "zipf":
        p = (np.arange(L, dtype=np.float64) + 1.0) ** -1.1
        return p / p.sum()
    raise ValueError(dist)


def draw_adapter_ids(g: np.random.Generator, n: int, L: int, dist: str,
                     no_adapter_frac: float) -> np.ndarray:
    if L == 0:
        return np.full(n, -1, dtype=np.int32)
    ids = g.choice(L, size=n, p=adapter_probs(L, dist)).astype(np.int32)
    if no_adapter_frac > 0:
        ids[g.random(n) < no_adapter_frac] = -1
    return ids


# ----------------------------------------------------------------------------- MoE slices

def moe_tokens(s: MoEShape, M: int, batch: int = 0) -> tuple[torch.Tensor, torch.Tensor]:
    """x bf16 [M, H] and per-token adapter id int32 [M] (-1 = base only).

    `batch` selects one of several independent batches of the same size."""
    key = (M,) if batch == 0 else (M, batch)
    x = to_bf16(normal_f32(rng(s.wid, T_X, *key), (M, s.H), 1.0))
    ids = draw_adapter_ids(rng(s.wid, T_ADAPTER, *key), M, s.L, s.adapter_dist, s.no_adapter_frac)
    return x, torch.from_numpy(ids)


def moe_router(s: MoEShape) -> tuple[torch.Tensor, torch.Tensor | None]:
    """Router weight bf16 stored [E, H] and optional per-expert bias fp32 [E]."""
    wr = to_bf16(normal_f32(rng(s.wid, T_WR), (s.E, s.H), 1.0 / s.H))
    bias = None
    if s.bias:
        bias = torch.from_numpy(normal_f32(rng(s.wid, T_BIAS), (s.E,), 0.5))
    return wr, bias


def moe_logits_in(s: MoEShape, M: int) -> torch.Tensor:
    """Given router logits fp32 [M, E] (N(0,1), plus the bias where the workload has one)."""
    lg = normal_f32(rng(s.wid, T_LOGITS, M), (M, s.E), 1.0)
    if s.bias:
        lg = lg + moe_router(s)[1].numpy()[None, :]
    return torch.from_numpy(np.ascontiguousarray(lg, dtype=np.float32))


def moe_expert(s: MoEShape, e: int):
    """Expert e: (w_gu [2I, H], w_d [H, I], scale_gu, scale_d) at stored precision.

    Rows are output features, contiguous over the reduction dim (K-major).  The
    first I rows of w_gu are the gate projection, the last I the up projection."""
    gu = normal_f32(rng(s.wid, T_WGU, e), (2 * s.I, s.H), 1.0 / s.H)
    d = normal_f32(rng(s.wid, T_WD, e), (s.H, s.I), 1.0 / s.I)
    if s.wdtype == "bf16":
        return to_bf16(gu), to_bf16(d), 1.0, 1.0
    qg, sg = quant_e4m3(gu)
    qd, sd = quant_e4m3(d)
    return qg, qd, sg, sd


def moe_adapter(s: MoEShape, a: int, e: int):
    """Adapter a on expert e, bf16: A_gu [r, H], B_gu [r, 2I], A_d [r, I], B_d [r, H]; with
    separate gate and up adapters (gu_split) A_gu [2, r, H] and B_gu [2, r, I] (gate, up).

    A is stored transposed (r rows, each contiguous over h_in); B as r rows over h_out."""
    if s.gu_split:
        ag = to_bf16(normal_f32(rng(s.wid, T_AGU, a, e), (2, s.r, s.H), 1.0 / s.H))
        bg = to_bf16(normal_f32(rng(s.wid, T_BGU, a, e), (2, s.r, s.I), 1.0 / s.r))
    else:
        ag = to_bf16(normal_f32(rng(s.wid, T_AGU, a, e), (s.r, s.H), 1.0 / s.H))
        bg = to_bf16(normal_f32(rng(s.wid, T_BGU, a, e), (s.r, 2 * s.I), 1.0 / s.r))
    ad = to_bf16(normal_f32(rng(s.wid, T_AD, a, e), (s.r, s.I), 1.0 / s.I))
    bd = to_bf16(normal_f32(rng(s.wid, T_BD, a, e), (s.r, s.H), 1.0 / s.r))
    return ag, bg, ad, bd


def _pool():
    return _cf.ThreadPoolExecutor(max_workers=max(1, min(32, os.cpu_count() or 1)))


def moe_weights(s: MoEShape, device="cpu") -> dict:
    """All layer weights stacked: w_gu [E,2I,H], w_d [E,H,I], scales [E,2] fp32,
    A_gu [L,E,r,H], B_gu [L,E,r,2I], A_d [L,E,r,I], B_d [L,E,r,H], router, bias.

    Built slice by slice (threaded generation, copies into preallocated tensors)."""
    wdt = torch.bfloat16 if s.wdtype == "bf16" else torch.float8_e4m3fn
    out = {
        "w_gu": torch.empty((s.E, 2 * s.I, s.H), dtype=wdt, device=device),
        "w_d": torch.empty((s.E, s.H, s.I), dtype=wdt, device=device),
        "scales": torch.ones((s.E, 2), dtype=torch.float32),
        "a_gu": torch.empty((s.L, s.E, 2, s.r, s.H) if s.gu_split else (s.L, s.E, s.r, s.H),
                            dtype=torch.bfloat16, device=device),
        "b_gu": torch.empty((s.L, s.E, 2, s.r, s.I) if s.gu_split else (s.L, s.E, s.r, 2 * s.I),
                            dtype=torch.bfloat16, device=device),
        "a_d": torch.empty((s.L, s.E, s.r, s.I), dtype=torch.bfloat16, device=device),
        "b_d": torch.empty((s.L, s.E, s.r, s.H), dtype=torch.bfloat16, device=device),
    }
    with _pool() as ex:
        for e, (gu, d, sg, sd) in enumerate(ex.map(lambda e: moe_expert(s, e), range(s.E))):
            out["w_gu"][e].copy_(gu)
            out["w_d"][e].copy_(d)
            out["scales"][e, 0] = sg
            out["scales"][e, 1] = sd
        keys = [(a, e) for a in range(s.L) for e in range(s.E)]
        for (a, e), (ag, bg, ad, bd) in zip(keys, ex.map(lambda ae: moe_adapter(s, *ae), keys)):
            out["a_gu"][a, e].copy_(ag)
            out["b_gu"][a, e].copy_(bg)
            out["a_d"][a, e].copy_(ad)
            out["b_d"][a, e].copy_(bd)
    wr, bias = moe_router(s)
    out["w_router"] = wr.to(device)
    out["bias"] = None if bias is None else bias.to(device)
    out["scales"] = out["scales"].to(device)
    return out


def moe_weights_device(s: MoEShape, device, seed: int = 0) -> dict:
    """The same layout and distributions as moe_weights, drawn on the device by torch's
    seeded generator (one stream per workload and seed) instead of the per-slice numpy
    streams: gigabytes in well under a second, for timing runs whose results are not
    compared with the oracle.  The router weight and bias come from the numpy streams
    (moe_router), so routing of a given token batch is the same as with moe_weights."""
    g = torch.Generator(device=device)
    g.manual_seed(BASE_SEED * 1000 + s.wid * 10 + seed)
    wdt = torch.bfloat16 if s.wdtype == "bf16" else torch.float8_e4m3fn

    def draw(shape, var):
        return torch.randn(shape, generator=g, device=device, dtype=torch.float32).mul_(float(np.sqrt(var)))

    out = {"w_gu": torch.empty((s.E, 2 * s.I, s.H), dtype=wdt, device=device),
           "w_d": torch.empty((s.E, s.H, s.I), dtype=wdt, device=device),
           "scales": torch.ones((s.E, 2), dtype=torch.float32, device=device)}
    for e in range(s.E):
        for name, shape, var, col in (("w_gu", (2 * s.I, s.H), 1.0 / s.H, 0), ("w_d", (s.H, s.I), 1.0 / s.I, 1)):
            w = draw(shape, var)
            if s.wdtype == "bf16":
                out[name][e].copy_(w)
            else:  # per-tensor e4m3: scale = amax / 448, code = RNE(w / scale)
                amax = float(w.abs().max())
                sc = np.float32(amax / 448.0) if amax > 0 else np.float32(1.0)
                out[name][e].copy_((w / torch.tensor(sc, dtype=torch.float32, device=device)).to(wdt))
                out["scales"][e, col] = float(sc)
    sp = (2,) if s.gu_split else ()
    for name, lead, cols, var in (("a_gu", sp, s.H, 1.0 / s.H),
                                  ("b_gu", sp, s.I if s.gu_split else 2 * s.I, 1.0 / s.r),
                                  ("a_d", (), s.I, 1.0 / s.I), ("b_d", (), s.H, 1.0 / s.r)):
        t = torch.empty((s.L, s.E, *lead, s.r, cols), dtype=torch.bfloat16, device=device)
        for a in range(s.L):
            t[a].copy_(draw((s.E, *lead, s.r, cols), var))
        out[name] = t
    wr, bias = moe_router(s)
    out["w_router"] = wr.to(device)
    out["bias"] = None if bias is None else bias.to(device)
    return out


# ----------------------------------------------------------------------------- dense slices

def dense_tokens(s: DenseShape, T: int | None = None):
    """x [T, h_in] and the adapter id per token, tokens grouped into contiguous
    segments (stable sort by adapter id, segments = maximal runs).

    Returns x, token_adapter [T], seg_offsets [S+1], seg_adapter [S] (int32)."""
    T = s.T if T is None else T
    xf = normal_f32(rng(s.wid, T_DX, T), (T, s.h_in), 1.0)
    x = torch.from_numpy(xf) if s.dtype == "f32" else to_bf16(xf)
    ids = draw_adapter_ids(rng(s.wid, T_DADAPTER, T), T, s.L, s.adapter_dist, s.no_adapter_frac)
    ids = np.sort(ids, kind="stable")
    offs, segs = [0], []
    for i in range(T):
        if i == 0 or ids[i] != ids[i - 1]:
            if i > 0:
                offs.append(i)
            segs.append(int(ids[i]))
    if T > 0:
        offs.append(T)
    return (x, torch.from_numpy(ids.astype(np.int32)),
            torch.tensor(offs, dtype=torch.int32), torch.tensor(segs, dtype=torch.int32))


def dense_weights(s: DenseShape, device="cpu") -> dict:
    """W stored [h_out, h_in]; A [L, r, h_in]; B [L, r, h_out] at the layer's dtype."""
    conv = (lambda a: torch.from_numpy(a)) if s.dtype == "f32" else to_bf16
    w = conv(normal_f32(rng(s.wid, T_DW), (s.h_out, s.h_in), 1.0 / s.h_in))
    a = torch.stack([conv(normal_f32(rng(s.wid, T_DA, i), (s.r, s.h_in), 1.0 / s.h_in))
                     for i in range(s.L)]) if s.L else torch.empty((0, s.r, s.h_in))
    b = torch.stack([conv(normal_f32(rng(s.wid, T_DB, i), (s.r, s.h_out), 1.0 / s.r))
                     for i in range(s.L)]) if s.L else torch.empty((0, s.r, s.h_out))
    return {"w": w.to(device), "a": a.to(device), "b": b.to(device)}


# ----------------------------------------------------------------------------- raw views

def bits(t: torch.Tensor) -> np.ndarray:
    """Raw storage of a CPU tensor as numpy: bf16 -> uint16, e4m3 -> uint8, fp32 -> float32."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    if t.dtype == torch.float32:
        return t.numpy()
    if t.dtype in (torch.int32, torch.int64):
        return t.numpy()
    raise TypeError(t.dtype)
