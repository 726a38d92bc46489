"""GPU parity of moe_lora_forward (tcgen05 grouped GEMMs + SGMV LoRA) against the oracle."""
import os

import numpy as np
import pytest
import torch

import moe_lora_b200 as ml
from tests.gpu_cases import FP8_DESIGN_BOUND, TOL_BF16, TOL_FP8, CpuWeightsOracle, moe_weights_both, run_moe_case
from workloads import synth

pytestmark = pytest.mark.gpu

# Small shapes that still span several K blocks (64), several weight tiles (64 gate
# rows / 128 down rows), several token chunks, and ragged tails in every dimension.
SMALL = [
    synth.MoEShape("s_a", 200, E=8, k=2, H=384, I=192, L=3, r=16, no_adapter_frac=0.2),
    synth.MoEShape("s_ragged", 201, E=6, k=3, H=520, I=136, L=2, r=8, no_adapter_frac=0.25),
    synth.MoEShape("s_r64", 202, E=4, k=2, H=256, I=128, L=4, r=64, adapter_dist="zipf"),
    synth.MoEShape("s_r128", 203, E=5, k=2, H=264, I=200, L=2, r=128),
    synth.MoEShape("s_noadapter", 204, E=8, k=4, H=256, I=256, L=2, r=32, no_adapter_frac=1.0),
    synth.MoEShape("s_L0", 205, E=8, k=2, H=192, I=128, L=0, r=16),
    synth.MoEShape("s_kE", 206, E=4, k=4, H=128, I=64, L=1, r=16),
    synth.MoEShape("s_E1", 207, E=1, k=1, H=256, I=384, L=3, r=16),
    synth.MoEShape("s_bias_zipf", 208, E=16, k=8, H=512, I=320, L=8, r=32, bias=True, adapter_dist="zipf"),
    # r K >= 65536: the LoRA shrink splits K over CTAs (slices of 1024, ragged last slice)
    synth.MoEShape("s_split", 209, E=4, k=2, H=1032, I=1096, L=3, r=64, no_adapter_frac=0.2),
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: s.name)
@pytest.mark.parametrize("M", [1, 3, 37, 300])
def test_forward_small_shapes(shape, M):
    res = run_moe_case(shape, M)
    assert res["err"] <= TOL_BF16, res["err"]


@pytest.mark.parametrize("where", ["delta", "tc"])
@pytest.mark.parametrize("bn", [16, 32, 64, 128, 256])
def test_forward_every_n_tile(bn, where, monkeypatch):
    """Every N tile, with the LoRA delta from the SIMT LoRA kernel (fp32) and from the
    tensor-core LoRA kernel (bf16), each added by the GEMM epilogue."""
    monkeypatch.setenv("MOE_LORA_FORCE_BN", str(bn))
    monkeypatch.setenv("MOE_LORA_EXPAND", where)
    res = run_moe_case(SMALL[0], 300)
    assert res["err"] <= TOL_BF16, res["err"]
    res = run_moe_case(SMALL[1], 37)
    assert res["err"] <= TOL_BF16, res["err"]


@pytest.mark.parametrize("where", ["delta", "tc"])
@pytest.mark.parametrize("shape,M", [(SMALL[1], 37), (SMALL[2], 300), (SMALL[3], 37), (SMALL[7], 37),
                                     (SMALL[8], 300), (SMALL[8], 1), (SMALL[9], 37), (SMALL[9], 300)],
                         ids=lambda v: getattr(v, "name", str(v)))
def test_forward_expand_placement(shape, M, where, monkeypatch):
    """Every placement of the LoRA work on ragged shapes, r = 8 .. 128, E = 1."""
    monkeypatch.setenv("MOE_LORA_EXPAND", where)
    res = run_moe_case(shape, M)
    assert res["err"] <= TOL_BF16, res["err"]


@pytest.mark.parametrize("variant", ["single", "pair", "tokens_in_m"])
@pytest.mark.parametrize("shape,M", [(SMALL[0], 300), (SMALL[2], 700), (SMALL[3], 300), (SMALL[7], 600),
                                     (SMALL[8], 400), (SMALL[9], 300)], ids=lambda v: getattr(v, "name", str(v)))
def test_forward_n256_single_pair_and_unswapped(shape, M, variant, monkeypatch):
    """Tiles of 256 tokens on one CTA and on CTA pairs (cta_group::2: ragged last chunks,
    the pair's N rounded to 32 and split between the CTAs, odd chunk counts), and the
    unswapped tile (128 tokens in M, 256 weight rows in N); r = 64 and 128, E = 1, K with
    a ragged last K block, I and H not multiples of the weight tile."""
    monkeypatch.setenv("MOE_LORA_FORCE_BN", "256")
    monkeypatch.setenv("MOE_LORA_EXPAND", "tc")
    monkeypatch.setenv("MOE_LORA_PAIR", "1" if variant == "pair" else "0")
    if variant == "tokens_in_m":
        monkeypatch.setenv("MOE_LORA_SWAP", "0")
    res = run_moe_case(shape, M)
    assert res["err"] <= TOL_BF16, (shape.name, res["err"])


@pytest.fixture(scope="module")
def decode_weights():
    return moe_weights_both(synth.MOE_DECODE_BF16)


@pytest.mark.parametrize("M", [1, 8, 32, 64])
def test_forward_moe_decode_bf16_full(decode_weights, M):
    res = run_moe_case(synth.MOE_DECODE_BF16, M, weights=decode_weights)
    assert res["err"] <= TOL_BF16, res["err"]
    ml.check_status(res["rt"]["workspace"])


def test_forward_deterministic(decode_weights):
    s = synth.MOE_DECODE_BF16
    a = run_moe_case(s, 64, weights=decode_weights)
    y2 = ml.forward(a["x"].cuda(), a["rt"], a["dev"], k=s.k, L=s.L)
    torch.cuda.synchronize()
    assert torch.equal(a["y"], y2)


def test_all_adapters_none_equals_zero_b(decode_weights):
    """Early exit of adapter -1 and a zero expand B give the same bits."""
    s = synth.MOE_DECODE_BF16
    cpu, dev, _ = decode_weights
    x, ad = synth.moe_tokens(s, 32)
    lin = synth.moe_logits_in(s, 32).cuda()
    none = torch.full_like(ad, -1).cuda()
    rt0 = ml.route(none, s.k, s.L, logits_in=lin)
    y0 = ml.forward(x.cuda(), rt0, dev, k=s.k, L=s.L)
    devz = dict(dev)
    devz["b_gu"] = torch.zeros_like(dev["b_gu"])
    devz["b_d"] = torch.zeros_like(dev["b_d"])
    rt1 = ml.route(ad.cuda(), s.k, s.L, logits_in=lin)
    y1 = ml.forward(x.cuda(), rt1, devz, k=s.k, L=s.L)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)


@pytest.fixture(scope="module")
def prefill_weights():
    return moe_weights_both(synth.MOE_PREFILL_BF16)


def test_forward_moe_prefill_bf16_full(prefill_weights):
    """All 4096 tokens of the prefill layer against the oracle: every expert's ragged
    last 256-row chunk and every (expert, adapter) segment boundary is checked.  The
    oracle view decodes one expert (and its adapters) at a time, so the fp64 weights
    are never all resident."""
    cpu, dev, _ = prefill_weights
    s = synth.MOE_PREFILL_BF16
    res = run_moe_case(s, 4096, weights=(cpu, dev, CpuWeightsOracle(s, cpu, cache=False)))
    print(f"prefill M=4096: max|err|/max|ref| = {res['err']:.3e} over {len(res['tokens'])} tokens")
    assert len(res["tokens"]) == 4096
    assert res["err"] <= TOL_BF16, res["err"]
    ml.check_status(res["rt"]["workspace"])


# ---------------------------------------------------------------- adapter formats: separate
# gate and up adapters, per-projection scales
SPLIT = [
    synth.MoEShape("sp_a", 230, E=8, k=2, H=384, I=192, L=3, r=16, gu_split=True, no_adapter_frac=0.2),
    synth.MoEShape("sp_r64", 231, E=4, k=2, H=256, I=128, L=4, r=64, gu_split=True, adapter_dist="zipf"),
    synth.MoEShape("sp_r8", 232, E=6, k=3, H=520, I=256, L=2, r=8, gu_split=True, no_adapter_frac=0.25),
]


@pytest.mark.parametrize("where", ["delta", "tc"])
@pytest.mark.parametrize("shape", SPLIT, ids=lambda s: s.name)
@pytest.mark.parametrize("M", [37, 300])
def test_forward_split_gate_up_with_scales(shape, M, where, monkeypatch):
    monkeypatch.setenv("MOE_LORA_EXPAND", where)
    res = run_moe_case(shape, M, scale_gu=0.5, scale_d=2.0)
    assert res["err"] <= TOL_BF16, res["err"]


def test_forward_split_ragged_intermediate_decode():
    """Separate gate and up adapters with I not a multiple of 64 (the CUDA-core LoRA path)."""
    s = synth.MoEShape("sp_ragged", 233, E=6, k=3, H=520, I=136, L=2, r=32, gu_split=True)
    res = run_moe_case(s, 37, scale_gu=1.5, scale_d=0.25)
    assert res["err"] <= TOL_BF16, res["err"]


@pytest.mark.parametrize("M", [64, 1024])
def test_forward_split_decode_bf16_shape(M):
    """The bf16 decode layer's shape (E=64, H=2048, I=1408) with separate gate and up
    adapters and scales: M=64 runs the CUDA-core LoRA path, M=1024 (128 rows per expert)
    the tensor-core one."""
    s = synth.MOE_DECODE_BF16.with_(name="decode_split", wid=234, gu_split=True)
    res = run_moe_case(s, M, scale_gu=0.25, scale_d=0.5)
    assert res["err"] <= TOL_BF16, res["err"]


def test_forward_split_prefill_shape_sampled():
    """The prefill layer's shape (M=4096, E=128, H=4096, I=1536, r=64) with separate gate
    and up adapters and scales, on 320 tokens the oracle computes one by one."""
    s = synth.MOE_PREFILL_BF16.with_(name="prefill_split", wid=235, gu_split=True)
    toks = np.unique(np.concatenate([np.arange(32), np.arange(4096 - 32, 4096),
                                     np.random.default_rng(2).choice(4096, 256, replace=False)]))
    cpu, dev, _ = moe_weights_both(s)
    res = run_moe_case(s, 4096, weights=(cpu, dev, CpuWeightsOracle(s, cpu, cache=False)), tokens=toks,
                       scale_gu=2.0, scale_d=0.5)
    assert res["err"] <= TOL_BF16, res["err"]


# ---------------------------------------------------------------- FP8 (e4m3) expert weights
def check_fp8(res, label, record_property):
    """The stated FP8 gate and the tighter bound of the two-plane activation design;
    the achieved error is printed and recorded for every case."""
    print(f"fp8 {label}: max|err|/max|ref| = {res['err']:.3e}")
    record_property("fp8_rel_err", res["err"])
    assert res["err"] <= TOL_FP8, res["err"]
    assert res["err"] <= FP8_DESIGN_BOUND, res["err"]


SMALL_FP8 = [
    synth.MoEShape("f8_a", 220, E=8, k=2, H=384, I=192, L=3, r=16, wdtype="e4m3", no_adapter_frac=0.2),
    synth.MoEShape("f8_ragged", 221, E=6, k=3, H=528, I=144, L=2, r=32, wdtype="e4m3", bias=True,
                   adapter_dist="zipf", no_adapter_frac=0.25),
    synth.MoEShape("f8_L0", 222, E=4, k=2, H=256, I=128, L=0, r=16, wdtype="e4m3"),
]


@pytest.mark.parametrize("shape", SMALL_FP8, ids=lambda s: s.name)
@pytest.mark.parametrize("M", [1, 5, 37, 200])
def test_forward_fp8_small_shapes(shape, M, record_property):
    check_fp8(run_moe_case(shape, M), f"{shape.name} M={M}", record_property)


@pytest.mark.parametrize("where", ["delta", "tc"])
@pytest.mark.parametrize("bn", [16, 32, 64, 128, 256])
def test_forward_fp8_every_n_tile(bn, where, monkeypatch, record_property):
    """Every N tile of the e4m3 GEMM (256 is clamped to 128: the two activation planes
    make the MMA's N twice the tile's)."""
    monkeypatch.setenv("MOE_LORA_FORCE_BN", str(bn))
    monkeypatch.setenv("MOE_LORA_EXPAND", where)
    check_fp8(run_moe_case(SMALL_FP8[1], 150), f"{SMALL_FP8[1].name} bn={bn} {where}", record_property)


F8_PAIR = synth.MoEShape("f8_pair", 223, E=6, k=3, H=512, I=256, L=2, r=32, wdtype="e4m3", bias=True,
                         adapter_dist="zipf", no_adapter_frac=0.25)


@pytest.mark.parametrize("variant", ["single", "pair"])
@pytest.mark.parametrize("M", [37, 300])
def test_forward_fp8_single_and_pair(M, variant, monkeypatch, record_property):
    """e4m3 tiles of 128 tokens on one CTA and on CTA pairs (cta_group::2, M = 256: the
    leader stages the hi activation plane, its peer the lo plane), over even weight-tile
    counts with a router bias that skews the groups, so chunks are ragged and uneven."""
    monkeypatch.setenv("MOE_LORA_FORCE_BN", "128")
    monkeypatch.setenv("MOE_LORA_PAIR", "1" if variant == "pair" else "0")
    check_fp8(run_moe_case(F8_PAIR, M), f"{F8_PAIR.name} M={M} {variant}", record_property)


@pytest.fixture(scope="module")
def fp8_weights():
    return moe_weights_both(synth.MOE_DECODE_FP8)


@pytest.mark.parametrize("M", [1, 4, 16, 64])
def test_forward_moe_decode_fp8_full(fp8_weights, M, record_property):
    res = run_moe_case(synth.MOE_DECODE_FP8, M, weights=fp8_weights)
    check_fp8(res, f"{synth.MOE_DECODE_FP8.name} M={M}", record_property)
    ml.check_status(res["rt"]["workspace"])


def test_forward_moe_prefill_fp8_sampled(fp8_weights, record_property):
    """FP8 prefill: the e4m3 experts and rank-32 adapters of the FP8 decode layer at 4096
    tokens (256 pairs per expert: the tensor-core LoRA kernel and N tiles of 256 on the
    kind::f8f6f4 GEMM), on 320 tokens the oracle computes one by one (the first and last
    32, and 256 drawn at random)."""
    s = synth.MOE_DECODE_FP8
    cpu, dev, _ = fp8_weights
    toks = np.unique(np.concatenate([np.arange(32), np.arange(4096 - 32, 4096),
                                     np.random.default_rng(3).choice(4096, 256, replace=False)]))
    res = run_moe_case(s, 4096, weights=(cpu, dev, CpuWeightsOracle(s, cpu, cache=False)), tokens=toks)
    check_fp8(res, f"{s.name} M=4096 ({len(toks)} tokens)", record_property)
    ml.check_status(res["rt"]["workspace"])
