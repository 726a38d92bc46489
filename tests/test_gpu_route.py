"""GPU parity of moe_lora_route against the oracle (bit-exact ids, pairs, offsets)."""
import numpy as np
import pytest
import torch

import moe_lora_b200 as ml
from oracle import formats
from oracle import moe_lora_ref as ref
from tests.gpu_cases import oracle_routing_from_logits
from tests.oracle_inputs import MoEOracleWeights
from workloads import synth

pytestmark = pytest.mark.gpu


def _logits(M, E, seed, ties):
    g = np.random.default_rng(seed)
    if ties:  # few distinct values: many exact ties
        lg = g.integers(-4, 5, size=(M, E)).astype(np.float32) * np.float32(0.25)
    else:
        lg = g.standard_normal((M, E), dtype=np.float32)
    return torch.from_numpy(lg)


def _adapters(M, L, seed, none_frac=0.2):
    g = np.random.default_rng(seed + 1)
    a = g.integers(0, max(L, 1), size=M).astype(np.int32)
    if L == 0:
        a[:] = -1
    a[g.random(M) < none_frac] = -1
    return a


def _check_exact(M, E, k, L, seed, ties=False):
    lg = _logits(M, E, seed, ties)
    ad = _adapters(M, L, seed)
    rt = ml.route(torch.from_numpy(ad).cuda(), k, L, logits_in=lg.cuda(), want_logits=True)
    torch.cuda.synchronize()
    ids, w, sp, so = oracle_routing_from_logits(lg, ad.astype(np.int64), E, k, L)
    assert np.array_equal(rt["topk_ids"].cpu().numpy(), ids)
    np.testing.assert_allclose(rt["topk_w"].cpu().numpy(), w, rtol=0, atol=1e-6)
    assert np.array_equal(rt["sorted_pairs"].cpu().numpy(), sp)
    assert np.array_equal(rt["seg_offsets"].cpu().numpy(), so)
    assert np.array_equal(rt["logits"].cpu().numpy(), lg.numpy())   # logits_in passed through
    ml.check_status(rt["workspace"])


@pytest.mark.parametrize("M,E,k,L", [(1, 8, 2, 2), (2, 4, 4, 1), (37, 16, 4, 3), (64, 64, 8, 8),
                                     (257, 128, 8, 16), (4096, 128, 8, 16), (64, 128, 8, 32),
                                     (300, 256, 8, 64), (50, 256, 1, 0), (33, 5, 5, 0)])
def test_route_exact_against_oracle(M, E, k, L):
    _check_exact(M, E, k, L, seed=M * 7 + E)


@pytest.mark.parametrize("M,E,k,L", [(64, 16, 8, 4), (500, 32, 4, 2)])
def test_route_exact_with_ties(M, E, k, L):
    _check_exact(M, E, k, L, seed=99, ties=True)


def test_route_m0_zero_offsets():
    lg = torch.zeros((0, 8), device="cuda")
    rt = ml.route(torch.zeros(0, dtype=torch.int32, device="cuda"), 2, 3, logits_in=lg)
    torch.cuda.synchronize()
    assert rt["seg_offsets"].cpu().numpy().tolist() == [0] * (8 * 4 + 1)


def test_route_bad_adapter_id_sets_device_status():
    lg = _logits(16, 8, 5, False).cuda()
    ad = torch.zeros(16, dtype=torch.int32)
    ad[3] = 7  # L = 2: out of range
    rt = ml.route(ad.cuda(), 2, 2, logits_in=lg)
    with pytest.raises(ml.MoELoRAError) as ei:
        ml.check_status(rt["workspace"])
    assert ei.value.status == ml.ERR_DEVICE_CHECK
    # treated as no adapter: key a' = L
    ad_ok = ad.clone()
    ad_ok[3] = -1
    ids, w, sp, so = oracle_routing_from_logits(lg.cpu(), ad_ok.numpy().astype(np.int64), 8, 2, 2)
    assert np.array_equal(rt["sorted_pairs"].cpu().numpy(), sp)


@pytest.mark.parametrize("shape,M", [(synth.MOE_DECODE_BF16, 64), (synth.MOE_PREFILL_BF16, 4096),
                                     (synth.MOE_DECODE_FP8, 64), (synth.MOE_DECODE_BF16, 1)])
def test_router_logits_from_x(shape, M):
    """Logits x W_r^T + b within fp32 accumulation error of the fp64 oracle; ids equal to
    the oracle's except where the oracle's own k-th/(k+1)-th gap is inside that error."""
    OW = MoEOracleWeights(shape)
    wr_cpu, bias_cpu = synth.moe_router(shape)
    x, ad = synth.moe_tokens(shape, M)
    rt = ml.route(ad.cuda(), shape.k, shape.L, x=x.cuda(), w_router=wr_cpu.cuda(),
                  bias=None if bias_cpu is None else bias_cpu.cuda(), want_logits=True)
    torch.cuda.synchronize()
    wr, bias = OW.router()
    lg = ref.router_logits(formats.to_f64(synth.bits(x), "bf16"), wr, bias)
    lg_gpu = rt["logits"].cpu().numpy().astype(np.float64)
    tol = 1e-4 * max(1.0, float(np.max(np.abs(lg))))
    assert float(np.max(np.abs(lg_gpu - lg))) <= tol
    ids, w = ref.route_topk(lg, shape.k)
    srt = -np.sort(-lg, axis=1)
    gap = srt[:, shape.k - 1] - srt[:, shape.k] if shape.k < shape.E else np.full(M, np.inf)
    clear = gap > 4 * tol
    gids = rt["topk_ids"].cpu().numpy()
    assert np.array_equal(np.sort(gids[clear], 1), np.sort(ids[clear], 1))
    assert clear.mean() >= 0.95


def test_route_deterministic():
    shape = synth.MOE_PREFILL_BF16
    lin = synth.moe_logits_in(shape, 4096).cuda()
    _, ad = synth.moe_tokens(shape, 4096)
    a = ml.route(ad.cuda(), shape.k, shape.L, logits_in=lin)
    b = ml.route(ad.cuda(), shape.k, shape.L, logits_in=lin)
    torch.cuda.synchronize()
    for key in ("topk_ids", "topk_w", "sorted_pairs", "seg_offsets"):
        assert torch.equal(a[key], b[key])


@pytest.mark.parametrize("M,E,k,L,H", [(1, 64, 8, 8, 2048), (64, 128, 8, 32, 7168), (128, 64, 8, 8, 512),
                                       (129, 64, 8, 8, 512), (40, 256, 4, 64, 264), (7, 5, 5, 0, 64),
                                       (300, 128, 8, 16, 1024), (260, 256, 4, 4, 264), (1000, 20, 2, 3, 136)])
def test_route_from_x_exact_on_gpu_logits(M, E, k, L, H):
    """All routing launches (one launch for M k <= 1024; above it SIMT logits for M < 256
    and tensor-core logits from M = 256, then top-k and sort kernels):
    ids, weights, pairs and offsets equal the oracle's routing of the GPU's own fp32
    logits; the logits themselves agree with the fp64 oracle within fp32 error."""
    g = np.random.default_rng(M * 31 + E)
    xb = torch.from_numpy(g.standard_normal((M, H), dtype=np.float32)).to(torch.bfloat16)
    wr = torch.from_numpy(g.standard_normal((E, H), dtype=np.float32) / np.sqrt(H)).to(torch.bfloat16)
    bias = torch.from_numpy(g.standard_normal(E).astype(np.float32) * np.float32(0.7))
    ad = _adapters(M, L, M + E)
    rt = ml.route(torch.from_numpy(ad).cuda(), k, L, x=xb.cuda(), w_router=wr.cuda(), bias=bias.cuda(),
                  want_logits=True)
    torch.cuda.synchronize()
    lg_gpu = rt["logits"].cpu()
    ids, w, sp, so = oracle_routing_from_logits(lg_gpu, ad.astype(np.int64), E, k, L)
    assert np.array_equal(rt["topk_ids"].cpu().numpy(), ids)
    np.testing.assert_allclose(rt["topk_w"].cpu().numpy(), w, rtol=0, atol=1e-6)
    assert np.array_equal(rt["sorted_pairs"].cpu().numpy(), sp)
    assert np.array_equal(rt["seg_offsets"].cpu().numpy(), so)
    x64 = formats.to_f64(synth.bits(xb), "bf16")
    w64 = formats.to_f64(synth.bits(wr), "bf16")
    lg = ref.router_logits(x64, w64, bias.numpy().astype(np.float64))
    tol = 1e-4 * max(1.0, float(np.max(np.abs(lg))))
    assert float(np.max(np.abs(lg_gpu.numpy().astype(np.float64) - lg))) <= tol
    ml.check_status(rt["workspace"])
    # a second call on the same workspace gives the same bits (phase-1 ticket re-armed)
    rt2 = ml.route(torch.from_numpy(ad).cuda(), k, L, x=xb.cuda(), w_router=wr.cuda(), bias=bias.cuda(),
                   want_logits=True, workspace=rt["workspace"])
    torch.cuda.synchronize()
    for key in ("logits", "topk_ids", "topk_w", "sorted_pairs", "seg_offsets"):
        assert torch.equal(rt[key], rt2[key])
