"""Pins for the oracle's LoRA expert FFN and weighted combine (CPU only)."""
import numpy as np
import pytest
import torch

from oracle import brute, formats
from oracle import moe_lora_ref as ref
from tests.oracle_inputs import MoEOracleWeights, moe_tokens_f64
from workloads import synth

TINY = synth.MoEShape("tiny", 100, E=5, k=2, H=12, I=6, L=2, r=3, M_list=(7,),
                      no_adapter_frac=0.3)


def _route(shape, M):
    W = MoEOracleWeights(shape)
    _, _, x64, ad = moe_tokens_f64(shape, M)
    wr, bias = W.router()
    ids, w = ref.route_topk(ref.router_logits(x64, wr, bias), shape.k)
    return W, x64, ad, ids, w


def _brute_inputs(shape, W):
    experts = {e: tuple(v.tolist() if isinstance(v, np.ndarray) else v for v in W.expert(e))
               for e in range(shape.E)}
    lora = {(a, e): tuple(m.tolist() for m in W.adapter(a, e))
            for a in range(shape.L) for e in range(shape.E)}
    return experts, lora


@pytest.mark.parametrize("wdtype,bias", [("bf16", False), ("e4m3", True)])
def test_forward_matches_brute_loops(wdtype, bias):
    s = TINY.with_(wdtype=wdtype, bias=bias, wid=101 if bias else 100)
    M = 7
    W, x64, ad, ids, w = _route(s, M)
    y = ref.moe_lora_forward(x64, ids, w, ad, s.I, W.expert, W.adapter)
    experts, lora = _brute_inputs(s, W)
    yb = brute.moe_layer(x64.tolist(), ids.tolist(), w.tolist(), ad.tolist(), s.I, experts, lora)
    np.testing.assert_allclose(y, np.array(yb), rtol=1e-12, atol=1e-12)
    # the subset-of-tokens entry gives the same rows
    ys = ref.moe_lora_forward(x64, ids, w, ad, s.I, W.expert, W.adapter, tokens=[5, 0, 3])
    np.testing.assert_allclose(ys, y[[5, 0, 3]], rtol=1e-13, atol=1e-13)


def test_e1_k1_no_adapter_is_dense_swiglu_mlp_library():
    s = TINY.with_(E=1, k=1, no_adapter_frac=1.0)
    M = 9
    W, x64, ad, ids, w = _route(s, M)
    assert np.all(ids == 0) and np.all(w == 1.0) and np.all(ad == -1)
    y = ref.moe_lora_forward(x64, ids, w, ad, s.I, W.expert, W.adapter)
    wgu, wd, _, _ = W.expert(0)
    xt = torch.from_numpy(x64)
    g = torch.nn.functional.linear(xt, torch.from_numpy(wgu[: s.I]))
    u = torch.nn.functional.linear(xt, torch.from_numpy(wgu[s.I:]))
    yl = torch.nn.functional.linear(torch.nn.functional.silu(g) * u, torch.from_numpy(wd))
    np.testing.assert_allclose(y, yl.numpy(), rtol=1e-12, atol=1e-13)


class _Patched:
    """Adapter accessor with A and/or B replaced."""

    def __init__(self, W, zero_a=False, zero_b=False, scale_bd=1.0, zero_gu=False):
        self.W, self.za, self.zb, self.c, self.zgu = W, zero_a, zero_b, scale_bd, zero_gu

    def __call__(self, a, e):
        ag, bg, adn, bd = self.W.adapter(a, e)
        if self.za:
            ag, adn = ag * 0, adn * 0
        if self.zb:
            bg, bd = bg * 0, bd * 0
        if self.zgu:
            ag = ag * 0
        return ag, bg, adn, bd * self.c


def _base_only(W, x64, ids, w, s):
    return ref.moe_lora_forward(x64, ids, w, np.full(x64.shape[0], -1), s.I, W.expert, W.adapter)


def test_zero_b_or_zero_a_reduces_to_base():
    s = TINY.with_(no_adapter_frac=0.0)
    W, x64, ad, ids, w = _route(s, 8)
    base = _base_only(W, x64, ids, w, s)
    for kw in ({"zero_b": True}, {"zero_a": True}):
        y = ref.moe_lora_forward(x64, ids, w, ad, s.I, W.expert, _Patched(W, **kw))
        np.testing.assert_array_equal(y, base)
    y = ref.moe_lora_forward(x64, ids, w, ad, s.I, W.expert, W.adapter)
    assert np.max(np.abs(y - base)) > 1e-3 * np.max(np.abs(base))   # the delta is not negligible


def test_one_adapter_equals_merged_weights():
    s = TINY.with_(no_adapter_frac=0.0)
    W, x64, _, ids, w = _route(s, 8)
    ad = np.ones(8, dtype=np.int64)            # every token on adapter 1
    y = ref.moe_lora_forward(x64, ids, w, ad, s.I, W.expert, W.adapter)

    def merged(e):  # W' = W + (A^T B)^T per projection, built in fp64
        wgu, wd, sg, sd = W.expert(e)
        ag, bg, adn, bd = W.adapter(1, e)
        return wgu + (ag.T @ bg).T / sg, wd + (adn.T @ bd).T / sd, sg, sd

    ym = ref.moe_lora_forward(x64, ids, w, np.full(8, -1), s.I, merged, W.adapter)
    np.testing.assert_allclose(y, ym, rtol=1e-11, atol=1e-12)


def test_delta_linear_in_down_b():
    s = TINY.with_(no_adapter_frac=0.0)
    W, x64, ad, ids, w = _route(s, 8)
    y0 = ref.moe_lora_forward(x64, ids, w, ad, s.I, W.expert, _Patched(W, zero_gu=True, scale_bd=0.0))
    y1 = ref.moe_lora_forward(x64, ids, w, ad, s.I, W.expert, _Patched(W, zero_gu=True, scale_bd=1.0))
    y3 = ref.moe_lora_forward(x64, ids, w, ad, s.I, W.expert, _Patched(W, zero_gu=True, scale_bd=-2.5))
    np.testing.assert_allclose(y3 - y0, -2.5 * (y1 - y0), rtol=1e-11, atol=1e-13)


def test_weights_sum_to_one_on_workload_router():
    s = synth.MOE_DECODE_BF16
    W = MoEOracleWeights(s)
    _, _, x64, _ = moe_tokens_f64(s, 8)
    wr, bias = W.router()
    _, w = ref.route_topk(ref.router_logits(x64, wr, bias), s.k)
    np.testing.assert_allclose(w.sum(1), 1.0, atol=1e-15)


# ---------------------------------------------------------------- separate gate / up adapters
SPLIT = TINY.with_(name="tiny_split", wid=130, gu_split=True)


def test_split_gate_up_matches_brute_loops_with_scales():
    """Separate gate and up adapters and per-projection scales against scalar loops."""
    M = 7
    W, x64, ad, ids, w = _route(SPLIT, M)
    ag, bg, _, _ = W.adapter(0, 0)
    assert ag.shape == (2, SPLIT.r, SPLIT.H) and bg.shape == (2, SPLIT.r, SPLIT.I)
    y = ref.moe_lora_forward(x64, ids, w, ad, SPLIT.I, W.expert, W.adapter, scale_gu=0.5, scale_d=2.0)
    experts, lora = _brute_inputs(SPLIT, W)
    yb = brute.moe_layer(x64.tolist(), ids.tolist(), w.tolist(), ad.tolist(), SPLIT.I, experts, lora,
                         split=True, scale_gu=0.5, scale_d=2.0)
    np.testing.assert_allclose(y, np.array(yb), rtol=1e-12, atol=1e-12)


def test_split_gate_up_is_fused_rank_2r_with_block_diagonal_b():
    """Two adapters on the gate and up halves equal one fused adapter of rank 2r whose A
    stacks A_gate over A_up and whose B is block-diagonal (B_gate on the gate columns, B_up
    on the up columns) -- a different computation path through the fused layout."""
    M = 7
    W, x64, ad, ids, w = _route(SPLIT, M)
    I, r = SPLIT.I, SPLIT.r

    def fused(a, e):
        ag, bg, a_d, b_d = W.adapter(a, e)
        bf = np.zeros((2 * r, 2 * I))
        bf[:r, :I] = bg[0]
        bf[r:, I:] = bg[1]
        return np.concatenate([ag[0], ag[1]], axis=0), bf, a_d, b_d

    ys = ref.moe_lora_forward(x64, ids, w, ad, I, W.expert, W.adapter)
    yf = ref.moe_lora_forward(x64, ids, w, ad, I, W.expert, fused)
    np.testing.assert_allclose(ys, yf, rtol=1e-12, atol=1e-13)


def test_scale_equals_b_scaled():
    """A projection's scale multiplies its delta: the same as scaling that projection's B."""
    M = 7
    W, x64, ad, ids, w = _route(TINY, M)

    def scaled_b(a, e):
        ag, bg, a_d, b_d = W.adapter(a, e)
        return ag, 0.25 * bg, a_d, -3.0 * b_d

    y1 = ref.moe_lora_forward(x64, ids, w, ad, TINY.I, W.expert, W.adapter, scale_gu=0.25, scale_d=-3.0)
    y2 = ref.moe_lora_forward(x64, ids, w, ad, TINY.I, W.expert, scaled_b)
    np.testing.assert_allclose(y1, y2, rtol=1e-12, atol=1e-13)
