"""moe_lora_route_noalloc: routing for callers that cannot allocate device memory.

Such callers (a plugin or custom-op interface that hands over only input and output
buffers) cannot pass a workspace, and may not call cudaMalloc themselves because it
can synchronise the device, is not allowed during stream capture, or breaks a memory
budget planned in advance.  The entry point keeps its scratch in a fixed array inside
the library.  These tests call it through the C ABI and compare it with moe_lora_route
(which takes a caller-allocated workspace) on two calls in a row, with different sizes,
so that the second call runs on scratch the first one left behind.

The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import moe_lora_b200 as ml
from workloads import synth

pytestmark = pytest.mark.gpu

_P, _I = ctypes.c_void_p, ctypes.c_int


def _fn():
    f = ml.lib().moe_lora_route_noalloc
    f.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]
    f.restype = _I
    return f


def _call_noalloc(adapter_ids, k, L, E, *, x=None, w_router=None, bias=None, logits_in=None):
    M = adapter_ids.shape[0]
    H = 0 if x is None else x.shape[1]
    dev = adapter_ids.device
    out = {"topk_ids": torch.full((M, k), -7, dtype=torch.int32, device=dev),
           "topk_w": torch.full((M, k), -7.0, dtype=torch.float32, device=dev),
           "sorted_pairs": torch.full((M * k,), -7, dtype=torch.int32, device=dev),
           "seg_offsets": torch.full((E * (L + 1) + 1,), -7, dtype=torch.int32, device=dev)}
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    st = _fn()(p(x), p(w_router), p(bias), p(logits_in), p(adapter_ids), M, H, E, k, L, None,
               p(out["topk_ids"]), p(out["topk_w"]), p(out["sorted_pairs"]), p(out["seg_offsets"]),
               torch.cuda.current_stream().cuda_stream)
    assert st == ml.OK, ml.lib().moe_lora_last_error()
    return out


def _same(a, b):
    assert torch.equal(a["topk_ids"], b["topk_ids"])
    assert torch.equal(a["sorted_pairs"], b["sorted_pairs"])
    assert torch.equal(a["seg_offsets"], b["seg_offsets"])
    np.testing.assert_allclose(a["topk_w"].cpu().numpy(), b["topk_w"].cpu().numpy(), rtol=0, atol=1e-6)


def test_noalloc_route_matches_workspace_route_two_calls_in_a_row():
    # call 1: router logits computed from x into the scratch (no logits_out), bias, E=128
    s1 = synth.MOE_DECODE_FP8
    x1, a1 = synth.moe_tokens(s1, 64)
    wr1, b1 = synth.moe_router(s1)
    x1, a1, wr1, b1 = x1.cuda(), a1.cuda(), wr1.cuda(), b1.cuda()
    got1 = _call_noalloc(a1, s1.k, s1.L, s1.E, x=x1, w_router=wr1, bias=b1)
    ref1 = ml.route(a1, s1.k, s1.L, x=x1, w_router=wr1, bias=b1)
    # call 2: a different size on the scratch call 1 left behind (given logits, E=64, L=8)
    s2 = synth.MOE_DECODE_BF16
    _, a2 = synth.moe_tokens(s2, 300, batch=3)
    lin2 = synth.moe_logits_in(s2, 300).cuda()
    a2 = a2.cuda()
    a2[::7] = -1
    got2 = _call_noalloc(a2, s2.k, s2.L, s2.E, logits_in=lin2)
    ref2 = ml.route(a2, s2.k, s2.L, logits_in=lin2)
    torch.cuda.synchronize()
    _same(got1, ref1)
    _same(got2, ref2)
    # and once more with call 1's inputs: stale key counts from call 2 must not leak in
    got3 = _call_noalloc(a1, s1.k, s1.L, s1.E, x=x1, w_router=wr1, bias=b1)
    torch.cuda.synchronize()
    _same(got3, ref1)


def test_noalloc_route_largest_scratch_case():
    """The limits themselves: M = 1024, E = 256, k = 8, L = 64, logits computed from x on
    the tensor cores into the scratch (M * E fp32 values, the largest region), twice."""
    s = synth.MoEShape("noalloc_max", 230, E=256, k=8, H=512, I=64, L=64, r=16, bias=True)
    x, a = synth.moe_tokens(s, 1024)
    wr, b = synth.moe_router(s)
    x, a, wr, b = x.cuda(), a.cuda(), wr.cuda(), b.cuda()
    a[::5] = -1
    ref = ml.route(a, s.k, s.L, x=x, w_router=wr, bias=b)
    for _ in range(2):
        got = _call_noalloc(a, s.k, s.L, s.E, x=x, w_router=wr, bias=b)
        torch.cuda.synchronize()
        _same(got, ref)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    f = _fn()
    fake = 0x7F0000000000
    st = f(None, None, None, fake, fake, 1025, 0, 64, 8, 8, None, fake, fake, fake, fake, None)
    assert st == ml.ERR_UNSUPPORTED
    assert b"M <= 1024" in ml.lib().moe_lora_last_error()
    st = f(None, None, None, fake, fake, 16, 0, 257, 8, 8, None, fake, fake, fake, fake, None)
    assert st == ml.ERR_UNSUPPORTED
    st = f(None, None, None, fake, fake, 16, 0, 8, 9, 8, None, fake, fake, fake, fake, None)  # k > E
    assert st == ml.ERR_UNSUPPORTED
    st = f(None, None, None, fake, fake, 16, 0, 64, 8, 65, None, fake, fake, fake, fake, None)  # L = 65
    assert st == ml.ERR_UNSUPPORTED
