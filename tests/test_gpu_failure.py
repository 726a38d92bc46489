"""Failure paths of moe_lora_forward, exercised without faulting or hanging the GPU.

1. A bounded device wait that runs out: a test-only switch (MOE_LORA_TEST_STALL=<ms>)
   makes CTA 0 of the gate_up GEMM skip the copies of its first pipeline stage and
   shortens every bounded wait to that many milliseconds.  The MMA thread's wait on the
   stage expires, the CTA raises its abort flag, drains its own copies and MMAs, frees
   TMEM and returns; moe_lora_check_status reports MOE_LORA_ERR_TIMEOUT, and the next
   call on the same context passes parity.
2. Segment offsets that are not monotone (two entries swapped, every value still inside
   [0, M k]): the work-list kernel flags MOE_LORA_ERR_DEVICE_CHECK, every kernel keeps
   its accesses inside the operands, and the next call passes parity.
"""
import pytest
import torch

import moe_lora_b200 as ml
from tests.gpu_cases import TOL_BF16, moe_weights_both, run_moe_case
from workloads import synth

pytestmark = pytest.mark.gpu

SHAPE = synth.MoEShape("fail_a", 240, E=8, k=2, H=384, I=192, L=3, r=16, no_adapter_frac=0.2)


@pytest.fixture(scope="module")
def weights():
    return moe_weights_both(SHAPE)


def _forward(weights, M, seg_fn=None):
    cpu, dev, _ = weights
    x, ad = synth.moe_tokens(SHAPE, M)
    rt = ml.route(ad.cuda(), SHAPE.k, SHAPE.L, logits_in=synth.moe_logits_in(SHAPE, M).cuda())
    if seg_fn is not None:
        rt = dict(rt, seg_offsets=seg_fn(rt["seg_offsets"].clone()))
    ws = ml.new_workspace(ml.workspace_size(ml.OP_FORWARD_BF16, M, SHAPE.H, SHAPE.I, SHAPE.E, SHAPE.k, SHAPE.L,
                                            SHAPE.r), "cuda")
    ml.forward(x.cuda(), rt, dev, k=SHAPE.k, L=SHAPE.L, workspace=ws)
    return ws


@pytest.mark.parametrize("where,M", [("delta", 37), ("tc", 300)])
def test_bounded_wait_runs_out_and_reports_timeout(weights, where, M, monkeypatch):
    monkeypatch.setenv("MOE_LORA_EXPAND", where)
    monkeypatch.setenv("MOE_LORA_TEST_STALL", "5")
    ws = _forward(weights, M)
    with pytest.raises(ml.MoELoRAError) as ei:
        ml.check_status(ws)
    assert ei.value.status == ml.ERR_TIMEOUT
    monkeypatch.delenv("MOE_LORA_TEST_STALL")
    ml.check_status(ws)  # the status word was cleared by the read
    res = run_moe_case(SHAPE, M, weights=weights)
    assert res["err"] <= TOL_BF16, res["err"]


def _swap_first_increase(so: torch.Tensor) -> torch.Tensor:
    """Swap the first pair of adjacent, different offsets: the CSR is no longer monotone
    but every value stays inside [0, M k]."""
    h = so.cpu()
    for i in range(h.numel() - 1):
        if h[i] < h[i + 1]:
            h[i], h[i + 1] = int(h[i + 1]), int(h[i])
            break
    return h.to(so.device)


@pytest.mark.parametrize("where,M", [("delta", 37), ("tc", 300)])
def test_forward_rejects_non_monotone_offsets(weights, where, M, monkeypatch):
    monkeypatch.setenv("MOE_LORA_EXPAND", where)
    ws = _forward(weights, M, seg_fn=_swap_first_increase)
    with pytest.raises(ml.MoELoRAError) as ei:
        ml.check_status(ws)
    assert ei.value.status == ml.ERR_DEVICE_CHECK
    res = run_moe_case(SHAPE, M, weights=weights)
    assert res["err"] <= TOL_BF16, res["err"]
