"""The C-ABI library without a GPU: it loads, exports every declared entry point,
sizes workspaces, and rejects bad arguments on the host before touching the device.

Every call below fails host-side validation, so nothing is ever launched (the fake
device addresses are never dereferenced)."""
import ctypes
import os
import re

import pytest

import moe_lora_b200 as ml
from moe_lora_b200 import _lib

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe_lora.h")
FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced
MIS = FAKE + 4          # misaligned


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_LORA_API\s+[\w\s\*]+?\b(\w+)\s*\(", txt)))


def test_library_loads_and_exports_every_declared_symbol():
    L = ml.lib()
    names = declared_symbols()
    assert len(names) >= 9
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(ml.EXPORTS)
    assert "sm_100a" in ml.version()


def test_workspace_sizes():
    # route: status + counts + per-token keys + logits
    assert ml.workspace_size(ml.OP_ROUTE, 64, 2048, 0, 64, 8, 8, 0) >= 256 + 64 * 9 * 4 + 64 * 4 + 64 * 64 * 4
    f = ml.workspace_size(ml.OP_FORWARD, 64, 2048, 1408, 64, 8, 8, 16)
    mk = 64 * 8
    assert f >= mk * 2048 * 2 + mk * 1408 * 2 + 2 * mk * 16 * 4 + mk * 4 + mk * 2048 * 4
    assert ml.workspace_size(ml.OP_FORWARD, 0, 2048, 1408, 64, 8, 8, 16) == 256
    fb = ml.workspace_size(ml.OP_FORWARD_BF16, 64, 2048, 1408, 64, 8, 8, 16)
    fe = ml.workspace_size(ml.OP_FORWARD_E4M3, 64, 2048, 1408, 64, 8, 8, 16)
    assert 0 < fb < fe == f   # e4m3 experts add the activation planes
    assert ml.workspace_size(ml.OP_SGMV_SHRINK) == 256
    assert ml.workspace_size(99) == 0
    assert ml.workspace_size(ml.OP_FORWARD, -1) == 0


def _fwd(**kw):
    a = dict(x=FAKE, M=4, H=64, I=64, E=4, k=2, L=2, r=16, topk_w=FAKE, sorted_pairs=FAKE,
             seg_offsets=FAKE, w_gu=FAKE, w_d=FAKE, wdt=ml.ML_BF16, scales=None, agu=FAKE, bgu=FAKE,
             ad=FAKE, bd=FAKE, fmt=None, y=FAKE, ws=FAKE, wsb=1 << 30)
    a.update(kw)
    return ml.lib().moe_lora_forward(a["x"], a["M"], a["H"], a["I"], a["E"], a["k"], a["L"], a["r"],
                                     a["topk_w"], a["sorted_pairs"], a["seg_offsets"], a["w_gu"], a["w_d"],
                                     a["wdt"], a["scales"], a["agu"], a["bgu"], a["ad"], a["bd"], a["fmt"],
                                     a["y"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(y=None), ml.ERR_INVALID_ARG),
    (dict(x=MIS), ml.ERR_INVALID_ARG),
    (dict(ws=None), ml.ERR_INVALID_ARG),
    (dict(wsb=100), ml.ERR_INVALID_ARG),
    (dict(k=5), ml.ERR_UNSUPPORTED),            # k > E
    (dict(E=300, k=2), ml.ERR_UNSUPPORTED),     # E > 256
    (dict(r=12), ml.ERR_UNSUPPORTED),           # rank outside the supported set
    (dict(r=256), ml.ERR_UNSUPPORTED),
    (dict(H=60), ml.ERR_UNSUPPORTED),           # not a multiple of 8
    (dict(L=65), ml.ERR_UNSUPPORTED),
    (dict(M=-1), ml.ERR_INVALID_ARG),
    (dict(wdt=7), ml.ERR_INVALID_ARG),
    (dict(agu=None), ml.ERR_INVALID_ARG),       # adapters present but A missing
    (dict(seg_offsets=MIS), ml.ERR_INVALID_ARG),
    (dict(fmt=ctypes.pointer(ml.AdapterFormat(2, 1.0, 1.0))), ml.ERR_INVALID_ARG),   # bad layout
    (dict(fmt=ctypes.pointer(ml.AdapterFormat(1, 1.0, 1.0)), r=128), ml.ERR_UNSUPPORTED),  # split: r <= 64
])
def test_forward_host_validation(kw, code):
    assert _fwd(**kw) == code
    assert ml.lib().moe_lora_last_error()


def test_forward_m0_is_ok_without_launch():
    assert _fwd(M=0, x=None, y=None, topk_w=None, sorted_pairs=None) == ml.OK


def _route(**kw):
    a = dict(x=FAKE, wr=FAKE, bias=None, lin=None, ad=FAKE, M=4, H=64, E=8, k=2, L=2, lout=None,
             ids=FAKE, w=FAKE, sp=FAKE, so=FAKE, ws=FAKE, wsb=1 << 30)
    a.update(kw)
    return ml.lib().moe_lora_route(a["x"], a["wr"], a["bias"], a["lin"], a["ad"], a["M"], a["H"], a["E"],
                                   a["k"], a["L"], a["lout"], a["ids"], a["w"], a["sp"], a["so"], a["ws"],
                                   a["wsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(so=None), ml.ERR_INVALID_ARG),
    (dict(ad=None), ml.ERR_INVALID_ARG),
    (dict(x=None), ml.ERR_INVALID_ARG),          # neither x nor logits_in
    (dict(k=9), ml.ERR_UNSUPPORTED),
    (dict(E=0), ml.ERR_INVALID_ARG),
    (dict(H=12), ml.ERR_UNSUPPORTED),
    (dict(wsb=8), ml.ERR_INVALID_ARG),
    (dict(M=(1 << 20), k=2), ml.ERR_UNSUPPORTED),
    (dict(bias=MIS), ml.ERR_INVALID_ARG),
])
def test_route_host_validation(kw, code):
    assert _route(**kw) == code


@pytest.mark.parametrize("fn", ["sgmv_shrink", "sgmv_expand"])
@pytest.mark.parametrize("kw,code", [
    (dict(r=24), ml.ERR_UNSUPPORTED),
    (dict(S=0), ml.ERR_INVALID_ARG),
    (dict(dt=ml.ML_E4M3), ml.ERR_INVALID_ARG),
    (dict(seg=None), ml.ERR_INVALID_ARG),
    (dict(h=100), ml.ERR_UNSUPPORTED),
    (dict(ws=None), ml.ERR_INVALID_ARG),
])
def test_sgmv_host_validation(fn, kw, code):
    a = dict(src=FAKE, w=FAKE, seg=FAKE, sad=FAKE, S=2, T=8, h=64, r=16, L=2, dt=ml.ML_BF16, out=FAKE,
             ws=FAKE, wsb=256)
    a.update(kw)
    f = getattr(ml.lib(), fn)
    assert f(a["src"], a["w"], a["seg"], a["sad"], a["S"], a["T"], a["h"], a["r"], a["L"], a["dt"], a["out"],
             a["ws"], a["wsb"], None) == code


@pytest.mark.parametrize("kw,code", [
    (dict(y=None), ml.ERR_INVALID_ARG),
    (dict(h_out=20), ml.ERR_UNSUPPORTED),
    (dict(r=3), ml.ERR_UNSUPPORTED),
    (dict(wsb=10), ml.ERR_INVALID_ARG),
])
def test_dense_host_validation(kw, code):
    a = dict(x=FAKE, w=FAKE, A=FAKE, B=FAKE, seg=FAKE, sad=FAKE, S=1, T=8, h_in=64, h_out=64, r=16, L=2,
             dt=ml.ML_BF16, y=FAKE, ws=FAKE, wsb=1 << 20)
    a.update(kw)
    assert ml.lib().dense_lora_forward(a["x"], a["w"], a["A"], a["B"], a["seg"], a["sad"], a["S"], a["T"],
                                       a["h_in"], a["h_out"], a["r"], a["L"], a["dt"], a["y"], a["ws"],
                                       a["wsb"], None) == code


def test_binding_refuses_host_tensors():
    import torch
    with pytest.raises(ValueError):
        _lib._ptr(torch.zeros(4))


def test_product_package_does_not_import_oracle():
    import sys
    import subprocess
    code = ("import sys, moe_lora_b200, moe_lora_b200.build, moe_lora_b200._lib; "
            "bad = [m for m in sys.modules if m == 'oracle' or m.startswith('oracle.')]; "
            "assert not bad, bad")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    subprocess.run([sys.executable, "-c", code], check=True, cwd=root)
