"""GPU parity of sgmv_shrink / sgmv_expand / dense_lora_forward against the oracle."""
import numpy as np
import pytest
import torch

import moe_lora_b200 as ml
from oracle import moe_lora_ref as ref
from tests.gpu_cases import TOL_BF16, rel_err
from tests.oracle_inputs import dense_f64
from workloads import synth

pytestmark = pytest.mark.gpu

CASES = [
    synth.SGMV_F32,
    synth.SGMV_F32.with_(name="f32_ragged", wid=300, T=37, h_in=520, h_out=392, L=3, r=8,
                         no_adapter_frac=0.3),
    synth.DENSE_DECODE_BF16,
    synth.DENSE_DECODE_BF16.with_(name="bf16_ragged", wid=301, T=37, h_in=520, h_out=392, L=5, r=32,
                                  no_adapter_frac=0.3),
    synth.DENSE_DECODE_BF16.with_(name="bf16_prefillish", wid=302, T=300, h_in=256, h_out=640, L=4,
                                  r=64, adapter_dist="uniform"),
    synth.DENSE_DECODE_BF16.with_(name="bf16_r128", wid=303, T=9, h_in=128, h_out=136, L=2, r=128),
    # r h_in >= 65536: split LoRA shrink with a ragged last K slice
    synth.DENSE_DECODE_BF16.with_(name="bf16_split", wid=304, T=45, h_in=2056, h_out=264, L=5, r=32,
                                  no_adapter_frac=0.2),
    # 8 weight tiles, the last one 104 rows, K = 4096
    synth.DENSE_DECODE_BF16.with_(name="bf16_k4096_ragged_m", wid=306, T=50, h_in=4096, h_out=1000, L=6, r=16,
                                  no_adapter_frac=0.2),
    # two token chunks (256 + a ragged 44) of 5 weight tiles each
    synth.DENSE_DECODE_BF16.with_(name="bf16_two_chunks", wid=307, T=300, h_in=2048, h_out=640, L=4,
                                  r=32),
]


def _dev(d):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


@pytest.mark.parametrize("s", CASES, ids=lambda s: s.name)
def test_sgmv_shrink_expand(s):
    d = dense_f64(s)
    x, offs, segs = d["x"].cuda(), d["offs"].cuda(), d["segs"].cuda()
    A, B = d["w"]["a"].cuda(), d["w"]["b"].cuda()
    z = ml.sgmv_shrink(x, A, offs, segs)
    torch.cuda.synchronize()
    z_ref = ref.sgmv_shrink(d["x64"], d["a64"], d["offs"].numpy(), d["segs"].numpy())
    tol = 1e-5 if s.dtype == "f32" else 1e-3
    assert rel_err(z, z_ref) <= tol
    # expand into a copy of the base output y0 = x W
    y0 = torch.zeros((s.T, s.h_out), dtype=x.dtype, device="cuda")
    z_in = torch.from_numpy(z_ref.astype(np.float32)).cuda()   # oracle z: tests expand alone
    ml.sgmv_expand(z_in, B, offs, segs, y0)
    torch.cuda.synchronize()
    d_ref = ref.sgmv_expand(z_ref.astype(np.float32).astype(np.float64), d["b64"], d["offs"].numpy(),
                            d["segs"].numpy(), s.h_out)
    assert rel_err(y0, d_ref) <= (1e-5 if s.dtype == "f32" else 1e-2)


@pytest.mark.parametrize("T", [5, 33, 64])
def test_dense_n64_tile(T, monkeypatch):
    """The dense projection's N tile of 64 with the SIMT LoRA kernel's fp32 delta added in
    the epilogue: tiny, ragged and full token counts, a ragged last weight tile and a K
    that ends inside a block."""
    monkeypatch.setenv("MOE_LORA_FORCE_BN", "64")
    monkeypatch.setenv("MOE_LORA_EXPAND", "delta")
    s = synth.DENSE_DECODE_BF16.with_(name="bf16_n64", wid=309, T=T, h_in=1000, h_out=1000, L=5, r=16,
                                      no_adapter_frac=0.2)
    d = dense_f64(s)
    y = ml.dense_lora_forward(d["x"].cuda(), d["w"]["w"].cuda(), d["w"]["a"].cuda(), d["w"]["b"].cuda(),
                              d["offs"].cuda(), d["segs"].cuda())
    torch.cuda.synchronize()
    y_ref = ref.dense_lora_forward(d["x64"], d["w64"], d["a64"], d["b64"], d["offs"].numpy(),
                                   d["segs"].numpy())
    err = rel_err(y, y_ref)
    assert err <= TOL_BF16, err


@pytest.mark.parametrize("where", ["delta", "tc"])
@pytest.mark.parametrize("s", CASES, ids=lambda s: s.name)
def test_dense_lora_forward(s, where, monkeypatch):
    """bf16: the expand inside the GEMM (extra MMA K steps), as the SIMT LoRA kernel's
    fp32 delta and as the tensor-core LoRA kernel's bf16 delta, each added by the GEMM
    epilogue (fp32 cases take the SIMT path)."""
    monkeypatch.setenv("MOE_LORA_EXPAND", where)
    d = dense_f64(s)
    y = ml.dense_lora_forward(d["x"].cuda(), d["w"]["w"].cuda(), d["w"]["a"].cuda(), d["w"]["b"].cuda(),
                              d["offs"].cuda(), d["segs"].cuda())
    torch.cuda.synchronize()
    y_ref = ref.dense_lora_forward(d["x64"], d["w64"], d["a64"], d["b64"], d["offs"].numpy(),
                                   d["segs"].numpy())
    err = rel_err(y, y_ref)
    assert err <= (1e-5 if s.dtype == "f32" else TOL_BF16), err


def test_dense_no_adapters_L0():
    s = synth.DENSE_DECODE_BF16.with_(name="L0", wid=304, T=20, h_in=256, h_out=256, L=0, r=16)
    d = dense_f64(s)
    y = ml.dense_lora_forward(d["x"].cuda(), d["w"]["w"].cuda(), d["w"]["a"].cuda(), d["w"]["b"].cuda(),
                              d["offs"].cuda(), d["segs"].cuda())
    torch.cuda.synchronize()
    assert rel_err(y, d["x64"] @ d["w64"].T) <= TOL_BF16


def test_sgmv_bad_adapter_sets_status():
    s = CASES[1]
    d = dense_f64(s)
    segs = d["segs"].clone()
    segs[0] = s.L + 3
    ws = ml.new_workspace(256, "cuda")
    ml.sgmv_shrink(d["x"].cuda(), d["w"]["a"].cuda(), d["offs"].cuda(), segs.cuda(), workspace=ws)
    with pytest.raises(ml.MoELoRAError) as ei:
        ml.check_status(ws)
    assert ei.value.status == ml.ERR_DEVICE_CHECK


@pytest.mark.parametrize("where", ["delta", "tc"])
def test_dense_many_segments(where, monkeypatch):
    """Tokens in arrival order (not grouped by adapter): every maximal run of one adapter
    is a segment, ~200 of them, interleaved with segments without an adapter, so the
    LoRA work list holds ~200 short items and one GEMM tile meets many of them."""
    monkeypatch.setenv("MOE_LORA_EXPAND", where)
    s = synth.DENSE_DECODE_BF16.with_(name="bf16_many_segs", wid=305, T=300, h_in=256, h_out=640, L=4,
                                      r=64, adapter_dist="uniform")
    d = dense_f64(s)
    ids = np.random.default_rng(305).integers(-1, s.L, size=s.T)
    starts = [0] + [i for i in range(1, s.T) if ids[i] != ids[i - 1]]
    offs = np.array(starts + [s.T], dtype=np.int32)
    segs = ids[starts].astype(np.int32)
    assert len(segs) > 150
    y = ml.dense_lora_forward(d["x"].cuda(), d["w"]["w"].cuda(), d["w"]["a"].cuda(), d["w"]["b"].cuda(),
                              torch.from_numpy(offs).cuda(), torch.from_numpy(segs).cuda())
    torch.cuda.synchronize()
    y_ref = ref.dense_lora_forward(d["x64"], d["w64"], d["a64"], d["b64"], offs, segs)
    err = rel_err(y, y_ref)
    assert err <= TOL_BF16, err



def test_dense_tc_lora_every_row_box(monkeypatch):
    """Segments whose lengths sit on both sides of every rows'-box height of the tensor-core
    LoRA kernel (16, 24, 32, 48, 64, 128 rows), and one longer than an item (two items)."""
    monkeypatch.setenv("MOE_LORA_EXPAND", "tc")
    lens = [1, 16, 17, 24, 25, 32, 33, 48, 49, 64, 65, 127, 128, 200]
    T = sum(lens)
    s = synth.DENSE_DECODE_BF16.with_(name="bf16_boxes", wid=308, T=T, h_in=256, h_out=384, L=4, r=32,
                                      adapter_dist="uniform")
    d = dense_f64(s)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    segs = (np.arange(len(lens)) % s.L).astype(np.int32)
    y = ml.dense_lora_forward(d["x"].cuda(), d["w"]["w"].cuda(), d["w"]["a"].cuda(), d["w"]["b"].cuda(),
                              torch.from_numpy(offs).cuda(), torch.from_numpy(segs).cuda())
    torch.cuda.synchronize()
    y_ref = ref.dense_lora_forward(d["x64"], d["w64"], d["a64"], d["b64"], offs, segs)
    err = rel_err(y, y_ref)
    assert err <= TOL_BF16, err
