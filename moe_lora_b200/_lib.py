"""ctypes binding to libmoe_lora.so (argument marshalling only).

Every function here checks tensor placement and dtype, allocates the outputs and the
workspace with torch when the caller does not pass them, and calls the C ABI on the
current torch CUDA stream.  All arithmetic happens in the CUDA kernels of the library;
there is no fallback: a missing library or a non-OK status raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_lora.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_DEVICE_CHECK, ERR_TIMEOUT = range(6)
ML_F32, ML_BF16, ML_E4M3 = 0, 1, 2
OP_ROUTE, OP_FORWARD, OP_SGMV_SHRINK, OP_SGMV_EXPAND, OP_DENSE, OP_FORWARD_BF16, OP_FORWARD_E4M3 = range(7)

EXPORTS = ("moe_lora_route", "moe_lora_forward", "sgmv_shrink", "sgmv_expand", "dense_lora_forward",
           "moe_lora_workspace_size", "moe_lora_check_status", "moe_lora_last_error", "moe_lora_version",
           "moe_lora_profile_enable", "moe_lora_profile_read", "moe_lora_launch_count",
           "moe_lora_route_noalloc")
KERNEL_IDS = {"router_logits": 0, "topk": 1, "sort": 2, "shrink": 3, "gemm_gateup": 4, "gemm_down": 5,
              "combine": 6, "expand": 7, "dense_f32": 8, "gemm_dense": 9, "quant": 10,
              "lora": 11, "route": 12, "lora_down": 13,
              "gather": 14}


class AdapterFormat(ctypes.Structure):
    """moe_lora_adapter_format: gate_up adapter layout (0 fused, 1 separate gate and up
    adapters) and the per-projection scales of the LoRA deltas."""
    _fields_ = [("gate_up_split", ctypes.c_int), ("scale_gu", ctypes.c_float), ("scale_d", ctypes.c_float)]


class MoELoRAError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"moe_lora status {status}: {msg}")
        self.status = status


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m moe_lora_b200.build` "
                               "(there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        L.moe_lora_route.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _SZ, _P]
        L.moe_lora_forward.argtypes = [_P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _I, _P,
                                       _P, _P, _P, _P, ctypes.POINTER(AdapterFormat), _P, _P, _SZ, _P]
        L.sgmv_shrink.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _SZ, _P]
        L.sgmv_expand.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _SZ, _P]
        L.dense_lora_forward.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _SZ, _P]
        L.moe_lora_workspace_size.argtypes = [_I] * 8
        L.moe_lora_workspace_size.restype = _SZ
        L.moe_lora_check_status.argtypes = [_P, _P]
        L.moe_lora_last_error.restype = ctypes.c_char_p
        L.moe_lora_version.restype = ctypes.c_char_p
        L.moe_lora_profile_enable.argtypes = [_I]
        L.moe_lora_profile_enable.restype = _I
        L.moe_lora_profile_read.argtypes = [_I, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_I)]
        L.moe_lora_profile_read.restype = _I
        L.moe_lora_launch_count.restype = ctypes.c_longlong
        for name in ("moe_lora_route", "moe_lora_forward", "sgmv_shrink", "sgmv_expand",
                     "dense_lora_forward", "moe_lora_check_status"):
            getattr(L, name).restype = _I
        _lib = L
    return _lib


def _check(status: int):
    if status != OK:
        raise MoELoRAError(status, lib().moe_lora_last_error().decode())


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the library must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dt(t: torch.Tensor) -> int:
    return {torch.float32: ML_F32, torch.bfloat16: ML_BF16, torch.float8_e4m3fn: ML_E4M3}[t.dtype]


def workspace_size(op: int, M=0, H=0, I=0, E=0, k=0, L=0, r=0) -> int:
    return int(lib().moe_lora_workspace_size(op, M, H, I, E, k, L, r))


def new_workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def check_status(workspace: torch.Tensor, stream=None) -> None:
    _check(lib().moe_lora_check_status(_ptr(workspace), _stream(stream)))


def version() -> str:
    return lib().moe_lora_version().decode()


def profile_enable(max_launches: int) -> None:
    _check(lib().moe_lora_profile_enable(int(max_launches)))


def profile_read(kernel: str) -> tuple[float, int]:
    ms, n = ctypes.c_double(0.0), _I(0)
    _check(lib().moe_lora_profile_read(KERNEL_IDS[kernel], ctypes.byref(ms), ctypes.byref(n)))
    return ms.value, n.value


def launch_count() -> int:
    return int(lib().moe_lora_launch_count())


# ------------------------------------------------------------------------------ MoE layer

def route(adapter_ids: torch.Tensor, k: int, L: int, *, x=None, w_router=None, bias=None,
          logits_in=None, want_logits=False, out=None, workspace=None, stream=None) -> dict:
    """moe_lora_route.  Returns topk_ids [M,k], topk_w [M,k], sorted_pairs [M*k],
    seg_offsets [E*(L+1)+1] (and logits [M,E] when asked)."""
    dev = adapter_ids.device
    M = adapter_ids.shape[0]
    if logits_in is not None:
        E = logits_in.shape[1]
        H = 0
    else:
        E, H = w_router.shape
    o = out if out is not None else {}

    def buf(name, shape, dtype):
        t = o.get(name)
        return t if t is not None else torch.empty(shape, dtype=dtype, device=dev)

    ids = buf("topk_ids", (M, k), torch.int32)
    w = buf("topk_w", (M, k), torch.float32)
    sp = buf("sorted_pairs", (max(M * k, 1),), torch.int32)
    so = buf("seg_offsets", (E * (L + 1) + 1,), torch.int32)
    lg = buf("logits", (M, E), torch.float32) if want_logits else None
    if workspace is None:
        workspace = new_workspace(workspace_size(OP_ROUTE, M, H, 0, E, k, L, 0), dev)
    _check(lib().moe_lora_route(_ptr(x), _ptr(w_router), _ptr(bias), _ptr(logits_in), _ptr(adapter_ids),
                                M, H, E, k, L, _ptr(lg), _ptr(ids), _ptr(w), _ptr(sp), _ptr(so),
                                _ptr(workspace), workspace.numel(), _stream(stream)))
    res = {"topk_ids": ids, "topk_w": w, "sorted_pairs": sp[: M * k], "seg_offsets": so,
           "workspace": workspace}
    if want_logits:
        res["logits"] = lg
    return res


def forward(x: torch.Tensor, routing: dict, weights: dict, *, k: int, L: int, y=None, workspace=None,
            stream=None, scale_gu: float = 1.0, scale_d: float = 1.0) -> torch.Tensor:
    """moe_lora_forward.  weights: w_gu [E,2I,H], w_d [E,H,I] (bf16 or e4m3), scales [E,2]
    (e4m3 only), a_gu [L,E,r,H], b_gu [L,E,r,2I] -- or separate gate and up adapters
    a_gu [L,E,2,r,H], b_gu [L,E,2,r,I] -- a_d [L,E,r,I], b_d [L,E,r,H] (bf16).
    scale_gu / scale_d multiply each projection's delta."""
    M, H = x.shape
    E, twoI, _ = weights["w_gu"].shape
    I = twoI // 2
    split = L > 0 and weights["a_gu"].dim() == 5
    r = weights["a_gu"].shape[-2] if L > 0 else 0
    fmt = AdapterFormat(1 if split else 0, float(scale_gu), float(scale_d))
    wdt = _dt(weights["w_gu"])
    if y is None:
        y = torch.empty((M, H), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        op = OP_FORWARD_E4M3 if wdt == ML_E4M3 else OP_FORWARD_BF16
        workspace = new_workspace(workspace_size(op, M, H, I, E, k, L, r), x.device)
    scales = weights.get("scales") if wdt == ML_E4M3 else None
    _check(lib().moe_lora_forward(
        _ptr(x), M, H, I, E, k, L, r, _ptr(routing["topk_w"]), _ptr(routing["sorted_pairs"]),
        _ptr(routing["seg_offsets"]), _ptr(weights["w_gu"]), _ptr(weights["w_d"]), wdt, _ptr(scales),
        _ptr(weights["a_gu"]) if L else None, _ptr(weights["b_gu"]) if L else None,
        _ptr(weights["a_d"]) if L else None, _ptr(weights["b_d"]) if L else None, ctypes.byref(fmt),
        _ptr(y), _ptr(workspace), workspace.numel(), _stream(stream)))
    return y


# ------------------------------------------------------------------------------ SGMV / dense

def sgmv_shrink(x, lora_a, seg_offsets, seg_adapter, *, z=None, workspace=None, stream=None):
    T, h_in = x.shape
    L, r, _ = lora_a.shape
    if z is None:
        z = torch.empty((T, r), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = new_workspace(workspace_size(OP_SGMV_SHRINK), x.device)
    S = seg_adapter.shape[0]
    _check(lib().sgmv_shrink(_ptr(x), _ptr(lora_a) if L else None, _ptr(seg_offsets), _ptr(seg_adapter),
                             S, T, h_in, r, L, _dt(x), _ptr(z), _ptr(workspace), workspace.numel(),
                             _stream(stream)))
    return z


def sgmv_expand(z, lora_b, seg_offsets, seg_adapter, y, *, workspace=None, stream=None):
    T, r = z.shape
    L, _, h_out = lora_b.shape
    if workspace is None:
        workspace = new_workspace(workspace_size(OP_SGMV_EXPAND), z.device)
    S = seg_adapter.shape[0]
    _check(lib().sgmv_expand(_ptr(z), _ptr(lora_b) if L else None, _ptr(seg_offsets), _ptr(seg_adapter),
                             S, T, h_out, r, L, _dt(y), _ptr(y), _ptr(workspace), workspace.numel(),
                             _stream(stream)))
    return y


def dense_lora_forward(x, w, lora_a, lora_b, seg_offsets, seg_adapter, *, y=None, workspace=None,
                       stream=None):
    T, h_in = x.shape
    h_out = w.shape[0]
    L, r, _ = lora_a.shape
    if y is None:
        y = torch.empty((T, h_out), dtype=x.dtype, device=x.device)
    if workspace is None:
        workspace = new_workspace(workspace_size(OP_DENSE, T, h_in, h_out, 1, 1, L, r), x.device)
    S = seg_adapter.shape[0]
    _check(lib().dense_lora_forward(_ptr(x), _ptr(w), _ptr(lora_a) if L else None,
                                    _ptr(lora_b) if L else None, _ptr(seg_offsets), _ptr(seg_adapter),
                                    S, T, h_in, h_out, r, L, _dt(x), _ptr(y), _ptr(workspace),
                                    workspace.numel(), _stream(stream)))
    return y
