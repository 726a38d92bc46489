"""Vectorised fp64 reference of the MoE + multi-LoRA layer and of dense SGMV.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Plain definitions written
out with numpy; the only library primitives are matrix products, argsort and
bincount.  Every input arrives already widened to fp64 from its stored precision
(``oracle.formats``); routing ids, permutations and offsets are int32.

What is computed (page citations per function):
  1. l[t,e]   = x_t . W_r[e] + bias[e]
  2. ids[t]   = the k experts of largest l[t,.], in descending order, ties to the
                lower expert index; w[t,j] = softmax over all E, then renormalised
                over the k selected (= softmax over the k selected logits)
  3. pairs p = t*k + j sorted stably by key (ids[t,j], a'(t)) with a' = a if a >= 0
     else L; seg_offsets = CSR over keys e*(L+1) + a'
  4. per pair: h  = s_gu * W_gu x_t + [a>=0] (x_t A_gu) B_gu            (2I values)
               act = silu(h[:I]) * h[I:]                                   (I values)
               o  = s_d * W_d act + [a>=0] (act A_d) B_d                   (H values)
  5. y_t = sum_j w[t,j] o_(t,j)
  6. SGMV: y_t = W x_t + [a(t)>=0] (x_t A_a(t)) B_a(t) over contiguous segments.

Storage conventions (same as the device ABI): W_gu [2I, H] and W_d [H, I] (rows
are output features); A stored transposed as [r, h_in]; B as [r, h_out]; the first
I rows of W_gu are the gate, the last I the up projection.
"""
from __future__ import annotations

import numpy as np


# ----------------------------------------------------------------------------- routing

def router_logits(x: np.ndarray, w_router: np.ndarray, bias: np.ndarray | None = None) -> np.ndarray:
    """l = x W_r^T (+ bias).  A router sends each token to its most relevant experts
    ([vLLM MoE-LoRA page], "Entendendo os Modelos MoE"); the logits are the plain
    linear router, with an optional per-expert bias that is part of the logits."""
    lg = x @ w_router.T
    if bias is not None:
        lg = lg + bias[None, :]
    return lg


def topk_order(logits: np.ndarray, k: int) -> np.ndarray:
    """The k largest logits per row, descending; equal logits go to the lower index.

    Top-k selection with k = 8 is the routing of the SageMaker MoE kernels page
    (first item).  The order is taken on the logits themselves (softmax is monotone)."""
    M, E = logits.shape
    order = np.argsort(-logits, axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def softmax(v: np.ndarray, axis: int = -1) -> np.ndarray:
    m = np.max(v, axis=axis, keepdims=True)
    ex = np.exp(v - m)
    return ex / np.sum(ex, axis=axis, keepdims=True)


def route_topk(logits: np.ndarray, k: int) -> tuple[np.ndarray, np.ndarray]:
    """ids [M,k] int32 and weights [M,k] fp64: softmax over all experts, take the
    top-k, renormalise over the selected ones so that each row sums to 1."""
    ids = topk_order(logits, k)
    p = softmax(logits, axis=1)
    sel = np.take_along_axis(p, ids.astype(np.int64), axis=1)
    return ids, sel / sel.sum(axis=1, keepdims=True)


def sort_keys(topk_ids: np.ndarray, adapter_ids: np.ndarray, L: int) -> np.ndarray:
    """Key of pair p = t*k + j: e*(L+1) + a', a' = a(t) if a(t) >= 0 else L.

    Expert routing and adapter selection are the two sparsity sources the MoE-LoRA
    kernel must combine ([vLLM MoE-LoRA page], "Implementação Técnica no vLLM")."""
    ap = np.where(adapter_ids >= 0, adapter_ids, L).astype(np.int64)
    return (topk_ids.astype(np.int64) * (L + 1) + ap[:, None]).reshape(-1)


def sort_pairs(topk_ids: np.ndarray, adapter_ids: np.ndarray, E: int, L: int):
    """Stable counting sort of the M*k pairs by (expert, adapter) key.

    Returns sorted_pairs int32 [M*k] (values p = t*k + j, ascending p within a key)
    and seg_offsets int32 [E*(L+1)+1], the CSR offsets of every key; tokens grouped
    into contiguous segments per adapter as in SGMV ([Punica review page], "提案手法")."""
    keys = sort_keys(topk_ids, adapter_ids, L)
    order = np.argsort(keys, kind="stable").astype(np.int32)
    counts = np.bincount(keys, minlength=E * (L + 1))
    offs = np.zeros(E * (L + 1) + 1, dtype=np.int64)
    np.cumsum(counts, out=offs[1:])
    return order, offs.astype(np.int32)


# ----------------------------------------------------------------------------- expert FFN

def silu(g: np.ndarray) -> np.ndarray:
    """silu(g) = g * sigmoid(g) = g / (1 + exp(-g))."""
    return g / (1.0 + np.exp(-g))


def lora_delta(v: np.ndarray, a_t: np.ndarray, b: np.ndarray) -> np.ndarray:
    """(v A) B for rows v [n, h_in], A stored as a_t [r, h_in], B as b [r, h_out].

    Shrink z = vA reduces h_in to r values, expand zB projects back to h_out
    ([vLLM MoE-LoRA page], "O Papel da Multi-LoRA")."""
    z = v @ a_t.T
    return z @ b


def swiglu(h: np.ndarray, I: int) -> np.ndarray:
    """act = silu(gate) * up with gate = h[:, :I] and up = h[:, I:]."""
    return silu(h[:, :I]) * h[:, I:]


def gate_up_lora_delta(v: np.ndarray, a_gu: np.ndarray, b_gu: np.ndarray, I: int) -> np.ndarray:
    """The gate_up adapter delta [n, 2I] in either layout.

    Fused (a_gu [r, H], b_gu [r, 2I]): one adapter on the fused projection.  Split
    (a_gu [2, r, H], b_gu [2, r, I]): the gate and the up projection each carry their own
    adapter, as every projection does on the vLLM MoE-LoRA page ("O Papel da
    Multi-LoRA": one A and one B per projection): gate columns (v A_g) B_g, up columns
    (v A_u) B_u."""
    if a_gu.ndim == 2:
        return lora_delta(v, a_gu, b_gu)
    return np.concatenate([lora_delta(v, a_gu[0], b_gu[0]), lora_delta(v, a_gu[1], b_gu[1])], axis=1)


def expert_ffn(xe: np.ndarray, adapters: np.ndarray, I: int, w_gu: np.ndarray, w_d: np.ndarray,
               s_gu: float, s_d: float, get_adapter, scale_gu: float = 1.0, scale_d: float = 1.0) -> np.ndarray:
    """One expert on its gathered rows xe [n, H] with per-row adapter id (-1 = none).

    gate_up expands H -> 2I, the gate is applied, down compresses I -> H
    ([vLLM MoE-LoRA page], "Entendendo os Modelos MoE"); each projection adds the
    row's own adapter delta, y = xW + xAB ("O Papel da Multi-LoRA"), with adapters
    owned per (adapter, expert) ("these operations per expert, per adapter").
    scale_gu / scale_d multiply each projection's delta (an alpha / r factor; 1 = the
    page's y = xW + xAB)."""
    h = s_gu * (xe @ w_gu.T)
    present = sorted(set(int(a) for a in adapters if a >= 0))
    lw = {a: get_adapter(a) for a in present}
    for a in present:
        rows = np.nonzero(adapters == a)[0]
        h[rows] += scale_gu * gate_up_lora_delta(xe[rows], lw[a][0], lw[a][1], I)
    act = swiglu(h, I)
    o = s_d * (act @ w_d.T)
    for a in present:
        rows = np.nonzero(adapters == a)[0]
        o[rows] += scale_d * lora_delta(act[rows], lw[a][2], lw[a][3])
    return o


def moe_lora_forward(x: np.ndarray, topk_ids: np.ndarray, topk_w: np.ndarray,
                     adapter_ids: np.ndarray, I: int, get_expert, get_adapter,
                     tokens: np.ndarray | None = None, scale_gu: float = 1.0,
                     scale_d: float = 1.0) -> np.ndarray:
    """y [M, H] (or only the rows listed in ``tokens``) in fp64.

    get_expert(e) -> (W_gu [2I,H], W_d [H,I], s_gu, s_d) widened to fp64;
    get_adapter(a, e) -> (A_gu [r,H], B_gu [r,2I], A_d [r,I], B_d [r,H]) fp64, or with
    separate gate and up adapters A_gu [2,r,H], B_gu [2,r,I] (gate_up_lora_delta).
    The selected experts' outputs are summed with the routing weights
    ([vLLM MoE-LoRA page], "Entendendo os Modelos MoE": outputs are aggregated)."""
    M, H = x.shape
    k = topk_ids.shape[1]
    rows_wanted = np.arange(M) if tokens is None else np.asarray(tokens)
    y = np.zeros((len(rows_wanted), H), dtype=np.float64)
    t_of = np.repeat(rows_wanted, k)
    j_of = np.tile(np.arange(k), len(rows_wanted))
    e_of = topk_ids[rows_wanted].reshape(-1)
    for e in np.unique(e_of):
        sel = np.nonzero(e_of == e)[0]
        t = t_of[sel]
        w_gu, w_d, s_gu, s_d = get_expert(int(e))
        o = expert_ffn(x[t], adapter_ids[t], I, w_gu, w_d, s_gu, s_d,
                       lambda a, e=int(e): get_adapter(a, e), scale_gu, scale_d)
        y[sel // k] += topk_w[t, j_of[sel]][:, None] * o
    return y


# ----------------------------------------------------------------------------- SGMV

def sgmv_shrink(x: np.ndarray, lora_a: np.ndarray, seg_offsets, seg_adapter) -> np.ndarray:
    """z_t = x_t A_a(t)^T per segment (segmented gather, [Punica review page], "提案手法");
    rows of segments with adapter -1 are zero."""
    T = x.shape[0]
    r = lora_a.shape[1]
    z = np.zeros((T, r), dtype=np.float64)
    for s in range(len(seg_adapter)):
        a = int(seg_adapter[s])
        lo, hi = int(seg_offsets[s]), int(seg_offsets[s + 1])
        if a >= 0 and hi > lo:
            z[lo:hi] = x[lo:hi] @ lora_a[a].T
    return z


def sgmv_expand(z: np.ndarray, lora_b: np.ndarray, seg_offsets, seg_adapter, h_out: int) -> np.ndarray:
    """delta_t = z_t B_a(t) per segment; zero for adapter -1."""
    T = z.shape[0]
    d = np.zeros((T, h_out), dtype=np.float64)
    for s in range(len(seg_adapter)):
        a = int(seg_adapter[s])
        lo, hi = int(seg_offsets[s]), int(seg_offsets[s + 1])
        if a >= 0 and hi > lo:
            d[lo:hi] = z[lo:hi] @ lora_b[a]
    return d


def dense_lora_forward(x, w, lora_a, lora_b, seg_offsets, seg_adapter) -> np.ndarray:
    """y = x W + (x A) B with W stored [h_out, h_in] ([vLLM MoE-LoRA page],
    "O Papel da Multi-LoRA"; batched over adapters by SGMV, [Punica review page])."""
    z = sgmv_shrink(x, lora_a, seg_offsets, seg_adapter)
    return x @ w.T + sgmv_expand(z, lora_b, seg_offsets, seg_adapter, w.shape[0])
