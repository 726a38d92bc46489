"""Glue between the seeded generator and the oracle (test side only).

Turns the generator's stored-precision tensors into the fp64 arrays the oracle
takes, regenerating expert and adapter slices lazily so that full-size workloads
never materialise their whole fp64 weight set.
"""
from __future__ import annotations

import functools

import numpy as np

from oracle import formats
from workloads import synth


class MoEOracleWeights:
    """fp64 views of one MoE workload's weights, regenerated per slice on demand."""

    def __init__(self, shape: synth.MoEShape, cache: bool = True):
        self.s = shape
        if cache:
            self.expert = functools.lru_cache(maxsize=None)(self._expert)
            self.adapter = functools.lru_cache(maxsize=None)(self._adapter)
        else:
            self.expert, self.adapter = self._expert, self._adapter

    def _expert(self, e: int):
        gu, d, sg, sd = synth.moe_expert(self.s, e)
        wdt = self.s.wdtype
        return (formats.to_f64(synth.bits(gu), wdt), formats.to_f64(synth.bits(d), wdt),
                float(sg), float(sd))

    def _adapter(self, a: int, e: int):
        return tuple(formats.to_f64(synth.bits(t), "bf16") for t in synth.moe_adapter(self.s, a, e))

    def router(self):
        wr, bias = synth.moe_router(self.s)
        return (formats.to_f64(synth.bits(wr), "bf16"),
                None if bias is None else bias.numpy().astype(np.float64))


def moe_tokens_f64(shape: synth.MoEShape, M: int):
    x, ids = synth.moe_tokens(shape, M)
    return x, ids, formats.to_f64(synth.bits(x), "bf16"), ids.numpy().astype(np.int64)


def dense_f64(shape: synth.DenseShape, T: int | None = None):
    x, tok_a, offs, segs = synth.dense_tokens(shape, T)
    w = synth.dense_weights(shape)
    dt = shape.dtype
    f = lambda t: formats.to_f64(synth.bits(t), dt)
    return dict(x=x, tok_a=tok_a, offs=offs, segs=segs, w=w,
                x64=f(x), w64=f(w["w"]), a64=f(w["a"]), b64=f(w["b"]))
