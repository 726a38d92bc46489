"""Plant plausible mistakes in the oracle (CPU, monkeypatched) and check that a pin fails.

Each mutation is a mistake one could make writing the reference: a sign, a swapped
operand, a dropped term, a wrong tie-break or key order.  A pin that still passed
under one of them would not be pinning that part.
"""
import numpy as np
import pytest

from oracle import moe_lora_ref as ref
from tests import test_oracle_forward as tf
from tests import test_oracle_golden as tg
from tests import test_oracle_routing as tr
from tests import test_oracle_sgmv as ts


def _orig(name):
    return getattr(ref, name)


MUTATIONS = {
    "silu_sign": ("silu", lambda g: g / (1.0 + np.exp(g))),
    "gate_up_swapped": ("swiglu", lambda h, I: ref.silu(h[:, I:]) * h[:, :I]),
    "lora_dropped": ("lora_delta", lambda v, a, b: np.zeros((v.shape[0], b.shape[1]))),
    "lora_scaled_by_half": ("lora_delta", lambda v, a, b: (v @ a.T) @ b * 0.5),
    "tie_to_higher_index": ("topk_order",
                            lambda lg, k: np.argsort(-lg[:, ::-1], axis=1, kind="stable")[:, :k]
                            .__rsub__(lg.shape[1] - 1).astype(np.int32)),
    "no_renormalise": ("route_topk",
                       lambda lg, k: (ref.topk_order(lg, k),
                                      np.take_along_axis(ref.softmax(lg, 1),
                                                         ref.topk_order(lg, k).astype(np.int64), 1))),
    "no_adapter_key_not_last": ("sort_keys",
                                lambda ids, ad, L: (ids.astype(np.int64) * (L + 1)
                                                    + np.maximum(ad, 0)[:, None]).reshape(-1)),
}

PINS = {
    "silu_sign": [lambda: tf.test_forward_matches_brute_loops("bf16", False),
                  tg.test_moe_k2_hand_case],
    "gate_up_swapped": [lambda: tf.test_forward_matches_brute_loops("bf16", False),
                        tf.test_e1_k1_no_adapter_is_dense_swiglu_mlp_library],
    "lora_dropped": [lambda: tf.test_forward_matches_brute_loops("e4m3", True),
                     tg.test_moe_k2_hand_case],
    "lora_scaled_by_half": [tf.test_one_adapter_equals_merged_weights],
    "tie_to_higher_index": [tr.test_tie_goes_to_lower_expert_and_descending_order,
                            tg.test_routing_hand_case],
    "no_renormalise": [tg.test_routing_hand_case,
                       lambda: tr.test_topk_matches_brute_full_sort(7, 6, 3, False)],
    "no_adapter_key_not_last": [tg.test_sort_hand_case,
                                lambda: tr.test_sort_matches_brute_and_invariants(30, 8, 2, 3, 1)],
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(name, monkeypatch):
    attr, bad = MUTATIONS[name]
    monkeypatch.setattr(ref, attr, bad)
    for pin in PINS[name]:
        with pytest.raises(AssertionError):
            pin()


def test_sgmv_pins_catch_dropped_expand(monkeypatch):
    monkeypatch.setattr(ref, "sgmv_expand", lambda z, b, o, s, h: np.zeros((z.shape[0], h)))
    with pytest.raises(AssertionError):
        ts.test_dense_matches_brute_per_token("f32")
    with pytest.raises(AssertionError):
        tg.test_sgmv_hand_case()
