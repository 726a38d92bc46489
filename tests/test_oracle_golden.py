"""The oracle against hand-derived cases in tests/golden/hand_cases.json (CPU only)."""
import json
import math
import os

import numpy as np

from oracle import moe_lora_ref as ref

with open(os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")) as f:
    CASES = json.load(f)

_NS = {"exp": math.exp, "s": lambda v: v / (1.0 + math.exp(-v))}


def _ev(expr):
    return eval(expr, {"__builtins__": {}}, _NS)  # closed forms written in the fixture


def test_moe_k2_hand_case():
    c = CASES["moe_k2"]
    x = np.array(c["x"], dtype=np.float64)
    ad = np.array(c["adapter_ids"])
    lg = ref.router_logits(x, np.array(c["w_router"], dtype=np.float64))
    ids, w = ref.route_topk(lg, c["k"])
    assert ids.tolist() == c["expected_ids"]
    np.testing.assert_allclose(w.reshape(-1), [_ev(e) for e in c["expected_w"]], rtol=1e-14)
    wgu, wd = np.array(c["w_gu"], float), np.array(c["w_d"], float)
    ag, bg = np.array(c["a_gu"], float), np.array(c["b_gu"], float)
    adn, bd = np.array(c["a_d"], float), np.array(c["b_d"], float)
    y = ref.moe_lora_forward(x, ids, w, ad, c["I"], lambda e: (wgu[e], wd[e], 1.0, 1.0),
                             lambda a, e: (ag[a, e], bg[a, e], adn[a, e], bd[a, e]))
    exp_y = [[_ev(v) for v in row] for row in c["expected_y"]]
    np.testing.assert_allclose(y, exp_y, rtol=1e-14)


def test_routing_hand_case():
    c = CASES["routing"]
    ids, w = ref.route_topk(np.array(c["logits"]), c["k"])
    assert ids.tolist() == c["expected_ids"]
    np.testing.assert_allclose(w, c["expected_w"], rtol=1e-14)


def test_sort_hand_case():
    c = CASES["sort"]
    pairs, offs = ref.sort_pairs(np.array(c["topk_ids"]), np.array(c["adapter_ids"]), c["E"], c["L"])
    assert pairs.tolist() == c["expected_sorted_pairs"]
    assert offs.tolist() == c["expected_seg_offsets"]


def test_sgmv_hand_case():
    c = CASES["sgmv"]
    y = ref.dense_lora_forward(np.array(c["x"], float), np.array(c["w"], float),
                               np.array(c["a"], float), np.array(c["b"], float),
                               np.array(c["seg_offsets"]), np.array(c["seg_adapter"]))
    np.testing.assert_array_equal(y, np.array(c["expected_y"], float))
