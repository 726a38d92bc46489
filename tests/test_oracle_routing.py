"""Pins for the oracle's routing (top-k, renormalised softmax) and (expert, adapter) sort."""
import numpy as np
import pytest
import scipy.special

from oracle import brute
from oracle import moe_lora_ref as ref


def _rand_logits(seed, M, E, ties=False):
    g = np.random.default_rng(seed)
    if ties:
        return g.integers(-3, 4, size=(M, E)).astype(np.float64)
    return g.standard_normal((M, E))


@pytest.mark.parametrize("M,E,k,ties", [(7, 6, 3, False), (9, 5, 2, True), (4, 8, 8, False),
                                        (5, 4, 1, True), (12, 16, 8, True)])
def test_topk_matches_brute_full_sort(M, E, k, ties):
    lg = _rand_logits(M * 100 + E, M, E, ties)
    ids, w = ref.route_topk(lg, k)
    for t in range(M):
        ranked = sorted(range(E), key=lambda e: (-lg[t, e], e))[:k]
        assert list(ids[t]) == ranked
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-15)


def test_brute_route_agrees_with_vectorised():
    g = np.random.default_rng(3)
    M, E, H, k = 6, 7, 5, 3
    x = g.standard_normal((M, H))
    wr = g.standard_normal((E, H))
    bias = g.standard_normal(E)
    lg = ref.router_logits(x, wr, bias)
    ids, w = ref.route_topk(lg, k)
    blg, bids, bw = brute.route(x.tolist(), wr.tolist(), bias.tolist(), k)
    np.testing.assert_allclose(lg, np.array(blg), rtol=1e-14, atol=1e-14)
    assert ids.tolist() == bids
    np.testing.assert_allclose(w, np.array(bw), rtol=1e-13)


def test_topk_equal_E_is_full_softmax_library():
    lg = _rand_logits(11, 6, 9)
    ids, w = ref.route_topk(lg, 9)
    full = scipy.special.softmax(lg, axis=1)
    np.testing.assert_allclose(np.take_along_axis(full, ids.astype(np.int64), 1), w, rtol=1e-14)


def test_k1_weight_is_one_and_argmax():
    lg = _rand_logits(12, 10, 5)
    ids, w = ref.route_topk(lg, 1)
    assert np.array_equal(ids[:, 0], np.argmax(lg, axis=1))
    assert np.all(w == 1.0)


def test_renormalised_softmax_equals_softmax_over_selected_logits():
    lg = _rand_logits(13, 8, 12)
    ids, w = ref.route_topk(lg, 4)
    sel = np.take_along_axis(lg, ids.astype(np.int64), 1)
    np.testing.assert_allclose(w, scipy.special.softmax(sel, axis=1), rtol=1e-13)


def test_tie_goes_to_lower_expert_and_descending_order():
    lg = np.array([[1.0, 1.0, 0.0, 1.0], [0.0, 2.0, 2.0, -1.0]])
    ids, w = ref.route_topk(lg, 3)
    assert ids.tolist() == [[0, 1, 3], [1, 2, 0]]
    np.testing.assert_allclose(w[0], [1 / 3] * 3, rtol=1e-15)


def _check_sort_invariants(ids, adapters, E, L, pairs, offs):
    M, k = ids.shape
    n = M * k
    assert sorted(pairs.tolist()) == list(range(n))
    ap = np.where(adapters >= 0, adapters, L)
    key = lambda p: int(ids[p // k, p % k]) * (L + 1) + int(ap[p // k])
    keys = [key(int(p)) for p in pairs]
    assert keys == sorted(keys)
    for i in range(1, n):
        if keys[i] == keys[i - 1]:
            assert pairs[i] // k > pairs[i - 1] // k       # ascending token within a key
    hist = np.zeros(E * (L + 1), dtype=np.int64)
    for kk in keys:
        hist[kk] += 1
    assert offs[0] == 0 and np.array_equal(np.diff(offs), hist)


@pytest.mark.parametrize("M,E,k,L,seed", [(9, 6, 3, 2, 0), (30, 8, 2, 3, 1), (1, 4, 4, 1, 2),
                                          (40, 16, 8, 4, 3), (0, 4, 2, 2, 4)])
def test_sort_matches_brute_and_invariants(M, E, k, L, seed):
    g = np.random.default_rng(seed)
    ids = np.stack([g.permutation(E)[:k] for _ in range(M)]).astype(np.int32) if M else \
        np.zeros((0, k), np.int32)
    adapters = g.integers(-1, L, size=M).astype(np.int32)
    pairs, offs = ref.sort_pairs(ids, adapters, E, L)
    bp, bo = brute.sort_pairs(ids.tolist(), adapters.tolist(), E, L)
    assert pairs.tolist() == bp
    assert offs.tolist() == bo
    assert len(offs) == E * (L + 1) + 1
    if M:
        _check_sort_invariants(ids, adapters, E, L, pairs, offs)
