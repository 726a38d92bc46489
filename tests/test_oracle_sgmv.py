"""Pins for the oracle's segmented SGMV shrink/expand and dense LoRA layer (CPU only)."""
import numpy as np
import pytest

from oracle import brute
from oracle import moe_lora_ref as ref
from tests.oracle_inputs import dense_f64
from workloads import synth

SMALL = synth.DenseShape("dense_small", 110, T=11, h_in=10, h_out=7, L=3, r=2,
                         dtype="f32", no_adapter_frac=0.25)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_dense_matches_brute_per_token(dtype):
    s = SMALL.with_(dtype=dtype)
    d = dense_f64(s)
    y = ref.dense_lora_forward(d["x64"], d["w64"], d["a64"], d["b64"], d["offs"].numpy(),
                               d["segs"].numpy())
    yb = brute.dense_lora(d["x64"].tolist(), d["w64"].tolist(), d["a64"].tolist(),
                          d["b64"].tolist(), d["tok_a"].tolist())
    np.testing.assert_allclose(y, np.array(yb), rtol=1e-12, atol=1e-13)


def test_segmentation_and_token_order_do_not_change_results():
    """Batching distinct adapters as segments gives the same per-token results as any
    other grouping ([Punica review page], "主な発見": same vs different models)."""
    s = SMALL.with_(no_adapter_frac=0.0)
    d = dense_f64(s)
    x, A, B, W = d["x64"], d["a64"], d["b64"], d["w64"]
    tok_a = d["tok_a"].numpy()
    y = ref.dense_lora_forward(x, W, A, B, d["offs"].numpy(), d["segs"].numpy())
    g = np.random.default_rng(5)
    perm = g.permutation(len(tok_a))
    # one segment per token, in a shuffled order
    offs1 = np.arange(len(tok_a) + 1)
    y1 = ref.dense_lora_forward(x[perm], W, A, B, offs1, tok_a[perm])
    np.testing.assert_allclose(y1, y[perm], rtol=1e-13, atol=1e-14)


def test_single_adapter_equals_merged_weights():
    s = SMALL.with_(no_adapter_frac=0.0)
    d = dense_f64(s)
    x, A, B, W = d["x64"], d["a64"], d["b64"], d["w64"]
    T = x.shape[0]
    y = ref.dense_lora_forward(x, W, A, B, np.array([0, T]), np.array([2]))
    wm = W + (A[2].T @ B[2]).T
    np.testing.assert_allclose(y, x @ wm.T, rtol=1e-12, atol=1e-13)


def test_no_adapter_segment_is_base_only():
    s = SMALL
    d = dense_f64(s)
    x, A, B, W = d["x64"], d["a64"], d["b64"], d["w64"]
    T = x.shape[0]
    y = ref.dense_lora_forward(x, W, A, B, np.array([0, T]), np.array([-1]))
    np.testing.assert_array_equal(y, x @ W.T)


def test_shrink_expand_shapes_and_zero_rows():
    s = SMALL
    d = dense_f64(s)
    z = ref.sgmv_shrink(d["x64"], d["a64"], d["offs"].numpy(), d["segs"].numpy())
    assert z.shape == (s.T, s.r)
    none_rows = d["tok_a"].numpy() < 0
    assert np.all(z[none_rows] == 0)
    dl = ref.sgmv_expand(z, d["b64"], d["offs"].numpy(), d["segs"].numpy(), s.h_out)
    assert dl.shape == (s.T, s.h_out) and np.all(dl[none_rows] == 0)
