"""The seeded generators draw what the workload recipe says, deterministically."""
import numpy as np

import synth


def test_tiny_recipe():
    w = synth.CONFIGS["tiny"]
    x = synth.make_inputs(w)
    N, d, V, K = x.shape
    assert (N, d, V, K) == (256, 256, 4096, 16)
    assert x.hidden_bits.dtype == np.uint16 and x.W_bits.dtype == np.uint16
    assert x.topk_idx.dtype == np.int32 and x.topk_logit.dtype == np.float32
    assert all(len(set(r.tolist())) == K for r in x.topk_idx)
    assert x.topk_idx.min() >= 0 and x.topk_idx.max() < V
    assert np.all(np.diff(x.topk_logit, axis=1) <= 0)
    assert x.mask.sum() == N
    y = synth.make_inputs(w)
    assert np.array_equal(x.hidden_bits, y.hidden_bits) and np.array_equal(x.topk_idx, y.topk_idx)


def test_zipf_recipe_small_slice():
    w = synth.CONFIGS["small"]
    x = synth.make_inputs(w, N=512)
    N, d, V, K = x.shape
    assert K == 100
    assert all(len(set(r.tolist())) == K for r in x.topk_idx)
    assert x.topk_idx.min() >= 0 and x.topk_idx.max() < V
    assert int((x.mask == 0).sum()) == round(0.05 * 512)
    assert np.all(np.diff(x.topk_logit, axis=1) <= 0)
    # bf16 weights have the right spread
    from oracle.kl import bf16_bits_to_f64
    Wf = bf16_bits_to_f64(x.W_bits[:2048])
    assert 0.018 < Wf.std() < 0.022


def test_affine_map_is_a_bijection():
    rng = np.random.default_rng(0)
    V = 128256
    a, b = synth._affine_params(rng, 4, V)
    r = np.arange(V, dtype=np.int64)
    for ai, bi in zip(a, b):
        assert np.unique((ai * r + bi) % V).size == V


def test_sample_rows_sorted_unique():
    s = synth.sample_rows(1000, 64, seed=3)
    assert s.size == 64 and np.all(np.diff(s) > 0)
