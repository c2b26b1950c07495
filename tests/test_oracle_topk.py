"""Pins of the teacher top-K oracle: brute force by Python sorting, exact ties,
and the selection invariant."""
import numpy as np

import synth
from oracle import kl as O
from oracle import topk as T


def test_brute_force_small():
    x = synth.custom_inputs(5, 6, 23, 1, seed=71, w_std=0.5)
    H = O.bf16_bits_to_f64(x.hidden_bits).tolist()
    W = O.bf16_bits_to_f64(x.W_bits).tolist()
    idx, val = T.teacher_topk(x.hidden_bits, x.W_bits, 7)
    for n in range(5):
        z = [sum(H[n][j] * W[v][j] for j in range(6)) for v in range(23)]
        want = sorted(range(23), key=lambda v: (-z[v], v))[:7]
        assert idx[n].tolist() == want
        np.testing.assert_allclose(val[n], [z[v] for v in want], rtol=1e-14)


def test_ties_go_to_the_smaller_index():
    x = synth.custom_inputs(4, 8, 40, 1, seed=72, w_std=0.5)
    W = x.W_bits.copy()
    W[30] = W[3]          # vocabulary entries 3 and 30 get identical logits
    W[17] = W[3]
    idx, val = T.teacher_topk(x.hidden_bits, W, 40)
    for n in range(4):
        order = idx[n].tolist()
        assert order.index(3) < order.index(17) < order.index(30)
        assert np.all(np.diff(val[n]) <= 0)


def test_selection_invariant_and_full_sort():
    x = synth.custom_inputs(16, 16, 300, 1, seed=73, w_std=0.3)
    z = T.teacher_logits(x.hidden_bits, x.W_bits)
    idx, val = T.teacher_topk(x.hidden_bits, x.W_bits, 50, row_chunk=5)
    for n in range(16):
        rest = np.setdiff1d(np.arange(300), idx[n])
        assert val[n].min() >= z[n, rest].max()
        assert len(set(idx[n].tolist())) == 50
    full, _ = T.teacher_topk(x.hidden_bits, x.W_bits, 300)
    np.testing.assert_array_equal(full, np.argsort(-z, axis=1, kind="stable"))
