"""Teacher top-K cache producer on the GPU vs the plain-sort oracle.

The GPU's logits are fp32 sums of bf16 products, the oracle's exact fp64, so
two entries whose logits differ by less than the fp32 rounding of a dot
product may legitimately swap places.  The checks therefore compare what is
unique (the sorted list of the K largest logit values, within that rounding,
and the index set wherever no near-tie straddles the K-th place) and check
that the rest is valid (distinct in-range indices, descending order, each
reported logit equal to that index's logit).
"""
import numpy as np
import pytest
import torch

import output_head_kl_b200 as K
import synth
from oracle import kl as O
from oracle import topk as T
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


def _gpu_topk(x, Kc):
    dx = H.to_device(x)
    N, d = dx.hidden.shape
    V = dx.W.shape[0]
    ws = torch.empty(K.kdkl_teacher_topk_workspace_bytes(N, d, V, Kc), dtype=torch.uint8, device="cuda")
    idx = torch.full((N, Kc), -7, dtype=torch.int32, device="cuda")
    val = torch.full((N, Kc), float("nan"), dtype=torch.float32, device="cuda")
    K.kdkl_teacher_topk(dx.hidden, dx.W, Kc, idx, val, ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy().astype(np.int64), val.cpu().numpy().astype(np.float64)


def _check_rows(x, gi, gv, rows, Kc):
    z = T.teacher_logits(x.hidden_bits, x.W_bits, rows)
    oi, ov = T.topk_from_logits(z, Kc)
    d = x.hidden_bits.shape[1]
    H64 = O.bf16_bits_to_f64(x.hidden_bits[rows])
    W64 = O.bf16_bits_to_f64(x.W_bits)
    exact_rows = 0
    for r in range(len(rows)):
        idx = gi[r]
        V = W64.shape[0]
        assert idx.min() >= 0 and idx.max() < V and len(set(idx.tolist())) == Kc
        assert np.all(np.diff(gv[r]) <= 0)
        # fp32 rounding bound of one dot product: d * 2^-24 * sum |h_j w_j|
        eps = 4 * d * 2.0 ** -24 * (np.abs(H64[r])[None, :] * np.abs(W64[idx])).sum(1).max() + 1e-30
        np.testing.assert_allclose(gv[r], z[r, idx], rtol=0, atol=eps)
        np.testing.assert_allclose(np.sort(z[r, idx])[::-1], ov[r], rtol=0, atol=2 * eps)
        # rows whose K-th and (K+1)-th logits are further apart than 8x this row's
        # observed fp32 error cannot swap entries: there the index sets must agree
        err = np.abs(gv[r] - z[r, idx]).max() + 1e-7
        srt = np.sort(z[r])[::-1]
        gap_ok = Kc == len(srt) or (srt[Kc - 1] - srt[Kc]) > 8 * err
        if gap_ok:
            assert set(idx.tolist()) == set(oi[r].tolist())
            exact_rows += 1
    return exact_rows


@pytest.mark.parametrize("Kc", [1, 16, 100, 128])
def test_topk_matches_oracle_ragged(Kc):
    x = synth.custom_inputs(700, 256, 5001, 1, seed=500 + Kc, w_std=0.05)
    gi, gv = _gpu_topk(x, Kc)
    rows = np.arange(700)
    exact = _check_rows(x, gi[rows], gv[rows], rows, Kc)
    assert exact >= 600


def test_topk_exact_ties_to_smaller_index():
    x = synth.custom_inputs(300, 128, 3000, 1, seed=510, w_std=0.05)
    W = x.W_bits.copy()
    for dst in (2500, 1300, 700):
        W[dst] = W[50]          # identical teacher logits for 50, 700, 1300, 2500
    x = synth.Inputs(x.hidden_bits, W, x.topk_idx, x.topk_logit, x.mask, x.tau)
    gi, gv = _gpu_topk(x, 128)
    for r in range(300):
        pos = {v: i for i, v in enumerate(gi[r].tolist())}
        present = [v for v in (50, 700, 1300, 2500) if v in pos]
        assert [pos[v] for v in present] == sorted(pos[v] for v in present)
        if present:
            assert len(set(gv[r][[pos[v] for v in present]].tolist())) == 1


def test_produced_cache_feeds_the_loss():
    """Teacher -> top-K cache (GPU) -> student loss (GPU) vs the oracle on that cache."""
    teacher = synth.custom_inputs(512, 192, 4000, 1, seed=520, w_std=0.08)
    gi, gv = _gpu_topk(teacher, 64)
    student = synth.custom_inputs(512, 256, 4000, 1, seed=521, mask_frac=0.05, w_std=0.05)
    x = synth.Inputs(student.hidden_bits, student.W_bits, gi.astype(np.int32), gv.astype(np.float32),
                     student.mask, 1.0)
    g = H.run_gpu(H.to_device(x), chunk_tokens=256)
    r = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, 1.0)
    assert g.flags == 0 and r.flags == 0
    H.assert_loss(g.loss, r.loss)
    H.assert_lse(g.lse, r.lse)
    H.assert_grad(g.dH, r.dH, "dHidden")
    H.assert_grad(g.dW, r.dW, "dW")


def test_topk_fullsize_sampled():
    """8B-class teacher head (d=4096, V=128256), K=100, 8192 tokens; 48 sampled rows."""
    w = synth.CONFIGS["8b"]
    x = synth.make_inputs(w, N=8192)
    gi, gv = _gpu_topk(x, 100)
    rows = synth.sample_rows(8192, 48, seed=530)
    exact = _check_rows(x, gi[rows], gv[rows], rows, 100)
    assert exact >= 24


def test_topk_long_vocabulary_splits():
    """38 row blocks of 256 at d = 64 over V = 60000 (235 column tiles): the planner keeps a
    single vocabulary split (38 units already fill a wave as well as 76 would), so each row's
    heap indices, kept relative to the split's first column, run past 32767."""
    N = 38 * 256
    x = synth.custom_inputs(N, 64, 60000, 1, seed=540, w_std=0.3)
    gi, gv = _gpu_topk(x, 100)
    assert gi.max() > 50000
    rows = synth.sample_rows(N, 64, seed=541)
    exact = _check_rows(x, gi[rows], gv[rows], rows, 100)
    assert exact >= 48
