"""Pins of the oracle's loss-design variants (student temperature, Hinton's
tau^2 factor, a hard-label cross-entropy term sharing the student softmax).

Each variant is checked against torch library routines (``F.kl_div``,
``F.cross_entropy``) differentiated by autograd in float64, through the same
projection z = H W^T, and by finite differences of the oracle's own loss.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import synth
from oracle import kl as O


def _torch_reference(x, variant, labels):
    H = torch.tensor(O.bf16_bits_to_f64(x.hidden_bits), requires_grad=True)
    W = torch.tensor(O.bf16_bits_to_f64(x.W_bits), requires_grad=True)
    N, V = H.shape[0], W.shape[0]
    t = np.full((N, V), -np.inf)
    np.put_along_axis(t, x.topk_idx.astype(np.int64), x.topk_logit.astype(np.float64) / x.tau, axis=1)
    logq = F.log_softmax(torch.tensor(t), -1)
    m = torch.tensor(x.mask.astype(np.float64))
    zs = (H @ W.T) / variant.student_tau
    logp = F.log_softmax(zs, -1)
    q = logq.exp()
    kl_rows = torch.where(q > 0, q * (logq - logp), torch.zeros_like(q)).sum(-1)
    total = variant.gamma * (kl_rows * m).sum()
    if variant.ce_weight:
        lab = torch.tensor(np.where(x.mask > 0, labels, -100).astype(np.int64))
        total = total + variant.ce_weight * F.cross_entropy(zs, lab, ignore_index=-100, reduction="sum")
    ref = total / m.sum()
    ref.backward()
    return ref.item(), H.grad.numpy(), W.grad.numpy(), (zs.detach().logsumexp(-1)).numpy()


def _labels(x, seed, bad_frac=0.2):
    rng = np.random.default_rng(seed)
    N, V = x.hidden_bits.shape[0], x.W_bits.shape[0]
    lab = rng.integers(0, V, size=N).astype(np.int32)
    lab[rng.random(N) < bad_frac] = -100          # rows without a hard label
    return lab


@pytest.mark.parametrize("variant", [
    O.Variant(student_tau=2.0, kd_scale_tau_sq=True),                       # Hinton: both softened, x tau^2
    O.Variant(kd_weight=0.0, ce_weight=1.0),                                # hard labels only
    O.Variant(student_tau=1.5, kd_weight=0.6, ce_weight=0.4),               # mixture, shared softmax
    O.Variant(student_tau=0.5, kd_weight=0.3, kd_scale_tau_sq=True, ce_weight=2.0),
])
def test_variants_match_torch_autograd(variant):
    x = synth.custom_inputs(9, 12, 31, 6, seed=61, tau=2.0 if variant.kd_scale_tau_sq else 1.0,
                            mask_frac=0.2, w_std=0.4)
    lab = _labels(x, 62)
    r = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau, variant=variant, labels=lab)
    loss, dH, dW, lse = _torch_reference(x, variant, lab)
    assert r.loss == pytest.approx(loss, rel=1e-12)
    np.testing.assert_allclose(r.dH, dH, rtol=1e-9, atol=1e-15)
    np.testing.assert_allclose(r.dW, dW, rtol=1e-9, atol=1e-15)
    np.testing.assert_allclose(r.lse, lse, rtol=1e-13)


def test_default_variant_is_plain_kl():
    x = synth.custom_inputs(7, 8, 19, 5, seed=63, mask_frac=0.1, w_std=0.5)
    a = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, 1.0)
    b = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, 1.0,
                  variant=O.Variant(ce_weight=0.0), labels=_labels(x, 1))
    assert a.loss == b.loss
    np.testing.assert_array_equal(a.dW, b.dW)


def test_variant_finite_differences():
    v = O.Variant(student_tau=1.7, kd_weight=0.8, kd_scale_tau_sq=True, ce_weight=0.5)
    x = synth.custom_inputs(5, 6, 11, 4, seed=64, mask_frac=0.2, w_std=0.7)
    lab = _labels(x, 65)
    H0 = O.bf16_bits_to_f64(x.hidden_bits)
    W0 = O.bf16_bits_to_f64(x.W_bits)
    args = (x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau)
    r = O.kl_loss(*args, W_f64=W0, H_f64=H0, variant=v, labels=lab)
    h = 1e-6
    rng = np.random.default_rng(2)
    for _ in range(8):
        n, j = rng.integers(0, 5), rng.integers(0, 6)
        Hp, Hm = H0.copy(), H0.copy()
        Hp[n, j] += h
        Hm[n, j] -= h
        fd = (O.kl_loss(*args, W_f64=W0, H_f64=Hp, want_grads=False, variant=v, labels=lab).loss
              - O.kl_loss(*args, W_f64=W0, H_f64=Hm, want_grads=False, variant=v, labels=lab).loss) / (2 * h)
        assert fd == pytest.approx(r.dH[n, j], rel=1e-6, abs=1e-10)
        vv, j = rng.integers(0, 11), rng.integers(0, 6)
        Wp, Wm = W0.copy(), W0.copy()
        Wp[vv, j] += h
        Wm[vv, j] -= h
        fd = (O.kl_loss(*args, W_f64=Wp, H_f64=H0, want_grads=False, variant=v, labels=lab).loss
              - O.kl_loss(*args, W_f64=Wm, H_f64=H0, want_grads=False, variant=v, labels=lab).loss) / (2 * h)
        assert fd == pytest.approx(r.dW[vv, j], rel=1e-6, abs=1e-10)


def test_gradient_rows_sum_to_zero_with_labels():
    v = O.Variant(student_tau=1.3, kd_weight=0.5, ce_weight=0.5)
    x = synth.custom_inputs(10, 8, 29, 5, seed=66, mask_frac=0.2, w_std=0.5)
    r = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, 1.0, variant=v,
                  labels=_labels(x, 67), want_G=True)
    assert np.abs(r.G.sum(axis=1)).max() < 1e-15
