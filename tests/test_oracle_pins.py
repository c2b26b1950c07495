"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test names the fact it pins: a closed form worked by hand, a textbook or
library routine the definition reduces to (``torch.nn.functional.kl_div`` /
``cross_entropy`` with autograd), an invariant of KL divergence, finite
differences of the oracle's own loss, or a symmetry of the definition.  Every
plausible slip in the oracle (a dropped entropy term, a wrong sign, a wrong
gather index, a transposed operand, a missing mask, a wrong normaliser, tau on
the wrong side) breaks at least one of them.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import synth
from oracle import kl as O


def _bits(x):
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _small(seed=1, N=9, d=12, V=37, K=5, tau=1.0, mask_frac=0.0, w_std=0.3):
    return synth.custom_inputs(N, d, V, K, seed=seed, tau=tau, mask_frac=mask_frac, w_std=w_std)


# ---------------------------------------------------------------------------
# bf16 handling


def test_bf16_widening_known_patterns():
    bits = np.array([0x3F80, 0xC000, 0x3F81, 0x0000, 0x8000, 0x4049], dtype=np.uint16)
    got = O.bf16_bits_to_f64(bits)
    assert got.tolist() == [1.0, -2.0, 1.0078125, 0.0, -0.0, 3.140625]


def test_bf16_rounding_ties_to_even():
    # 1 + 2^-8 sits halfway between 1.0 and 1 + 2^-7: ties go to the even mantissa (1.0)
    # 1 + 3*2^-8 sits halfway between 1 + 2^-7 and 1 + 2^-6: ties go to 1 + 2^-6
    vals = np.array([1.0, 1.00390625, 1.01171875, -2.5, 1.0 + 2.0 ** -9], dtype=np.float32)
    assert [hex(b) for b in _bits(vals)] == ["0x3f80", "0x3f80", "0x3f82", "0xc020", "0x3f80"]


# ---------------------------------------------------------------------------
# closed forms worked by hand


def test_closed_form_two_entry_teacher():
    """z = (0, 1, 2) from a unit hidden state; teacher = uniform over entries {0, 2}.

    P_S = e^z / S with S = 1 + e + e^2;  KL = sum_v P_T log(P_T / P_S)
      = 0.5 (log .5 - (0 - log S)) + 0.5 (log .5 - (2 - log S)) = log S - 1 - log 2.
    G = P_S - P_T; dH = G W; dW = G^T h.
    """
    W = np.array([[0.0, 0.5], [1.0, -1.0], [2.0, 0.25]], dtype=np.float32)
    H = np.array([[1.0, 0.0]], dtype=np.float32)
    idx = np.array([[0, 2]], dtype=np.int32)
    logit = np.array([[0.0, 0.0]], dtype=np.float32)
    mask = np.ones(1, dtype=np.uint8)
    r = O.kl_loss(_bits(H), _bits(W), idx, logit, mask, 1.0)
    S = 1.0 + math.e + math.e ** 2
    assert r.loss == pytest.approx(math.log(S) - 1.0 - math.log(2.0), rel=1e-14)
    assert r.lse[0] == pytest.approx(math.log(S), rel=1e-15)
    Ps = np.array([1.0, math.e, math.e ** 2]) / S
    G = Ps - np.array([0.5, 0.0, 0.5])
    np.testing.assert_allclose(r.dH[0], G @ W.astype(np.float64), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(r.dW, np.outer(G, [1.0, 0.0]), rtol=1e-13, atol=1e-15)


def test_closed_form_temperature_and_normaliser():
    """Two rows, one masked.  Teacher logits (0, ln 3) at tau = 1 give P_T = (1/4, 3/4).

    Row 0: z = (0, 0, 0, 0) -> P_S uniform 1/4 over V = 4, teacher on entries {3, 1}:
      KL = 1/4 log(1/4 / 1/4) + 3/4 log(3/4 / 1/4) = 3/4 log 3.
    Row 1 is masked: N_valid = 1, so loss = 3/4 log 3 and row 1 gets no gradient.
    With tau = 2 the same cache gives P_T proportional to (1, sqrt 3).
    """
    W = np.zeros((4, 2), dtype=np.float32)
    H = np.array([[1.0, 2.0], [3.0, -1.0]], dtype=np.float32)
    idx = np.array([[3, 1], [0, 2]], dtype=np.int32)
    logit = np.array([[0.0, math.log(3.0)], [5.0, -5.0]], dtype=np.float32)
    mask = np.array([1, 0], dtype=np.uint8)
    r = O.kl_loss(_bits(H), _bits(W), idx, logit, mask, 1.0)
    assert r.n_valid == 1
    assert r.loss == pytest.approx(0.75 * math.log(3.0), rel=1e-7)  # fp32 ln 3 input
    assert np.all(r.dH[1] == 0.0)
    r2 = O.kl_loss(_bits(H), _bits(W), idx, logit, mask, 2.0)
    s3 = math.sqrt(3.0)
    pa, pb = 1.0 / (1.0 + s3), s3 / (1.0 + s3)
    want = pa * math.log(pa / 0.25) + pb * math.log(pb / 0.25)
    assert r2.loss == pytest.approx(want, rel=1e-7)


def test_all_rows_masked_gives_zero():
    x = _small()
    mask = np.zeros_like(x.mask)
    r = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, mask, 1.0)
    assert r.loss == 0.0 and r.n_valid == 0
    assert not r.dH.any() and not r.dW.any()
    assert np.all(np.isfinite(r.lse))


# ---------------------------------------------------------------------------
# special cases that reduce to library routines


def test_K_equals_V_matches_torch_kl_div_and_autograd():
    """K = V, tau = 1: the loss is the llm-wiki note's dense idiom
    F.kl_div(log_softmax(z), log_softmax(t), log_target=True) summed / N."""
    rng = np.random.default_rng(5)
    N, V = 6, 11
    z = rng.normal(size=(N, V)) * 2
    t = rng.normal(size=(N, V)) * 3
    perm = np.stack([rng.permutation(V) for _ in range(N)]).astype(np.int32)
    logit = np.take_along_axis(t, perm, axis=1).astype(np.float32)   # cache entries in any order
    mask = np.ones(N, dtype=np.uint8)
    loss, G = O.kl_loss_from_logits(z, perm, logit, mask, 1.0)
    zt = torch.tensor(z, dtype=torch.float64, requires_grad=True)
    t_dense = np.empty_like(t)
    np.put_along_axis(t_dense, perm.astype(np.int64), logit.astype(np.float64), axis=1)
    tt = torch.tensor(t_dense, dtype=torch.float64)
    ref = F.kl_div(F.log_softmax(zt, -1), F.log_softmax(tt, -1), log_target=True, reduction="sum") / N
    ref.backward()
    assert loss == pytest.approx(ref.item(), rel=1e-12)
    np.testing.assert_allclose(G, zt.grad.numpy(), rtol=1e-10, atol=1e-14)


def test_K_equals_V_identical_logits_gives_zero():
    rng = np.random.default_rng(6)
    N, V = 4, 9
    z = rng.normal(size=(N, V)).astype(np.float32).astype(np.float64)
    idx = np.tile(np.arange(V, dtype=np.int32), (N, 1))
    loss, G = O.kl_loss_from_logits(z, idx, z.astype(np.float32), np.ones(N, np.uint8), 1.0)
    assert abs(loss) < 1e-13
    assert np.abs(G).max() < 1e-15


def test_K1_is_cross_entropy():
    """A one-hot teacher (K = 1) makes the KL the cross-entropy of the cached index."""
    rng = np.random.default_rng(7)
    N, V = 8, 13
    z = rng.normal(size=(N, V)) * 2
    target = rng.integers(0, V, size=N)
    idx = target[:, None].astype(np.int32)
    logit = rng.normal(size=(N, 1)).astype(np.float32)
    loss, G = O.kl_loss_from_logits(z, idx, logit, np.ones(N, np.uint8), 1.0)
    zt = torch.tensor(z, dtype=torch.float64, requires_grad=True)
    ref = F.cross_entropy(zt, torch.tensor(target))
    ref.backward()
    assert loss == pytest.approx(ref.item(), rel=1e-13)
    np.testing.assert_allclose(G, zt.grad.numpy(), rtol=1e-12, atol=1e-15)


def test_projection_path_matches_autograd():
    """Through the projection: loss(H, W) against torch autograd of the dense idiom in fp64."""
    x = _small(seed=11, N=7, d=10, V=23, K=6, mask_frac=0.3)
    r = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau)
    H = torch.tensor(O.bf16_bits_to_f64(x.hidden_bits), requires_grad=True)
    W = torch.tensor(O.bf16_bits_to_f64(x.W_bits), requires_grad=True)
    V = W.shape[0]
    t = np.full((H.shape[0], V), -np.inf)
    np.put_along_axis(t, x.topk_idx.astype(np.int64), x.topk_logit.astype(np.float64), axis=1)
    logq = F.log_softmax(torch.tensor(t), -1)
    m = torch.tensor(x.mask.astype(np.float64))
    logp = F.log_softmax(H @ W.T, -1)
    q = logq.exp()
    per_row = torch.where(q > 0, q * (logq - logp), torch.zeros_like(q)).sum(-1)
    ref = (per_row * m).sum() / m.sum()
    ref.backward()
    assert r.loss == pytest.approx(ref.item(), rel=1e-12)
    np.testing.assert_allclose(r.dH, H.grad.numpy(), rtol=1e-9, atol=1e-15)
    np.testing.assert_allclose(r.dW, W.grad.numpy(), rtol=1e-9, atol=1e-15)


# ---------------------------------------------------------------------------
# invariants


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_kl_nonnegative_and_lower_bound(seed):
    """Gibbs: each row's KL >= -log sum_k P_S(idx_k) >= 0 (zero tail outside the cache)."""
    x = _small(seed=seed, N=16, d=8, V=29, K=7, w_std=1.0)
    r = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau, want_grads=False)
    H = O.bf16_bits_to_f64(x.hidden_bits)
    W = O.bf16_bits_to_f64(x.W_bits)
    z = H @ W.T
    logp = z - r.lse[:, None]
    mass = np.exp(np.take_along_axis(logp, x.topk_idx.astype(np.int64), 1)).sum(1)
    assert np.all(r.kl >= -np.log(mass) - 1e-12)
    assert np.all(r.kl > 0)


def test_gradient_rows_sum_to_zero():
    x = _small(seed=4, N=12, d=8, V=31, K=5, mask_frac=0.25)
    r = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau, want_G=True)
    rs = r.G.sum(axis=1)
    assert np.abs(rs).max() < 1e-15
    assert np.all(r.G[x.mask == 0] == 0.0)
    assert np.any(r.G[x.mask == 1] != 0.0)


def test_lse_brute_force():
    """lse_n = log sum_v exp(sum_j H[n, j] W[v, j]) by plain Python loops."""
    x = _small(seed=9, N=3, d=4, V=6, K=2, w_std=1.0)
    r = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau, want_grads=False)
    H = O.bf16_bits_to_f64(x.hidden_bits).tolist()
    W = O.bf16_bits_to_f64(x.W_bits).tolist()
    for n in range(3):
        acc = 0.0
        for v in range(6):
            acc += math.exp(sum(H[n][j] * W[v][j] for j in range(4)))
        assert r.lse[n] == pytest.approx(math.log(acc), rel=1e-14)


def test_sparse_form_agrees_with_dense_form():
    """KL_n = sum_k P_k log P_k - sum_k P_k z[idx_k] + lse_n (sparse) vs the dense scatter."""
    x = _small(seed=12, N=10, d=9, V=41, K=8, w_std=0.5)
    r = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau, want_grads=False)
    H = O.bf16_bits_to_f64(x.hidden_bits)
    W = O.bf16_bits_to_f64(x.W_bits)
    idx = x.topk_idx.astype(np.int64)
    t = x.topk_logit.astype(np.float64)
    P = np.exp(t - t.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    zi = np.einsum("nd,nkd->nk", H, W[idx])
    kl = (P * np.log(P)).sum(1) - (P * zi).sum(1) + r.lse
    np.testing.assert_allclose(r.kl, kl, rtol=1e-12)


# ---------------------------------------------------------------------------
# finite differences of the oracle's own loss


def test_finite_differences_hidden_and_W():
    x = _small(seed=21, N=5, d=6, V=11, K=4, mask_frac=0.2, w_std=0.7)
    H0 = O.bf16_bits_to_f64(x.hidden_bits)
    W0 = O.bf16_bits_to_f64(x.W_bits)
    args = (x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau)
    r = O.kl_loss(*args, W_f64=W0, H_f64=H0)
    h = 1e-6
    rng = np.random.default_rng(0)
    for _ in range(12):
        n, j = rng.integers(0, 5), rng.integers(0, 6)
        Hp, Hm = H0.copy(), H0.copy()
        Hp[n, j] += h
        Hm[n, j] -= h
        fd = (O.kl_loss(*args, W_f64=W0, H_f64=Hp, want_grads=False).loss
              - O.kl_loss(*args, W_f64=W0, H_f64=Hm, want_grads=False).loss) / (2 * h)
        assert fd == pytest.approx(r.dH[n, j], rel=1e-6, abs=1e-10)
        v, j = rng.integers(0, 11), rng.integers(0, 6)
        Wp, Wm = W0.copy(), W0.copy()
        Wp[v, j] += h
        Wm[v, j] -= h
        fd = (O.kl_loss(*args, W_f64=Wp, H_f64=H0, want_grads=False).loss
              - O.kl_loss(*args, W_f64=Wm, H_f64=H0, want_grads=False).loss) / (2 * h)
        assert fd == pytest.approx(r.dW[v, j], rel=1e-6, abs=1e-10)


def test_grad_loss_scales_gradients():
    x = _small(seed=22)
    a = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau)
    b = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau, grad_loss=-2.5)
    np.testing.assert_allclose(b.dH, -2.5 * a.dH, rtol=1e-13, atol=1e-16)
    np.testing.assert_allclose(b.dW, -2.5 * a.dW, rtol=1e-13, atol=1e-16)


# ---------------------------------------------------------------------------
# symmetries and chunk invariance (the pages: the variants are equivalent)


def test_row_chunk_invariance():
    x = _small(seed=31, N=23, d=16, V=53, K=6, mask_frac=0.1)
    args = (x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau)
    base = O.kl_loss(*args, row_chunk=23)
    for R in (1, 7):
        r = O.kl_loss(*args, row_chunk=R)
        assert r.loss == pytest.approx(base.loss, rel=1e-13)
        np.testing.assert_allclose(r.lse, base.lse, rtol=1e-14)
        np.testing.assert_allclose(r.dH, base.dH, rtol=1e-12, atol=1e-17)
        np.testing.assert_allclose(r.dW, base.dW, rtol=1e-12, atol=1e-17)


def test_logit_shift_and_permutation_invariance():
    x = _small(seed=32, N=8, K=6)
    args = (x.hidden_bits, x.W_bits)
    base = O.kl_loss(*args, x.topk_idx, x.topk_logit, x.mask, 1.0)
    shifted = x.topk_logit + np.arange(8, dtype=np.float32)[:, None] * 4.0
    r = O.kl_loss(*args, x.topk_idx, shifted, x.mask, 1.0)
    assert r.loss == pytest.approx(base.loss, rel=1e-6)
    rng = np.random.default_rng(1)
    perm = np.stack([rng.permutation(6) for _ in range(8)])
    r = O.kl_loss(*args, np.take_along_axis(x.topk_idx, perm, 1), np.take_along_axis(x.topk_logit, perm, 1),
                  x.mask, 1.0)
    assert r.loss == pytest.approx(base.loss, rel=1e-13)
    np.testing.assert_allclose(r.dW, base.dW, rtol=1e-12, atol=1e-17)


def test_tau_acts_on_teacher_only():
    """tau = 2 on logits t equals tau = 1 on t / 2 (exactly representable halving)."""
    x = _small(seed=33)
    args = (x.hidden_bits, x.W_bits, x.topk_idx)
    a = O.kl_loss(*args, x.topk_logit, x.mask, 2.0)
    b = O.kl_loss(*args, x.topk_logit / np.float32(2.0), x.mask, 1.0)
    assert a.loss == pytest.approx(b.loss, rel=1e-14)
    np.testing.assert_allclose(a.dH, b.dH, rtol=1e-13, atol=1e-18)
    c = O.kl_loss(*args, x.topk_logit, x.mask, 1.0)
    assert abs(c.loss - a.loss) > 1e-3
    np.testing.assert_allclose(c.lse, a.lse, rtol=0, atol=0)   # the student side does not see tau


def test_masked_rows_do_not_matter():
    x = _small(seed=34, N=10, mask_frac=0.3)
    base = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, 1.0)
    H2 = x.hidden_bits.copy()
    H2[x.mask == 0] = _bits(np.full((int((x.mask == 0).sum()), H2.shape[1]), 7.0))
    r = O.kl_loss(H2, x.W_bits, x.topk_idx, x.topk_logit, x.mask, 1.0)
    assert r.loss == base.loss
    np.testing.assert_array_equal(r.dW, base.dW)
    assert np.any(r.lse[x.mask == 0] != base.lse[x.mask == 0])
    np.testing.assert_array_equal(r.lse[x.mask == 1], base.lse[x.mask == 1])


# ---------------------------------------------------------------------------
# data errors (R7, R8)


def test_out_of_range_entries_are_dropped_and_flagged():
    x = _small(seed=41, N=6, K=5)
    idx = x.topk_idx.copy()
    idx[2, 1] = x.W_bits.shape[0] + 3
    idx[4, 0] = -1
    r = O.kl_loss(x.hidden_bits, x.W_bits, idx, x.topk_logit, x.mask, 1.0)
    assert r.flags == O.FLAG_IDX_RANGE
    # same as a cache whose bad entries carry a -inf logit (probability 0)
    logit = x.topk_logit.copy()
    logit[2, 1] = -np.inf
    logit[4, 0] = -np.inf
    ok_idx = x.topk_idx
    r2 = O.kl_loss(x.hidden_bits, x.W_bits, ok_idx, logit, x.mask, 1.0)
    assert r2.flags == 0
    assert r.loss == pytest.approx(r2.loss, rel=1e-14)
    np.testing.assert_allclose(r.dH, r2.dH, rtol=1e-13, atol=1e-18)


def test_duplicates_add_up():
    """Two entries (t1, t2) on one index act like one entry with logit log(e^t1 + e^t2)."""
    x = _small(seed=42, N=4, K=4)
    idx = x.topk_idx.copy()
    logit = x.topk_logit.astype(np.float64)
    idx[1, 3] = idx[1, 0]
    r = O.kl_loss(x.hidden_bits, x.W_bits, idx, logit.astype(np.float32), x.mask, 1.0)
    assert r.flags == O.FLAG_IDX_DUP
    t = logit.astype(np.float32).astype(np.float64)
    merged = np.log(np.exp(t[1, 0]) + np.exp(t[1, 3]))
    idx3 = np.delete(idx[1], 3)
    l3 = np.delete(t[1], 3)
    l3[0] = merged
    single = O.kl_loss(x.hidden_bits[1:2], x.W_bits, idx3[None].astype(np.int32), l3[None], x.mask[1:2], 1.0)
    assert r.kl[1] == pytest.approx(single.kl[0], rel=1e-12)


def test_nonfinite_rows_are_masked_and_flagged():
    x = _small(seed=43, N=6, K=4)
    logit = x.topk_logit.copy()
    logit[1, 2] = np.nan
    logit[3, :] = -np.inf
    logit[5, 1] = -np.inf          # a single -inf entry is fine: probability 0
    r = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, logit, x.mask, 1.0)
    assert r.flags == O.FLAG_NONFINITE
    assert r.n_valid == 4
    assert np.all(r.dH[[1, 3]] == 0.0)
    assert r.kl[5] > 0 and np.isfinite(r.kl[5])
    keep = np.array([0, 2, 4, 5])
    sub = O.kl_loss(x.hidden_bits[keep], x.W_bits, x.topk_idx[keep], logit[keep], x.mask[keep], 1.0)
    assert r.loss == pytest.approx(sub.loss, rel=1e-14)
