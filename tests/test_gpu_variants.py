"""CUDA path vs the oracle for the compact cache format (uint16 indices + bf16
logits) and the loss-design variants (student temperature, tau^2 factor,
hard-label cross-entropy term), on seeded inputs with ragged tails."""
import numpy as np
import pytest
import torch

import output_head_kl_b200 as K
import synth
from oracle import kl as O
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


def _compact(x):
    """The same cache stored as uint16 indices and bf16 logits, and its exact widening."""
    idx16 = x.topk_idx.astype(np.uint16)
    lg16 = synth.f32_to_bf16_bits(x.topk_logit)
    widened = synth.Inputs(x.hidden_bits, x.W_bits, idx16.astype(np.int32),
                           O.bf16_bits_to_f64(lg16).astype(np.float32), x.mask, x.tau)
    return idx16, lg16, widened


def _parity(g, r):
    assert g.flags == r.flags
    H.assert_loss(g.loss, r.loss)
    H.assert_lse(g.lse, r.lse)
    H.assert_grad(g.dH, r.dH, "dHidden")
    H.assert_grad(g.dW, r.dW, "dW")


def test_compact_cache_matches_oracle_and_wide_cache():
    x = synth.custom_inputs(700, 192, 3001, 24, seed=301, cache="zipf", logit_std=3.0, mask_frac=0.05, w_std=0.05)
    idx16, lg16, wide = _compact(x)
    dx = H.to_device(wide)
    g_wide = H.run_gpu(dx, chunk_tokens=256)
    dx16 = H.to_device(wide)
    dx16.idx = torch.from_numpy(idx16.view(np.int16)).cuda()
    dx16.logit = torch.from_numpy(lg16.view(np.int16)).cuda()
    g16 = H.run_gpu(dx16, chunk_tokens=256, options=K.kdkl_options(cache_format=K.CACHE_U16_BF16))
    r = O.kl_loss(wide.hidden_bits, wide.W_bits, wide.topk_idx, wide.topk_logit, wide.mask, wide.tau)
    _parity(g16, r)
    assert g16.loss == g_wide.loss
    np.testing.assert_array_equal(g16.lse, g_wide.lse)
    np.testing.assert_array_equal(g16.dH, g_wide.dH)
    np.testing.assert_array_equal(g16.dW, g_wide.dW)


def test_compact_cache_rejects_large_vocab():
    x = synth.custom_inputs(4, 16, 70000, 2, seed=302)
    dx = H.to_device(x)
    ws = torch.empty(K.kdkl_workspace_bytes(4, 16, 70000, 2), dtype=torch.uint8, device="cuda")
    loss = torch.empty(1, device="cuda")
    lse = torch.empty(4, device="cuda")
    st = K.kdkl_forward_ex(dx.hidden, dx.W, dx.idx, dx.logit, dx.mask, 1.0, loss, lse, ws,
                           K.kdkl_options(cache_format=K.CACHE_U16_BF16), check=False)
    assert st == 2 and "65536" in K.kdkl_last_error()


VARIANTS = [
    (O.Variant(student_tau=2.0, kd_scale_tau_sq=True), 2.0),
    (O.Variant(student_tau=1.5, kd_weight=0.6, ce_weight=0.4), 1.0),
    (O.Variant(kd_weight=0.0, ce_weight=1.0), 1.0),
    (O.Variant(student_tau=0.7, kd_weight=0.3, kd_scale_tau_sq=True, ce_weight=2.0), 1.0),
]


@pytest.mark.parametrize("variant,tau", VARIANTS)
def test_loss_variants_match_oracle(variant, tau):
    x = synth.custom_inputs(600, 200, 2500, 20, seed=303, tau=tau, cache="zipf", logit_std=3.0, mask_frac=0.05,
                            w_std=0.08)
    rng = np.random.default_rng(304)
    lab = rng.integers(0, 2500, size=600).astype(np.int32)
    lab[rng.random(600) < 0.1] = -100
    lab[:40] = x.topk_idx[:40, 0]            # labels that coincide with a cached entry
    dx = H.to_device(x)
    labels = torch.from_numpy(lab).cuda()
    opts = K.kdkl_options(student_tau=variant.student_tau, kd_weight=variant.kd_weight,
                          kd_scale_tau_sq=variant.kd_scale_tau_sq, ce_weight=variant.ce_weight, labels=labels)
    g = H.run_gpu(dx, chunk_tokens=256, options=opts)
    r = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau, variant=variant, labels=lab)
    _parity(g, r)


def test_default_options_equal_plain_entry_points():
    x = synth.custom_inputs(300, 128, 1500, 8, seed=305, mask_frac=0.1, w_std=0.1)
    dx = H.to_device(x)
    a = H.run_gpu(dx)
    b = H.run_gpu(dx, options=K.kdkl_options())
    assert a.loss == b.loss
    np.testing.assert_array_equal(a.dW, b.dW)


def test_variant_with_full_cache_and_label_insertion():
    """K = 256 cached entries plus a label per row: the target list holds 257 entries."""
    x = synth.custom_inputs(260, 128, 3000, 256, seed=306, cache="zipf", logit_std=3.0, w_std=0.1)
    rng = np.random.default_rng(307)
    lab = rng.integers(0, 3000, size=260).astype(np.int32)
    v = O.Variant(student_tau=1.2, kd_weight=0.7, ce_weight=0.3)
    opts = K.kdkl_options(student_tau=v.student_tau, kd_weight=v.kd_weight, ce_weight=v.ce_weight,
                          labels=torch.from_numpy(lab).cuda())
    g = H.run_gpu(H.to_device(x), options=opts)
    r = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau, variant=v, labels=lab)
    _parity(g, r)


def test_global_normaliser_option_and_dp_step_single_rank():
    """n_valid_global replaces the local count (data-parallel normaliser); one rank of dp_step = plain path."""
    from output_head_kl_b200 import dp
    x = synth.custom_inputs(400, 128, 2000, 12, seed=308, mask_frac=0.1, w_std=0.1)
    dx = H.to_device(x)
    base = H.run_gpu(dx)
    nv = int((x.mask != 0).sum())
    doubled = torch.tensor([2 * nv], dtype=torch.int32, device="cuda")
    g = H.run_gpu(dx, options=K.kdkl_options(n_valid_global=doubled))
    assert g.loss == pytest.approx(base.loss / 2, rel=1e-6)
    np.testing.assert_allclose(g.dW, base.dW / 2, rtol=1e-5, atol=1e-12)
    res = dp.dp_step(dx.hidden, dx.W, dx.idx, dx.logit, dx.mask, dx.tau)
    torch.cuda.synchronize()
    assert int(res.n_valid_global.item()) == nv
    assert res.loss.item() == pytest.approx(base.loss, rel=1e-6)
    np.testing.assert_array_equal(res.dW.cpu().numpy(), base.dW.astype(np.float32))


def test_count_valid_matches_the_oracle_count_and_flags():
    """kdkl_count_valid leaves the oracle's N_valid (rows with a NaN logit or no in-range
    entry are not counted) at kdkl_n_valid_device, with the data-error flags; the forward on
    the same workspace then reports the same count."""
    N, d, V, Kc = 300, 64, 1000, 8
    x = synth.custom_inputs(N, d, V, Kc, seed=309, mask_frac=0.1, w_std=0.1)
    x.mask[5] = x.mask[7] = 1
    x.topk_logit[5, 2] = np.nan          # a non-finite teacher row: treated as masked
    x.topk_idx[7, :] = -1                # no in-range entry: treated as masked
    dx = H.to_device(x)
    ws = torch.empty(K.kdkl_workspace_bytes(N, d, V, Kc), dtype=torch.uint8, device="cuda")
    K.kdkl_count_valid(dx.idx, dx.logit, dx.mask, dx.tau, V, ws)
    count = K.n_valid_view(ws)
    nv = int(count.item())
    flags = K.kdkl_read_device_flags(ws)
    r = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau, want_grads=False)
    assert nv == r.n_valid == int((x.mask != 0).sum()) - 2
    assert flags == r.flags == (K.DEV_IDX_RANGE | K.DEV_NONFINITE)
    loss = torch.empty(1, device="cuda")
    lse = torch.empty(N, device="cuda")
    K.kdkl_forward(dx.hidden, dx.W, dx.idx, dx.logit, dx.mask, dx.tau, loss, lse, ws)
    assert int(count.item()) == nv
    K.kdkl_count_valid(dx.idx, dx.logit, dx.mask, dx.tau, V, ws, N=0)
    assert int(count.item()) == 0
