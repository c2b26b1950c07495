"""The fused forward + backward (each logit chunk computed once) vs the oracle, and
vs the separate forward and backward calls.

The fused step must give the oracle's loss, lse, dHidden and dW within the same
tolerances as the separate calls, for every option and chunking; and agree with
the separate calls far more tightly, since both run the same arithmetic on the
same logits and differ only in how each row's log-sum-exp partials are merged.
"""
import numpy as np
import pytest
import torch

import output_head_kl_b200 as K
import synth
from oracle import kl as O
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


def _fused(dx, *, chunk_tokens=0, options=None, grad_loss=None):
    N, d = dx.hidden.shape
    V, Kc = dx.W.shape[0], dx.idx.shape[1]
    ws = torch.empty(K.kdkl_forward_backward_workspace_bytes(N, d, V, Kc, chunk_tokens), dtype=torch.uint8,
                     device="cuda")
    loss = torch.full((1,), float("nan"), device="cuda")
    lse = torch.full((N,), float("nan"), device="cuda")
    dH = torch.full((N, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    dW = torch.full((V, d), float("nan"), device="cuda")
    g = None if grad_loss is None else torch.tensor([grad_loss], dtype=torch.float32, device="cuda")
    K.kdkl_forward_backward(dx.hidden, dx.W, dx.idx, dx.logit, dx.mask, dx.tau, loss, lse, dH, dW, ws, options,
                            grad_loss=g, chunk_tokens=chunk_tokens)
    flags = K.kdkl_read_device_flags(ws)
    torch.cuda.synchronize()
    return H.GpuResult(float(loss.item()), lse.cpu().numpy().astype(np.float64),
                       dH.float().cpu().numpy().astype(np.float64), dW.cpu().numpy().astype(np.float64), flags)


def _check(g, r):
    assert g.flags == r.flags
    H.assert_loss(g.loss, r.loss)
    H.assert_lse(g.lse, r.lse)
    H.assert_grad(g.dH, r.dH, "dHidden")
    H.assert_grad(g.dW, r.dW, "dW")


# dHidden is bf16: a G element whose value moves across a rounding boundary (the
# lse differs in its last bits) can move a dHidden element by one bf16 unit, i.e.
# up to 2^-8 of the largest element; the bound allows two such units.
DH_REL = 2.0 ** -7


def _close(a, b):
    """Fused vs separate calls on the same inputs."""
    assert abs(a.loss - b.loss) <= 1e-5 * max(abs(b.loss), 1e-6)
    assert np.abs(a.lse - b.lse).max() <= 1e-5
    assert np.abs(a.dH - b.dH).max() <= DH_REL * np.abs(b.dH).max()
    assert np.abs(a.dW - b.dW).max() <= 1e-3 * np.abs(b.dW).max()


@pytest.mark.parametrize("chunk", [0, 256, 100])
def test_ragged_shapes_vs_oracle_and_separate_calls(chunk):
    # N, V, d off the tile grid; chunk 100 rounds up to 256 (two chunks, the second 44 rows)
    x = synth.custom_inputs(300, 200, 1001, 7, seed=201, mask_frac=0.1, w_std=0.1)
    dx = H.to_device(x)
    g = _fused(dx, chunk_tokens=chunk)
    _check(g, O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau))
    _close(g, H.run_gpu(dx, chunk_tokens=chunk))


def test_tiny_and_small_configs():
    for name in ("tiny", "small"):
        x = synth.make_inputs(synth.CONFIGS[name])
        g = _fused(H.to_device(x))
        _check(g, O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau))


def test_many_chunks_grad_scale_and_data_errors():
    x = synth.custom_inputs(1300, 256, 3000, 16, seed=202, mask_frac=0.05, w_std=0.05, cache="zipf", logit_std=3.0)
    x.topk_idx[7, 3] = 3000 + 5                 # out of range
    x.topk_idx[11, 2] = x.topk_idx[11, 0]       # repeated
    x.topk_logit[20, :] = -np.inf               # row masked
    dx = H.to_device(x)
    g = _fused(dx, chunk_tokens=256, grad_loss=-1.5)
    r = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau, grad_loss=-1.5)
    _check(g, r)
    assert g.flags == (O.FLAG_IDX_RANGE | O.FLAG_IDX_DUP | O.FLAG_NONFINITE)
    assert np.all(g.dH[20] == 0.0)


def test_variants_and_compact_cache():
    x = synth.custom_inputs(520, 128, 4000, 24, seed=203, mask_frac=0.05, w_std=0.1, cache="zipf", logit_std=3.0)
    labels = np.random.default_rng(5).integers(0, 4000, size=520).astype(np.int32)
    labels[::7] = -100
    variant = O.Variant(student_tau=2.0, kd_weight=0.7, kd_scale_tau_sq=True, ce_weight=0.3)
    r = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau, variant=variant, labels=labels)
    dx = H.to_device(x)
    lab = torch.from_numpy(labels).cuda()
    opts = K.kdkl_options(student_tau=2.0, kd_weight=0.7, kd_scale_tau_sq=True, ce_weight=0.3, labels=lab)
    g = _fused(dx, chunk_tokens=256, options=opts)
    _check(g, r)
    _close(g, H.run_gpu(dx, chunk_tokens=256, options=opts))
    # 16-bit indices + bf16 logits: the cache widened back is what the oracle sees
    xc = synth.custom_inputs(300, 128, 3000, 12, seed=204, w_std=0.1)
    xc.topk_logit = O.bf16_bits_to_f64(synth.f32_to_bf16_bits(xc.topk_logit)).astype(np.float32)
    dxc = H.to_device(xc)
    dxc.idx = dxc.idx.to(torch.int16)
    dxc.logit = dxc.logit.to(torch.bfloat16)
    g = _fused(dxc, options=K.kdkl_options(cache_format=K.CACHE_U16_BF16))
    _check(g, O.kl_loss(xc.hidden_bits, xc.W_bits, xc.topk_idx, xc.topk_logit, xc.mask, xc.tau))


def test_every_row_masked_and_empty_batch():
    x = synth.custom_inputs(300, 64, 512, 4, seed=205)
    x.mask[:] = 0
    g = _fused(H.to_device(x))
    assert g.loss == 0.0 and np.all(g.dH == 0.0) and np.all(g.dW == 0.0)
    dx = H.to_device(synth.custom_inputs(8, 64, 512, 4, seed=206))
    ws = torch.empty(K.kdkl_forward_backward_workspace_bytes(0, 64, 512, 4), dtype=torch.uint8, device="cuda")
    loss = torch.full((1,), 7.0, device="cuda")
    dW = torch.full((512, 64), 7.0, device="cuda")
    K.kdkl_forward_backward(dx.hidden, dx.W, dx.idx, dx.logit, dx.mask, 1.0, loss, torch.empty(8, device="cuda"),
                            torch.empty(8, 64, dtype=torch.bfloat16, device="cuda"), dW, ws, N=0)
    torch.cuda.synchronize()
    assert loss.item() == 0.0 and torch.all(dW == 0)


def test_fullsize_8b_matches_separate_calls():
    """The bench's 8B-class workload: the fused step and the separate calls agree on
    every output element (compared on the device)."""
    x = synth.make_inputs(synth.CONFIGS["8b"])
    dx = H.to_device(x)
    N, d = dx.hidden.shape
    V, Kc = dx.W.shape[0], dx.idx.shape[1]
    out = {}
    for mode in ("separate", "fused"):
        loss = torch.empty(1, device="cuda")
        lse = torch.empty(N, device="cuda")
        dH = torch.empty(N, d, dtype=torch.bfloat16, device="cuda")
        dW = torch.empty(V, d, device="cuda")
        if mode == "fused":
            ws = torch.empty(K.kdkl_forward_backward_workspace_bytes(N, d, V, Kc), dtype=torch.uint8, device="cuda")
            K.kdkl_forward_backward(dx.hidden, dx.W, dx.idx, dx.logit, dx.mask, dx.tau, loss, lse, dH, dW, ws)
        else:
            ws = torch.empty(K.kdkl_workspace_bytes(N, d, V, Kc), dtype=torch.uint8, device="cuda")
            K.kdkl_forward(dx.hidden, dx.W, dx.idx, dx.logit, dx.mask, dx.tau, loss, lse, ws)
            K.kdkl_backward(dx.hidden, dx.W, dx.idx, dx.logit, dx.mask, dx.tau, lse, None, dH, dW, ws)
        assert K.kdkl_read_device_flags(ws) == 0
        out[mode] = (loss, lse, dH, dW)
        del ws
    (la, sa, ha, wa), (lb, sb, hb, wb) = out["fused"], out["separate"]
    assert abs(la.item() - lb.item()) <= 1e-5 * abs(lb.item())
    assert float((sa - sb).abs().max()) <= 1e-5
    assert float((ha.float() - hb.float()).abs().max()) <= DH_REL * float(hb.float().abs().max())
    assert float((wa - wb).abs().max()) <= 1e-3 * float(wb.abs().max())
