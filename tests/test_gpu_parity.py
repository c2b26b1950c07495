"""CUDA path vs the CPU oracle, element by element, on seeded inputs.

Sizes are ones the fp64 oracle finishes in seconds while still spanning
several 128-row tiles, several 256-column vocabulary tiles, several K blocks
and ragged tails in N, V and d; plus the edge cases of the method.
"""
import numpy as np
import pytest

import synth
from oracle import kl as O
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


def _oracle(x, **kw):
    return O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau, **kw)


def _full_parity(x, chunk_tokens=0, grad_loss=None):
    g = H.run_gpu(H.to_device(x), chunk_tokens=chunk_tokens, grad_loss=grad_loss)
    r = _oracle(x, grad_loss=1.0 if grad_loss is None else grad_loss)
    assert g.flags == r.flags
    H.assert_loss(g.loss, r.loss)
    H.assert_lse(g.lse, r.lse)
    H.assert_grad(g.dH, r.dH, "dHidden")
    H.assert_grad(g.dW, r.dW, "dW")
    return g, r


def test_tiny_config():
    _full_parity(synth.make_inputs(synth.CONFIGS["tiny"]))


def test_ragged_shapes_multi_tile():
    # N, V, d all off the tile grid: 3 row blocks (last one 44 rows), 4 vocab tiles
    # (last one 233 wide, V % 8 != 0), 4 K blocks (last one 8 wide)
    x = synth.custom_inputs(300, 200, 1001, 7, seed=101, mask_frac=0.1, w_std=0.1)
    _full_parity(x)


def test_small_config():
    _full_parity(synth.make_inputs(synth.CONFIGS["small"]))


def test_backward_chunks_agree():
    x = synth.custom_inputs(700, 256, 2048, 16, seed=102, mask_frac=0.05, w_std=0.05)
    g1, r = _full_parity(x, chunk_tokens=128)       # 6 chunks, the last one 60 rows
    g2 = H.run_gpu(H.to_device(x), chunk_tokens=0)  # one chunk
    np.testing.assert_array_equal(g1.dH, g2.dH)     # dHidden rows do not depend on the chunking
    H.assert_grad(g1.dW, g2.dW, "dW chunked vs single")


def test_grad_loss_scale():
    x = synth.custom_inputs(256, 128, 1024, 8, seed=103, w_std=0.1)
    _full_parity(x, grad_loss=-2.5)


def test_temperature_two():
    x = synth.custom_inputs(256, 256, 3000, 32, seed=104, tau=2.0, cache="zipf", logit_std=3.0,
                            mask_frac=0.05, w_std=0.05)
    _full_parity(x)


def test_data_errors_flagged_and_handled():
    x = synth.custom_inputs(260, 128, 1536, 12, seed=105, w_std=0.1)
    x.topk_idx[3, 2] = 1536 + 7          # out of range -> dropped
    x.topk_idx[9, 0] = -4
    x.topk_idx[17, 5] = x.topk_idx[17, 1]  # repeated index -> probabilities add
    x.topk_logit[33, 4] = np.nan          # NaN -> row masked
    x.topk_logit[40, :] = -np.inf         # all -inf -> row masked
    x.topk_logit[41, 7] = -np.inf         # one -inf entry is fine
    g, r = _full_parity(x)
    assert g.flags == (O.FLAG_IDX_RANGE | O.FLAG_IDX_DUP | O.FLAG_NONFINITE)
    assert np.all(g.dH[[33, 40]] == 0.0)


def test_every_row_masked():
    x = synth.custom_inputs(200, 64, 512, 4, seed=106)
    x.mask[:] = 0
    g = H.run_gpu(H.to_device(x))
    assert g.loss == 0.0
    assert np.all(g.dH == 0.0) and np.all(g.dW == 0.0)
    r = _oracle(x, want_grads=False)
    H.assert_lse(g.lse, r.lse)


def test_empty_batch():
    x = synth.custom_inputs(1, 64, 512, 4, seed=107)
    dx = H.to_device(x)
    dx.hidden = dx.hidden[:0]
    dx.idx = dx.idx[:0]
    dx.logit = dx.logit[:0]
    dx.mask = dx.mask[:0]
    import torch
    import output_head_kl_b200 as K
    ws = torch.empty(K.kdkl_workspace_bytes(0, 64, 512, 4), dtype=torch.uint8, device="cuda")
    hidden = torch.empty(8, 64, dtype=torch.bfloat16, device="cuda")
    loss = torch.full((1,), 7.0, device="cuda")
    lse = torch.empty(8, device="cuda")
    dW = torch.full((512, 64), 7.0, device="cuda")
    dH = torch.empty(8, 64, dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros(8, 4, dtype=torch.int32, device="cuda")
    lg = torch.zeros(8, 4, device="cuda")
    mk = torch.ones(8, dtype=torch.uint8, device="cuda")
    K.kdkl_forward(hidden, dx.W, idx, lg, mk, 1.0, loss, lse, ws, N=0)
    K.kdkl_backward(hidden, dx.W, idx, lg, mk, 1.0, lse, None, dH, dW, ws, N=0)
    torch.cuda.synchronize()
    assert loss.item() == 0.0
    assert torch.all(dW == 0)


def test_one_hot_teacher_is_cross_entropy():
    x = synth.custom_inputs(384, 128, 2000, 1, seed=108, w_std=0.2)
    _full_parity(x)


def test_full_teacher_K_equals_V():
    """K = V = 128 with teacher logits equal to the student's own logits: KL ~ 0, grads ~ 0.

    The true gradient is zero here, so it is compared on an absolute scale: the
    gradient of the same inputs against a shuffled teacher sets the scale."""
    x = synth.custom_inputs(256, 64, 128, 128, seed=109, w_std=0.3)
    Hf = O.bf16_bits_to_f64(x.hidden_bits)
    Wf = O.bf16_bits_to_f64(x.W_bits)
    z = Hf @ Wf.T
    x.topk_idx[:] = np.arange(128, dtype=np.int32)[None, :]
    x.topk_logit[:] = z.astype(np.float32)
    g = H.run_gpu(H.to_device(x))
    r = _oracle(x)
    assert abs(r.loss) < 1e-12
    assert abs(g.loss) < 1e-4
    H.assert_lse(g.lse, r.lse)
    shuffled = _oracle(synth.Inputs(x.hidden_bits, x.W_bits, x.topk_idx,
                                    np.ascontiguousarray(x.topk_logit[:, ::-1]), x.mask, x.tau))
    assert np.abs(g.dH).max() <= 1e-3 * np.abs(shuffled.dH).max()
    assert np.abs(g.dW).max() <= 1e-3 * np.abs(shuffled.dW).max()


def test_constant_W_column_gives_zero_dH_column():
    """Each G row sums to 0, so a constant column c of W gives dH[:, j] = c * sum_v G = 0."""
    x = synth.custom_inputs(512, 128, 4096, 16, seed=110, mask_frac=0.1, w_std=0.1)
    x.W_bits[:, 5] = synth.f32_to_bf16_bits(np.full(x.W_bits.shape[0], 0.25, dtype=np.float32))
    g, r = _full_parity(x)
    assert np.abs(g.dH[:, 5]).max() <= 1e-2 * np.abs(g.dH).max()
    assert np.abs(r.dH[:, 5]).max() < 1e-15


def test_largest_cache_K256():
    """K = 256 (the largest cache the ABI takes; eight entries per prepass lane)."""
    x = synth.custom_inputs(300, 128, 3000, 256, seed=111, cache="zipf", logit_std=3.0, mask_frac=0.05, w_std=0.1)
    _full_parity(x)


def test_ragged_cache_K255_with_duplicates():
    x = synth.custom_inputs(200, 64, 2000, 255, seed=112, w_std=0.1)
    x.topk_idx[5, 200] = x.topk_idx[5, 3]
    g, r = _full_parity(x)
    assert g.flags == O.FLAG_IDX_DUP


@pytest.mark.parametrize("N,d,V,Kc", [(130, 8, 100, 10), (3, 24, 257, 3), (5, 8, 40, 40)])
def test_minimal_shapes(N, d, V, Kc):
    """d = 8 (one 16-byte row: every box runs past d into zero fill), vocabularies narrower
    than one 256-wide tile or one column past it, and a batch smaller than one row block."""
    x = synth.custom_inputs(N, d, V, Kc, seed=150 + N, w_std=0.5, mask_frac=0.2 if N > 10 else 0.0)
    _full_parity(x)


def test_single_entry_vocabulary():
    """V = K = 1: teacher and student both put all mass on the one entry, so the loss and
    every gradient are zero up to rounding, and lse equals the one logit."""
    x = synth.custom_inputs(70, 16, 1, 1, seed=160, w_std=0.5)
    g = H.run_gpu(H.to_device(x))
    r = _oracle(x)
    assert r.loss == 0.0 and np.abs(r.dH).max() == 0.0
    assert abs(g.loss) < 1e-6
    H.assert_lse(g.lse, r.lse)
    z = O.bf16_bits_to_f64(x.hidden_bits) @ O.bf16_bits_to_f64(x.W_bits)[0]
    np.testing.assert_allclose(r.lse, z, rtol=0, atol=1e-12)
    hw = np.abs(O.bf16_bits_to_f64(x.hidden_bits)).max() * np.abs(O.bf16_bits_to_f64(x.W_bits)).max()
    assert np.abs(g.dH).max() <= 1e-5 * hw and np.abs(g.dW).max() <= 1e-5 * hw
