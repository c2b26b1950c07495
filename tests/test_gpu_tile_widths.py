"""The backward's dHidden / dW GEMMs at every supported tile width, and its planner.

The tile width is the N extent (over d) of one CTA pair's output tile.  Widths
that are not a multiple of 128 leave each CTA of the pair a B half that ends
inside a 64-column swizzle atom, and widths that are not a multiple of 32 end
inside a 32-column TMEM chunk of the epilogue; d is chosen so that every width
also meets a ragged last tile or an exact fit.  Each width is compared with the
oracle, and with every other width bit for bit: the width only partitions the
output, each element is still accumulated over the same reduction blocks in the
same order.
"""
import numpy as np
import pytest
import torch

import output_head_kl_b200 as K
import synth
from oracle import kl as O
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

WIDTHS = (256, 240, 224, 192, 160, 128)


def _oracle(x):
    return O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau)


# d = 480: 2 tiles of 256 (the last 224 wide), 2 x 240 exact, 3 of 224 (last 32),
# 3 of 192 (last 96), 3 x 160 exact, 4 of 128 (last 96).
# d = 2880: the large-vocabulary head's width: 12 x 240 exact, 15 x 192 exact,
# 18 x 160 exact, 13 of 224 (last 192), 12 of 256 (last 64), 23 of 128 (last 64).
@pytest.mark.parametrize("N,d,V,Kc", [(1000, 480, 3001, 20), (520, 2880, 2100, 12)])
def test_every_tile_width_matches_oracle_and_each_other(N, d, V, Kc):
    x = synth.custom_inputs(N, d, V, Kc, seed=131 + d, mask_frac=0.05, w_std=0.05, cache="zipf", logit_std=3.0)
    dx = H.to_device(x)
    r = _oracle(x)
    first = None
    for bn in WIDTHS:
        g = H.run_gpu(dx, chunk_tokens=512, options=K.kdkl_options(bwd_tile_n=bn))
        assert g.flags == r.flags
        H.assert_loss(g.loss, r.loss)
        H.assert_grad(g.dH, r.dH, f"dHidden (tile {bn})")
        H.assert_grad(g.dW, r.dW, f"dW (tile {bn})")
        if first is None:
            first = g
        else:
            np.testing.assert_array_equal(g.dH, first.dH, err_msg=f"dHidden, tile {bn} vs 256")
            np.testing.assert_array_equal(g.dW, first.dW, err_msg=f"dW, tile {bn} vs 256")


def test_auto_plan_is_the_reported_plan():
    """The backward with chunk_tokens = 0 runs the plan kdkl_backward_plan reports:
    forcing that tile width and chunk explicitly gives the same bits."""
    x = synth.custom_inputs(1800, 480, 2500, 16, seed=141, mask_frac=0.1, w_std=0.05)
    dx = H.to_device(x)
    N, d = dx.hidden.shape
    V, Kc = dx.W.shape[0], dx.idx.shape[1]
    bn, chunk = K.kdkl_backward_plan(N, d, V, Kc)
    assert bn in WIDTHS and chunk % 128 == 0
    auto = H.run_gpu(dx)
    forced = H.run_gpu(dx, chunk_tokens=chunk, options=K.kdkl_options(bwd_tile_n=bn))
    np.testing.assert_array_equal(auto.dH, forced.dH)
    np.testing.assert_array_equal(auto.dW, forced.dW)
    r = _oracle(x)
    H.assert_grad(auto.dH, r.dH, "dHidden")
    H.assert_grad(auto.dW, r.dW, "dW")


def test_plan_uses_this_device():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for args in [(32768, 4096, 128256, 100), (131072, 2880, 201088, 100), (300, 200, 1001, 7)]:
        assert K.kdkl_backward_plan(*args) == K.kdkl_backward_plan(*args, sm_count=sms)
