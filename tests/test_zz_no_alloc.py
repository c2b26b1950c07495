"""kdkl_forward_noalloc: the forward for callers that cannot allocate device memory.

Callers such as a loss hook that receives only inputs and outputs, or a
runtime that forbids allocations after start-up, cannot give kdkl a
workspace.  This entry point uses a scratch array built into the library
instead.  Its results must equal those of kdkl_forward with a caller
workspace, on two calls in a row (the second must not be disturbed by what
the first left in the shared scratch), and sizes beyond the built-in scratch
must be refused before any launch.

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import output_head_kl_b200 as K
import synth
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


def _forward_with_workspace(dx):
    N, d = dx.hidden.shape
    V, Kc = dx.W.shape[0], dx.idx.shape[1]
    ws = torch.empty(K.kdkl_workspace_bytes(N, d, V, Kc), dtype=torch.uint8, device="cuda")
    loss = torch.empty(1, device="cuda")
    lse = torch.empty(N, device="cuda")
    K.kdkl_forward(dx.hidden, dx.W, dx.idx, dx.logit, dx.mask, dx.tau, loss, lse, ws)
    torch.cuda.synchronize()
    return loss.item(), lse.cpu().numpy().astype(np.float64)


def _forward_noalloc(dx):
    N = dx.hidden.shape[0]
    loss = torch.full((1,), float("nan"), device="cuda")
    lse = torch.full((N,), float("nan"), device="cuda")
    K.kdkl_forward_noalloc(dx.hidden, dx.W, dx.idx, dx.logit, dx.mask, dx.tau, loss, lse)
    torch.cuda.synchronize()
    return loss.item(), lse.cpu().numpy().astype(np.float64)


def test_noalloc_forward_matches_workspace_forward_twice():
    first = synth.custom_inputs(1500, 256, 5000, 16, seed=201, mask_frac=0.05, w_std=0.05)
    second = synth.custom_inputs(2300, 192, 3001, 24, seed=202, tau=2.0, cache="zipf", logit_std=3.0,
                                 mask_frac=0.2, w_std=0.05)
    for x in (first, second):
        dx = H.to_device(x)
        ref_loss, ref_lse = _forward_with_workspace(dx)
        got_loss, got_lse = _forward_noalloc(dx)
        H.assert_loss(got_loss, ref_loss)
        H.assert_lse(got_lse, ref_lse)


def test_noalloc_refuses_sizes_beyond_its_scratch():
    # 30,000 tokens at K = 100 need more than the built-in 32 MiB: refused before any launch
    N, d, V, Kc = 30000, 64, 4096, 100
    x = synth.custom_inputs(N, d, V, Kc, seed=203, w_std=0.05)
    dx = H.to_device(x)
    loss = torch.full((1,), 5.0, device="cuda")
    lse = torch.full((N,), 5.0, device="cuda")
    st = K.kdkl_forward_noalloc(dx.hidden, dx.W, dx.idx, dx.logit, dx.mask, dx.tau, loss, lse, check=False)
    torch.cuda.synchronize()
    assert st == 4  # KDKL_ERR_UNSUPPORTED
    assert "scratch" in K.kdkl_last_error()
    assert loss.item() == 5.0 and bool(torch.all(lse == 5.0))
