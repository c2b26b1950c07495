"""Peak device memory of forward + backward is linear in N with no N x V term.

All buffers (inputs, outputs, workspace) come from torch, so
torch.cuda.max_memory_allocated sees every byte the path uses.  With the
chunk buffer fixed (chunk_tokens), the peak must follow a + b N exactly, and
b must be far below the V * 2 bytes per token an N x V bf16 logit buffer
would add.
"""
import numpy as np
import pytest
import torch

import output_head_kl_b200 as K
import synth
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


def _peak(N, d=512, V=32768, Kc=16, chunk=1024):
    x = synth.custom_inputs(N, d, V, Kc, seed=400 + N, w_std=0.05)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    dx = H.to_device(x)
    ws = torch.empty(K.kdkl_workspace_bytes(N, d, V, Kc, chunk), dtype=torch.uint8, device="cuda")
    loss = torch.empty(1, device="cuda")
    lse = torch.empty(N, device="cuda")
    dH = torch.empty(N, d, dtype=torch.bfloat16, device="cuda")
    dW = torch.empty(V, d, dtype=torch.float32, device="cuda")
    K.kdkl_forward(dx.hidden, dx.W, dx.idx, dx.logit, dx.mask, dx.tau, loss, lse, ws)
    K.kdkl_backward(dx.hidden, dx.W, dx.idx, dx.logit, dx.mask, dx.tau, lse, None, dH, dW, ws, chunk_tokens=chunk)
    torch.cuda.synchronize()
    assert np.isfinite(loss.item())
    peak = torch.cuda.max_memory_allocated() - base
    del dx, ws, loss, lse, dH, dW
    return peak


def test_peak_memory_linear_in_N():
    Ns = np.array([2048, 4096, 8192, 16384], dtype=float)
    P = np.array([_peak(int(n)) for n in Ns], dtype=float)
    b, a = np.polyfit(Ns, P, 1)
    resid = np.abs(P - (a + b * Ns)).max()
    assert resid < 2e6, (P, a, b)            # affine in N to within allocator rounding
    assert b < 4096, b                       # bytes per token: nowhere near V * 2 = 65536
