"""Peak device memory of forward + backward is linear in N with no N x V term.

Shapes of the long-context sweep (d = 4096, V = 128,256, K = 100), the workload
on which the paper's output-head benchmark runs from 4K to 256K tokens.

All buffers (inputs, outputs, workspace) come from torch, so
torch.cuda.max_memory_allocated sees every byte the path uses.  With the
chunk buffer fixed (chunk_tokens), the peak must follow a + b N exactly, and
b must be far below the V * 2 bytes per token that even a bf16 N x V logit
buffer would add (256 KB per token here).
"""
import numpy as np
import pytest
import torch

import output_head_kl_b200 as K
import synth
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

D, V, KC = 4096, 128256, 100
NS = (4096, 16384, 65536)


@pytest.fixture(scope="module")
def inputs():
    # one draw at the largest N; smaller N take its leading rows (the peak does not
    # depend on the values)
    return synth.custom_inputs(max(NS), D, V, KC, seed=400, cache="zipf", logit_std=3.0, mask_frac=0.05)


def _rows(x, N):
    return synth.Inputs(x.hidden_bits[:N], x.W_bits, x.topk_idx[:N], x.topk_logit[:N], x.mask[:N], x.tau)


def _peak(x, chunk):
    N = x.hidden_bits.shape[0]
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    dx = H.to_device(x)
    ws = torch.empty(K.kdkl_workspace_bytes(N, D, V, KC, chunk), dtype=torch.uint8, device="cuda")
    loss = torch.empty(1, device="cuda")
    lse = torch.empty(N, device="cuda")
    dH = torch.empty(N, D, dtype=torch.bfloat16, device="cuda")
    dW = torch.empty(V, D, dtype=torch.float32, device="cuda")
    K.kdkl_forward(dx.hidden, dx.W, dx.idx, dx.logit, dx.mask, dx.tau, loss, lse, ws)
    K.kdkl_backward(dx.hidden, dx.W, dx.idx, dx.logit, dx.mask, dx.tau, lse, None, dH, dW, ws, chunk_tokens=chunk)
    torch.cuda.synchronize()
    assert np.isfinite(loss.item())
    assert K.kdkl_read_device_flags(ws) == 0
    peak = torch.cuda.max_memory_allocated() - base
    del dx, ws, loss, lse, dH, dW
    return peak


def test_peak_memory_linear_in_N(inputs):
    Ns = np.array(NS, dtype=float)
    P = np.array([_peak(_rows(inputs, int(n)), chunk=4096) for n in NS], dtype=float)
    b, a = np.polyfit(Ns, P, 1)
    resid = np.abs(P - (a + b * Ns)).max()
    assert resid < 2e6, (P, a, b)                  # affine in N to within allocator rounding
    # bytes per token: hidden + dHidden (4 d), the cache (8 K) and the workspace's
    # per-row lists (8 (K + 4)) plus a few per-row scalars; nothing of order V
    assert b < 4 * D + 16 * KC + 1024, b
    assert b < 2 * V / 10, b
    # the bench's default chunk capacity (8192 tokens) keeps the same slope
    P2 = np.array([_peak(_rows(inputs, n), chunk=0) for n in (16384, 65536)], dtype=float)
    b2 = (P2[1] - P2[0]) / (65536 - 16384)
    assert abs(b2 - b) < 128, (b, b2)          # allocator rounding (2 MB) over 49,152 tokens
