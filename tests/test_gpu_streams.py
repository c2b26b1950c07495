"""Determinism and stream semantics of the C ABI on the GPU.

Every reduction in the path has a fixed order (register-resident per-row
sums, fixed-order block trees and final sums, dW read-modify-written in chunk
order, no floating-point atomics), so repeating a call must reproduce every
output bit for bit.  Calls are asynchronous on the caller's stream, so two
independent problems on two streams must each give their own single-stream
result."""
import numpy as np
import pytest
import torch

import output_head_kl_b200 as K
import synth
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


def _run(dx, stream, chunk=256):
    N, d = dx.hidden.shape
    V, Kc = dx.W.shape[0], dx.idx.shape[1]
    with torch.cuda.stream(stream):
        ws = torch.empty(K.kdkl_workspace_bytes(N, d, V, Kc, chunk), dtype=torch.uint8, device="cuda")
        loss = torch.empty(1, device="cuda")
        lse = torch.empty(N, device="cuda")
        dH = torch.empty(N, d, dtype=torch.bfloat16, device="cuda")
        dW = torch.empty(V, d, device="cuda")
        K.kdkl_forward(dx.hidden, dx.W, dx.idx, dx.logit, dx.mask, dx.tau, loss, lse, ws, stream=stream)
        K.kdkl_backward(dx.hidden, dx.W, dx.idx, dx.logit, dx.mask, dx.tau, lse, None, dH, dW, ws,
                        chunk_tokens=chunk, stream=stream)
    return loss, lse, dH, dW


def test_bitwise_deterministic():
    x = synth.custom_inputs(1000, 512, 9000, 32, seed=601, cache="zipf", logit_std=3.0, mask_frac=0.05, w_std=0.05)
    dx = H.to_device(x)
    s = torch.cuda.current_stream()
    a = _run(dx, s)
    b = _run(dx, s)
    torch.cuda.synchronize()
    for u, v in zip(a, b):
        assert torch.equal(u, v)


def test_two_streams_give_single_stream_results():
    x1 = synth.custom_inputs(900, 256, 7000, 16, seed=602, mask_frac=0.05, w_std=0.05)
    x2 = synth.custom_inputs(700, 192, 5000, 24, seed=603, mask_frac=0.05, w_std=0.05)
    d1, d2 = H.to_device(x1), H.to_device(x2)
    ref1 = _run(d1, torch.cuda.current_stream())
    ref2 = _run(d2, torch.cuda.current_stream())
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    s1.wait_stream(torch.cuda.current_stream())
    s2.wait_stream(torch.cuda.current_stream())
    o1 = _run(d1, s1)
    o2 = _run(d2, s2)
    torch.cuda.synchronize()
    for u, v in zip(o1, ref1):
        assert torch.equal(u, v)
    for u, v in zip(o2, ref2):
        assert torch.equal(u, v)
