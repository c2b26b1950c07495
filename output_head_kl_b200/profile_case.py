"""Runs one phase of the loss on seeded inputs, for kernel profilers (ncu) to capture.

    python -m output_head_kl_b200.profile_case --config 8b --phase fwd [--N n] [--reps r]

Phases: ``fwd`` (kdkl_forward), ``bwd`` (kdkl_backward, after one untimed forward),
``step`` (both), ``fused`` (kdkl_forward_backward), ``topk`` (kdkl_teacher_topk).
Only the buffers the phase needs are allocated, so that a capture of a
full-size launch keeps a small device footprint: the 8B-class forward holds
about 1.4 GB (hidden, W, the cache and the forward's part of the workspace);
its backward at N = 8192 (one chunk of the full-size chunk length) about 5.5 GB.
Each phase runs ``--warmup`` times, then ``--reps`` times, then synchronises.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main(argv=None) -> int:
    import torch

    import output_head_kl_b200 as K
    import synth

    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="8b", choices=sorted(synth.CONFIGS))
    ap.add_argument("--N", type=int, default=None)
    ap.add_argument("--phase", default="fwd", choices=["fwd", "bwd", "step", "fused", "topk"])
    ap.add_argument("--warmup", type=int, default=1)
    ap.add_argument("--reps", type=int, default=1)
    ap.add_argument("--chunk-tokens", type=int, default=0)
    a = ap.parse_args(argv)
    w = synth.CONFIGS[a.config]
    x = synth.make_inputs(w, N=a.N)
    N, d, V, Kc = x.shape
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    hidden, W = bf16(x.hidden_bits), bf16(x.W_bits)
    if a.phase == "topk":
        ws = torch.empty(K.kdkl_teacher_topk_workspace_bytes(N, d, V, Kc), dtype=torch.uint8, device=dev)
        idx = torch.empty(N, Kc, dtype=torch.int32, device=dev)
        val = torch.empty(N, Kc, dtype=torch.float32, device=dev)
        run = [lambda: K.kdkl_teacher_topk(hidden, W, Kc, idx, val, ws)]
    else:
        idx, logit = torch.from_numpy(x.topk_idx).to(dev), torch.from_numpy(x.topk_logit).to(dev)
        mask = torch.from_numpy(x.mask).to(dev)
        loss = torch.empty(1, dtype=torch.float32, device=dev)
        lse = torch.empty(N, dtype=torch.float32, device=dev)
        if a.phase == "fwd":
            # the forward only touches the workspace before the backward's chunk buffer
            ws_bytes = K.kdkl_workspace_bytes(N, d, V, Kc, 128)
        elif a.phase == "fused":
            ws_bytes = K.kdkl_forward_backward_workspace_bytes(N, d, V, Kc, a.chunk_tokens)
        else:
            ws_bytes = K.kdkl_workspace_bytes(N, d, V, Kc, a.chunk_tokens)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        fwd = lambda: K.kdkl_forward(hidden, W, idx, logit, mask, x.tau, loss, lse, ws)
        if a.phase == "fwd":
            run = [fwd]
        else:
            dH = torch.empty(N, d, dtype=torch.bfloat16, device=dev)
            dW = torch.empty(V, d, dtype=torch.float32, device=dev)
            bwd = lambda: K.kdkl_backward(hidden, W, idx, logit, mask, x.tau, lse, None, dH, dW, ws,
                                          chunk_tokens=a.chunk_tokens)
            if a.phase == "bwd":
                fwd()
                run = [bwd]
            elif a.phase == "step":
                run = [fwd, bwd]
            else:
                run = [lambda: K.kdkl_forward_backward(hidden, W, idx, logit, mask, x.tau, loss, lse, dH, dW, ws,
                                                       chunk_tokens=a.chunk_tokens)]
    for _ in range(a.warmup + a.reps):
        for f in run:
            f()
    torch.cuda.synchronize()
    flags = K.kdkl_read_device_flags(ws)
    print(f"profile_case {a.config} N={N} phase={a.phase} warmup={a.warmup} reps={a.reps} "
          f"device_bytes={torch.cuda.max_memory_allocated(dev) / 1e9:.2f}GB flags={flags}")
    return 0 if flags == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
