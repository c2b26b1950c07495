"""Where the GEMM kernels' cycles go: the profiling build's role counters.

    python -m output_head_kl_b200.profile_roles --config 8b [--N n] [--phase step|bwd|fused|topk] [--reps r]
                                                [--chunk-tokens c] [--bwd-tile-n w]

Loads ``_lib/libkdkl_prof.so`` (the library compiled with ``-DKDKL_PROFILE``, whose
GEMM CTAs count the SM cycles their roles spend at barrier waits, see
``include/kdkl_profile.h``), runs the phase ``--warmup`` times, clears the counters,
runs it ``--reps`` times and prints one JSON line (``bwd``: one untimed forward, then
the backward alone; ``--bwd-tile-n`` forces the dHidden / dW tile width).  Per GEMM kind:

* ``flops_per_sm_cycle``: the kind's dense flops (2·N·d·V per launch set) over the
  SM cycles of its CTAs (each MMA issuer's cycles times the CTAs it issues for); the
  tcgen05 bf16 rate behind the nominal 2.25 PFLOP/s is 8192 per SM per cycle;
* ``mma_cycles_per_tile`` and the issuer's shares of time waiting for a free
  accumulator (``mma_wait_accumulator``: the epilogue is behind) and for operands
  (``mma_wait_operands``: the TMA producer is behind, or the tensor pipe is full);
* the producer's shares waiting for a free stage and in the lockstep of CTA groups;
* the first epilogue warp's share waiting for a finished accumulator;
* ``mma_cta_spread``: the largest issuer total over the mean (load balance).

Counts are SM cycles (clock64), so the shares do not depend on the clock.
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

KIND_NAMES = {0: "fwd_lse", 1: "bwd_grad", 2: "bwd_dhidden", 3: "bwd_dw", 4: "teacher_topk", 5: "fused_fwd_store"}


def summarise(counters: np.ndarray, flops_per_kind: float) -> dict:
    """Per-kind shares from a [kind, cta, slot] counter array (see include/kdkl_profile.h)."""
    out = {}
    for k in range(counters.shape[0]):
        c = counters[k].astype(np.float64)
        mma = c[c[:, 0] > 0]
        prod = c[c[:, 4] > 0]
        epi = c[c[:, 8] > 0]
        if len(mma) == 0 or len(prod) == 0:
            continue
        ctas_per_issuer = len(prod) / len(mma)
        sm_cycles = mma[:, 0].sum() * ctas_per_issuer
        r = {
            "ctas": int(len(prod)),
            "mma_issuers": int(len(mma)),
            "tiles": int(mma[:, 3].sum()),
            "mma_cycles_per_tile": mma[:, 0].sum() / max(1.0, mma[:, 3].sum()),
            "mma_wait_accumulator": mma[:, 1].sum() / mma[:, 0].sum(),
            "mma_wait_operands": mma[:, 2].sum() / mma[:, 0].sum(),
            "mma_cta_spread": mma[:, 0].max() / mma[:, 0].mean(),
            "producer_wait_stage": prod[:, 5].sum() / prod[:, 4].sum(),
            "producer_wait_lockstep": prod[:, 6].sum() / prod[:, 4].sum(),
            "epilogue_wait_accumulator": (epi[:, 9].sum() / epi[:, 8].sum()) if len(epi) else None,
            "flops_per_sm_cycle": flops_per_kind / sm_cycles if sm_cycles > 0 else None,
        }
        out[KIND_NAMES.get(k, str(k))] = {a: (round(b, 4) if isinstance(b, float) else b) for a, b in r.items()}
    return out


def main(argv=None) -> int:
    import torch

    import output_head_kl_b200 as K
    import synth

    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="8b", choices=sorted(synth.CONFIGS))
    ap.add_argument("--N", type=int, default=None)
    ap.add_argument("--phase", default="step", choices=["step", "bwd", "fused", "topk"])
    ap.add_argument("--chunk-tokens", type=int, default=0)
    ap.add_argument("--bwd-tile-n", type=int, default=0)
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--reps", type=int, default=1)
    a = ap.parse_args(argv)

    K.LIB_PATH = K.PROFILE_LIB_PATH
    K.lib()
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
        ti = torch.empty(N, Kc, dtype=torch.int32, device=dev)
        tv = torch.empty(N, Kc, dtype=torch.float32, device=dev)

        def run():
            K.kdkl_teacher_topk(hidden, W, Kc, ti, tv, ws)
    else:
        idx, logit = torch.from_numpy(x.topk_idx).to(dev), torch.from_numpy(x.topk_logit).to(dev)
        mask = torch.from_numpy(x.mask).to(dev)
        loss = torch.empty(1, dtype=torch.float32, device=dev)
        lse = torch.empty(N, dtype=torch.float32, device=dev)
        dH = torch.empty(N, d, dtype=torch.bfloat16, device=dev)
        dW = torch.empty(V, d, dtype=torch.float32, device=dev)
        opts = K.kdkl_options(bwd_tile_n=a.bwd_tile_n)
        ch = a.chunk_tokens
        if a.phase == "fused":
            ws = torch.empty(K.kdkl_forward_backward_workspace_bytes(N, d, V, Kc, ch), dtype=torch.uint8, device=dev)

            def run():
                K.kdkl_forward_backward(hidden, W, idx, logit, mask, x.tau, loss, lse, dH, dW, ws, opts,
                                        chunk_tokens=ch)
        else:
            ws = torch.empty(K.kdkl_workspace_bytes(N, d, V, Kc, ch), dtype=torch.uint8, device=dev)

            def fwd():
                K.kdkl_forward_ex(hidden, W, idx, logit, mask, x.tau, loss, lse, ws, opts)

            def bwd():
                K.kdkl_backward_ex(hidden, W, idx, logit, mask, x.tau, lse, None, dH, dW, ws, opts, chunk_tokens=ch)

            if a.phase == "bwd":
                fwd()
                run = bwd
            else:
                def run():
                    fwd()
                    bwd()

    for _ in range(a.warmup):
        run()
    torch.cuda.synchronize()
    K.kdkl_profile_role_cycles_clear()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.reps):
        run()
    e1.record()
    torch.cuda.synchronize()
    counters = K.kdkl_profile_role_cycles_read()
    flags = K.kdkl_read_device_flags(ws)
    rec = {"workload": w.name, "N": N, "d": d, "V": V, "K": Kc, "phase": a.phase, "reps": a.reps,
           "chunk_tokens": a.chunk_tokens, "bwd_tile_n": a.bwd_tile_n,
           "ms_per_rep": e0.elapsed_time(e1) / a.reps, "device_flags": flags,
           "kinds": summarise(counters, 2.0 * N * d * V * a.reps)}
    print(json.dumps(rec), flush=True)
    return 0 if flags == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
