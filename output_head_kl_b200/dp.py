"""Token-sharded data parallelism for the fused KL loss over torch.distributed.

Each rank holds its own batch of tokens (its shard of the global batch) and a
replica of the output-head weight W.  One step:

1. forward on the local shard, normalised by the local valid-token count;
2. all-reduce the valid-token counts (the library exposes its count on the
   device, so nothing syncs the host); the global loss is the all-reduced sum
   of loss_r * n_r / n_total;
3. backward on the local shard, normalised by the global count (the
   `n_valid_global` option), so the local dW is this shard's term of the
   global gradient and dHidden is already final;
4. all-reduce dW (sum), the one real exchange of the step.

`ops` abstracts the four device calls so that the orchestration can be run
with other implementations (the tests drive it on CPU ranks with gloo).
"""
from __future__ import annotations

import dataclasses

import torch
import torch.distributed as dist


@dataclasses.dataclass
class StepResult:
    loss: torch.Tensor        # [1] global loss (identical on every rank)
    lse: torch.Tensor         # [N_local]
    dHidden: torch.Tensor     # [N_local, d]
    dW: torch.Tensor          # [V, d], all-reduced
    n_valid_global: torch.Tensor


class KernelOps:
    """The kdkl library calls used by one data-parallel step."""

    def __init__(self, chunk_tokens: int = 0, options=None):
        from . import lib
        lib()
        self.chunk_tokens = chunk_tokens
        self.options = options or {}

    def forward(self, hidden, W, idx, logit, mask, tau):
        from . import kdkl_forward_ex, kdkl_options, kdkl_workspace_bytes
        N, d = hidden.shape
        V, K = W.shape[0], idx.shape[1]
        ws = torch.empty(kdkl_workspace_bytes(N, d, V, K, self.chunk_tokens), dtype=torch.uint8,
                         device=hidden.device)
        loss = torch.empty(1, dtype=torch.float32, device=hidden.device)
        lse = torch.empty(N, dtype=torch.float32, device=hidden.device)
        kdkl_forward_ex(hidden, W, idx, logit, mask, tau, loss, lse, ws, kdkl_options(**self.options))
        count = ws[4:8].view(torch.int32).clone()     # the library's N_valid (kdkl_n_valid_device)
        return loss, lse, count, ws

    def backward(self, hidden, W, idx, logit, mask, tau, lse, ws, n_valid_global):
        from . import kdkl_backward_ex, kdkl_options
        N, d = hidden.shape
        V = W.shape[0]
        dH = torch.empty(N, d, dtype=torch.bfloat16, device=hidden.device)
        dW = torch.empty(V, d, dtype=torch.float32, device=hidden.device)
        opts = kdkl_options(n_valid_global=n_valid_global, **self.options)
        kdkl_backward_ex(hidden, W, idx, logit, mask, tau, lse, None, dH, dW, ws, opts,
                         chunk_tokens=self.chunk_tokens)
        return dH, dW


def dp_step(hidden, W, topk_idx, topk_logit, mask, tau, *, ops=None, group=None) -> StepResult:
    """One token-sharded data-parallel forward + backward (see the module docstring)."""
    ops = ops or KernelOps()
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    loss_local, lse, count, ws = ops.forward(hidden, W, topk_idx, topk_logit, mask, tau)
    total = count.clone()
    if world > 1:
        dist.all_reduce(total, op=dist.ReduceOp.SUM, group=group)
    contrib = torch.where(total > 0, loss_local * count.to(loss_local.dtype) / total.clamp(min=1).to(loss_local.dtype),
                          torch.zeros_like(loss_local))
    if world > 1:
        dist.all_reduce(contrib, op=dist.ReduceOp.SUM, group=group)
    dH, dW = ops.backward(hidden, W, topk_idx, topk_logit, mask, tau, lse, ws, total)
    if world > 1:
        dist.all_reduce(dW, op=dist.ReduceOp.SUM, group=group)
    return StepResult(contrib, lse, dH, dW, total)
