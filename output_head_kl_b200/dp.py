"""Token-sharded data parallelism for the fused KL loss over torch.distributed.

Each rank holds its own batch of tokens (its shard of the global batch) and a
replica of the output-head weight W.  One step:

1. count the shard's valid tokens (kdkl_count_valid) and all-reduce the counts
   on the device (nothing syncs the host);
2. forward on the shard with the global count as the normaliser
   (kdkl_options.n_valid_global): each rank's loss is its rows' share of the
   global loss, and an all-reduce (sum) gives the global loss;
3. backward on the shard with the same normaliser, so the local dW is this
   shard's term of the global gradient and dHidden is already final;
4. all-reduce dW (sum), the one real exchange of the step; with ``dw_buckets`` > 1
   it runs as that many asynchronous collectives over contiguous slices of
   vocabulary rows, so that a caller who leaves them pending (``wait_dw=False``)
   can update each slice of W as soon as its reduction completes while the later
   slices are still in flight.

All arithmetic of the loss and its normalisation runs in the library; this
module only issues the library calls and the collectives.  `ops` abstracts the
three device calls so that the orchestration can be run with other
implementations (the tests drive it on CPU ranks with gloo).
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
    dW: torch.Tensor          # [V, d], all-reduced (once dw_work has completed)
    n_valid_global: torch.Tensor
    # pending (row slice, work) pairs of dW's reduction when dp_step(wait_dw=False)
    dw_work: list = dataclasses.field(default_factory=list)


class KernelOps:
    """The kdkl library calls used by one data-parallel step."""

    def __init__(self, chunk_tokens: int = 0, options=None):
        from . import lib
        lib()
        self.chunk_tokens = chunk_tokens
        self.options = options or {}

    def count(self, hidden, W, idx, logit, mask, tau):
        """This shard's valid-token count as a device int32 [1] view into the workspace."""
        from . import kdkl_count_valid, kdkl_options, kdkl_workspace_bytes, n_valid_view
        N, d = hidden.shape
        V, K = W.shape[0], idx.shape[1]
        ws = torch.empty(kdkl_workspace_bytes(N, d, V, K, self.chunk_tokens), dtype=torch.uint8,
                         device=hidden.device)
        kdkl_count_valid(idx, logit, mask, tau, V, ws, kdkl_options(**self.options))
        return n_valid_view(ws), ws

    def forward(self, hidden, W, idx, logit, mask, tau, ws, n_valid_global):
        from . import kdkl_forward_ex, kdkl_options
        N = hidden.shape[0]
        loss = torch.empty(1, dtype=torch.float32, device=hidden.device)
        lse = torch.empty(N, dtype=torch.float32, device=hidden.device)
        kdkl_forward_ex(hidden, W, idx, logit, mask, tau, loss, lse, ws,
                        kdkl_options(n_valid_global=n_valid_global, **self.options))
        return loss, lse

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


def allreduce_dw_buckets(dW, buckets: int, group=None) -> list:
    """Starts the sum all-reduce of dW as `buckets` asynchronous collectives over
    contiguous slices of its rows (vocabulary entries), and returns the (row slice, work)
    pairs in row order.  Each element is still summed over the same ranks by one
    collective, so the result equals a single all-reduce of the whole tensor up to the
    order in which the ranks' terms are added (exactly, with two ranks)."""
    V = dW.shape[0]
    buckets = max(1, min(int(buckets), V)) if V else 1
    out = []
    for b in range(buckets):
        rows = slice(b * V // buckets, (b + 1) * V // buckets)
        out.append((rows, dist.all_reduce(dW[rows], op=dist.ReduceOp.SUM, group=group, async_op=True)))
    return out


def dp_step(hidden, W, topk_idx, topk_logit, mask, tau, *, ops=None, group=None, dw_buckets: int = 1,
            wait_dw: bool = True) -> StepResult:
    """One token-sharded data-parallel forward + backward (see the module docstring)."""
    ops = ops or KernelOps()
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    count, ws = ops.count(hidden, W, topk_idx, topk_logit, mask, tau)
    total = count.clone()
    if world > 1:
        dist.all_reduce(total, op=dist.ReduceOp.SUM, group=group)
    loss, lse = ops.forward(hidden, W, topk_idx, topk_logit, mask, tau, ws, total)
    if world > 1:
        dist.all_reduce(loss, op=dist.ReduceOp.SUM, group=group)
    dH, dW = ops.backward(hidden, W, topk_idx, topk_logit, mask, tau, lse, ws, total)
    work = []
    if world > 1:
        if dw_buckets > 1:
            work = allreduce_dw_buckets(dW, dw_buckets, group)
        else:
            dist.all_reduce(dW, op=dist.ReduceOp.SUM, group=group)
    if wait_dw:
        for _, w in work:
            w.wait()
        work = []
    return StepResult(loss, lse, dH, dW, total, work)
