"""The data-parallel step's orchestration on CPU ranks (gloo, world size 2).

Each rank runs its shard through stand-in ops built on the CPU oracle (the
kernels need a GPU); the step's collectives and normalisation must then give
exactly the single-process result on the whole batch: the same loss on every
rank, the same all-reduced dW, and each shard's rows of dHidden.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synth
from oracle import kl as O
from output_head_kl_b200 import dp


class OracleOps:
    """Stand-in for the kernels: the oracle on this rank's shard, same contract as the
    library (count; loss and gradients normalised by the count passed in)."""

    def __init__(self, x):
        self.x = x

    def count(self, hidden, W, idx, logit, mask, tau):
        r = O.kl_loss(self.x.hidden_bits, self.x.W_bits, self.x.topk_idx, self.x.topk_logit, self.x.mask, tau,
                      want_grads=False)
        self.nv = r.n_valid
        return torch.tensor([r.n_valid], dtype=torch.int32), None

    def forward(self, hidden, W, idx, logit, mask, tau, ws, n_valid_global):
        r = O.kl_loss(self.x.hidden_bits, self.x.W_bits, self.x.topk_idx, self.x.topk_logit, self.x.mask, tau,
                      want_grads=False)
        scale = (self.nv / int(n_valid_global.item())) if self.nv else 0.0   # the oracle uses the local count
        return torch.tensor([r.loss * scale], dtype=torch.float64), torch.tensor(r.lse)

    def backward(self, hidden, W, idx, logit, mask, tau, lse, ws, n_valid_global):
        r = O.kl_loss(self.x.hidden_bits, self.x.W_bits, self.x.topk_idx, self.x.topk_logit, self.x.mask, tau)
        scale = (self.nv / int(n_valid_global.item())) if self.nv else 0.0
        return torch.tensor(r.dH * scale), torch.tensor(r.dW * scale)


def _shard(x, rank, world):
    n = x.hidden_bits.shape[0]
    sl = slice(rank * n // world, (rank + 1) * n // world)
    return synth.Inputs(x.hidden_bits[sl], x.W_bits, x.topk_idx[sl], x.topk_logit[sl], x.mask[sl], x.tau)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = synth.custom_inputs(37, 16, 101, 6, seed=81, mask_frac=0.2, w_std=0.3)
        x.mask[:18] = 1 - x.mask[:18] * 0   # rank 0's shard gets a different valid count than rank 1's
        x.mask[2:9] = 0
        s = _shard(x, rank, world)
        res = dp.dp_step(None, None, None, None, None, x.tau, ops=OracleOps(s))
        out[rank] = (float(res.loss.item()), res.dW.numpy().copy(), res.dHidden.numpy().copy(),
                     int(res.n_valid_global.item()))
    finally:
        dist.destroy_process_group()


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_dp_step_equals_single_process():
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_worker, args=(2, _port(), out), nprocs=2, join=True, start_method="spawn")
    x = synth.custom_inputs(37, 16, 101, 6, seed=81, mask_frac=0.2, w_std=0.3)
    x.mask[:18] = 1 - x.mask[:18] * 0
    x.mask[2:9] = 0
    full = O.kl_loss(x.hidden_bits, x.W_bits, x.topk_idx, x.topk_logit, x.mask, x.tau)
    (l0, dW0, dH0, n0), (l1, dW1, dH1, n1) = out[0], out[1]
    assert n0 == n1 == full.n_valid
    assert abs(l0 - full.loss) < 1e-12 and l0 == l1
    np.testing.assert_allclose(dW0, full.dW, rtol=1e-12, atol=1e-18)
    np.testing.assert_array_equal(dW0, dW1)
    np.testing.assert_allclose(np.concatenate([dH0, dH1]), full.dH, rtol=1e-12, atol=1e-18)


def _bucket_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(1000 + rank)
        base = torch.randn(101, 16, generator=g, dtype=torch.float32)
        whole = base.clone()
        dist.all_reduce(whole)
        res = {}
        for buckets in (1, 3, 7, 500):
            t = base.clone()
            work = dp.allreduce_dw_buckets(t, buckets)
            slices = [sl for sl, _ in work]
            for _, w in work:
                w.wait()
            res[buckets] = (t.numpy().copy(), [(sl.start, sl.stop) for sl in slices])
        # the step itself, with the reduction left pending and then completed by the caller
        x = synth.custom_inputs(37, 16, 101, 6, seed=81, mask_frac=0.2, w_std=0.3)
        s = _shard(x, rank, world)
        one = dp.dp_step(None, None, None, None, None, x.tau, ops=OracleOps(s))
        pend = dp.dp_step(None, None, None, None, None, x.tau, ops=OracleOps(s), dw_buckets=4, wait_dw=False)
        n_pending = len(pend.dw_work)
        for _, w in pend.dw_work:
            w.wait()
        out[rank] = (whole.numpy().copy(), res, one.dW.numpy().copy(), pend.dW.numpy().copy(), n_pending)
    finally:
        dist.destroy_process_group()


def test_bucketed_dw_reduction_equals_one_all_reduce():
    """dW reduced in slices of vocabulary rows (asynchronous collectives, one per slice)
    equals one all-reduce of the whole tensor; the slices partition the rows in order; and
    a step that leaves the slices pending gives the same dW once the caller waits."""
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_bucket_worker, args=(2, _port(), out), nprocs=2, join=True, start_method="spawn")
    for rank in (0, 1):
        whole, res, dw_one, dw_pend, n_pending = out[rank]
        for buckets, (t, slices) in res.items():
            np.testing.assert_array_equal(t, whole, err_msg=f"buckets={buckets}")
            assert slices[0][0] == 0 and slices[-1][1] == 101
            assert all(a[1] == b[0] for a, b in zip(slices, slices[1:]))
            assert len(slices) == min(buckets, 101)
        assert n_pending == 4
        np.testing.assert_array_equal(dw_pend, dw_one)
    np.testing.assert_array_equal(out[0][0], out[1][0])
