"""Token-sharded data parallelism with the real kernels, on one GPU.

Two spawned ranks, both on cuda:0, run `dp.dp_step` on their halves of one
batch with gloo collectives (the exchanges pass through the host; no kernel
waits on the other rank).  The result must be the single-process step on the
whole batch: the same valid count and loss on both ranks, the same all-reduced
dW on both ranks (bit for bit) and equal to the whole-batch dW, and each
rank's dHidden rows equal to the whole-batch rows.  dW reduced in slices of
vocabulary rows, left pending by the step and completed by the caller, must equal
the one-collective dW bit for bit.  Per-row results can differ
from the whole-batch run only by rounding, because the forward's vocabulary
split count (and so the order of its log-sum-exp merge) depends on the batch
size.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synth
from output_head_kl_b200 import dp
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

SHAPE = dict(N=600, d=256, V=3001, K=16)


def _inputs():
    x = synth.custom_inputs(SHAPE["N"], SHAPE["d"], SHAPE["V"], SHAPE["K"], seed=171, mask_frac=0.1, w_std=0.05,
                            cache="zipf", logit_std=3.0)
    x.mask[:40] = 0          # the two halves get different valid counts
    return x


def _half(x, rank):
    n = x.hidden_bits.shape[0] // 2
    sl = slice(rank * n, (rank + 1) * n)
    return synth.Inputs(x.hidden_bits[sl], x.W_bits, x.topk_idx[sl], x.topk_logit[sl], x.mask[sl], x.tau)


def _step(x, **kw):
    d = H.to_device(x)
    r = dp.dp_step(d.hidden, d.W, d.idx, d.logit, d.mask, d.tau, **kw)
    for _, w in r.dw_work:       # a bucketed reduction left pending: the caller completes it
        w.wait()
    torch.cuda.synchronize()
    return (float(r.loss.item()), r.dW.cpu().numpy().astype(np.float64), r.dHidden.float().cpu().numpy(),
            int(r.n_valid_global.item()))


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        out[rank] = _step(_half(_inputs(), rank))
        # dW reduced in 5 slices of vocabulary rows, left pending by the step
        out[10 + rank] = _step(_half(_inputs(), rank), dw_buckets=5, wait_dw=False)[1]
    finally:
        dist.destroy_process_group()


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_equal_one_process():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_worker, args=(2, _port(), out), nprocs=2, join=True, start_method="spawn")
    (l0, dW0, dH0, n0), (l1, dW1, dH1, n1) = out[0], out[1]
    loss, dW, dH, n = _step(_inputs())            # this process, no process group: the whole batch
    assert n0 == n1 == n == int(_inputs().mask.sum())
    assert l0 == l1
    assert abs(l0 - loss) <= 1e-5 * abs(loss)
    np.testing.assert_array_equal(dW0, dW1)
    np.testing.assert_array_equal(out[10], dW0)   # the bucketed reduction gives the same dW
    np.testing.assert_array_equal(out[11], dW1)
    assert np.abs(dW0 - dW).max() <= 1e-3 * np.abs(dW).max()
    dH_ranks = np.concatenate([dH0, dH1])
    assert np.abs(dH_ranks - dH).max() <= 1e-3 * np.abs(dH).max()
    assert np.all(dH_ranks[:40] == 0)              # masked rows
