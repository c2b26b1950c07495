"""Failure detection on the GPU without a GPU fault: a bounded wait runs out.

The kernels' every wait gives up after a limit, records KDKL_DEV_TIMEOUT and
returns.  The self-test waits through the same routine on a barrier that
nothing completes; the host must then read the timeout bit, the wait must
have lasted about the limit, and the context must still run the loss."""
import numpy as np
import pytest
import torch

import output_head_kl_b200 as K
import synth
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_stays_usable():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    limit = 20_000_000   # 20 ms
    K.kdkl_selftest_wait_timeout(ws, limit)
    flags = K.kdkl_read_device_flags(ws)
    assert flags == K.DEV_TIMEOUT
    waited = int(ws[8:16].cpu().numpy().view(np.uint64)[0])
    assert limit <= waited < limit + 50_000_000
    x = synth.make_inputs(synth.CONFIGS["tiny"])
    g = H.run_gpu(H.to_device(x))
    assert g.flags == 0 and np.isfinite(g.loss)


def test_selftest_rejects_bad_limits():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(K.KDKLError):
        K.kdkl_selftest_wait_timeout(ws, 10)
