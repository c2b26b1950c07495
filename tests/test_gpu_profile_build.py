"""The profiling build counts cycles and computes exactly what the product build computes.

``_lib/libkdkl_prof.so`` is the library compiled with ``-DKDKL_PROFILE``: its GEMM CTAs
add the SM cycles their TMA producer, MMA issuer and first epilogue warp spend in the
kernel and at their barrier waits to a device counter array.  The counting must not
change a result (same kernels, same order of every floating-point operation), and
the counts must be consistent with the launches that made them: every tile the MMA
issuers count is one the epilogues count once per CTA of the issuing pair, a wait is
never longer than its role's total, and no kernel runs above the tcgen05 bf16 rate of
8192 flops per SM cycle.
"""
import numpy as np
import pytest
import torch

import output_head_kl_b200 as K
import synth
from output_head_kl_b200 import profile_roles
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

SHAPE = dict(N=5000, d=1024, V=20000, K=24)
CHUNK = 2048


def _inputs():
    return synth.custom_inputs(SHAPE["N"], SHAPE["d"], SHAPE["V"], SHAPE["K"], seed=733, cache="zipf",
                               logit_std=3.0, mask_frac=0.05, w_std=0.05)


def _use_profiling_library(monkeypatch):
    monkeypatch.setattr(K, "LIB_PATH", K.PROFILE_LIB_PATH)
    monkeypatch.setattr(K, "_lib", None)
    assert K.lib()._name == K.PROFILE_LIB_PATH


def test_profiling_build_is_bit_identical_and_counts_consistently(monkeypatch):
    x = _inputs()
    dx = H.to_device(x)
    base = H.run_gpu(dx, chunk_tokens=CHUNK)
    assert base.flags == 0

    _use_profiling_library(monkeypatch)
    K.kdkl_profile_role_cycles_clear()
    got = H.run_gpu(dx, chunk_tokens=CHUNK)
    counters = K.kdkl_profile_role_cycles_read()
    assert got.flags == 0
    assert got.loss == base.loss
    for name in ("lse", "dH", "dW"):
        np.testing.assert_array_equal(getattr(got, name), getattr(base, name), err_msg=name)

    N, d, V = SHAPE["N"], SHAPE["d"], SHAPE["V"]
    c = counters.astype(np.int64)
    for kind in (0, 1, 2, 3):   # forward, gradient, dHidden, dW all ran
        ck = c[kind]
        issuers = ck[ck[:, 0] > 0]
        ctas = ck[ck[:, 4] > 0]
        assert len(issuers) > 0 and len(ctas) > 0, kind
        per = len(ctas) // len(issuers)
        assert per in (1, 2) and len(ctas) == per * len(issuers), kind
        # waits within totals, for every role of every CTA
        for tot, waits in ((0, (1, 2)), (4, (5, 6)), (8, (9,))):
            for wcol in waits:
                assert (ck[:, wcol] <= ck[:, tot]).all(), (kind, wcol)
        # the epilogue warps of a pair see each tile its issuer counted
        assert ck[:, 11].sum() == per * issuers[:, 3].sum(), kind
    # the forward's tiles: every (row block, 256-column tile) once
    rows = 256 if len(c[0][c[0][:, 4] > 0]) == 2 * len(c[0][c[0][:, 0] > 0]) else 128
    assert c[0][:, 3].sum() == -(-N // rows) * -(-V // 256)
    # no kernel above the tensor pipe's rate
    s = profile_roles.summarise(counters, 2.0 * N * d * V)
    assert set(s) >= {"fwd_lse", "bwd_grad", "bwd_dhidden", "bwd_dw"}
    for name, r in s.items():
        assert 0 < r["flops_per_sm_cycle"] <= 8192 * 1.02, (name, r)
        assert 0 <= r["mma_wait_accumulator"] <= 1 and 0 <= r["mma_wait_operands"] <= 1


def test_counters_clear_and_refuse_a_wrong_size(monkeypatch):
    _use_profiling_library(monkeypatch)
    K.kdkl_profile_role_cycles_clear()
    torch.cuda.synchronize()
    assert not K.kdkl_profile_role_cycles_read().any()
    st = K.lib().kdkl_profile_read_role_cycles(np.zeros(4, dtype=np.uint64).ctypes.data, 32)
    assert st == 2   # KDKL_ERR_SHAPE
