"""Host side of the profiling build: it exports its header's entry points (and all of
kdkl.h), the product library does not carry the counters, and the report turns a
counter array into the shares it claims to give."""
import ctypes
import os
import re

import numpy as np

import output_head_kl_b200 as K
from output_head_kl_b200 import build, profile_roles

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared(header):
    text = open(os.path.join(ROOT, "include", header)).read()
    return sorted(set(re.findall(r"\b(kdkl_[a-z_]+)\s*\(", text)))


def test_profiling_library_exports_both_headers():
    build.build()
    prof = ctypes.CDLL(build.PROFILE_LIB)
    names = _declared("kdkl_profile.h")
    assert names == ["kdkl_profile_clear_role_cycles", "kdkl_profile_read_role_cycles",
                     "kdkl_profile_role_cycles_shape"]
    for n in names + _declared("kdkl.h"):
        assert hasattr(prof, n), n
    product = ctypes.CDLL(build.LIB)
    assert not any(hasattr(product, n) for n in names)


def test_shape_query_needs_no_device():
    prof = ctypes.CDLL(build.PROFILE_LIB)
    k, c, s = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    assert prof.kdkl_profile_role_cycles_shape(ctypes.byref(k), ctypes.byref(c), ctypes.byref(s)) == K.KDKL_OK
    assert (k.value, c.value, s.value) == (8, 256, 12)
    assert prof.kdkl_profile_role_cycles_shape(None, ctypes.byref(c), ctypes.byref(s)) == 1   # KDKL_ERR_NULL


def test_summary_of_a_made_up_pair_launch():
    # two pairs (4 CTAs): issuers are CTAs 0 and 2; 10 tiles each of 1000 cycles
    c = np.zeros((8, 256, 12), dtype=np.uint64)
    for cta in range(4):
        c[2, cta, 4:8] = (10_000, 1_000, 500, 3)          # producer: total, stage, lockstep, units
        c[2, cta, 8:12] = (10_000, 2_500, 0, 10)          # epilogue: total, wait, -, tiles
    c[2, 0, 0:4] = (10_000, 200, 1_800, 10)               # issuer: total, accumulator, operands, tiles
    c[2, 2, 0:4] = (12_000, 0, 3_000, 10)
    s = profile_roles.summarise(c, flops_per_kind=2.2e8)
    assert list(s) == ["bwd_dhidden"]
    r = s["bwd_dhidden"]
    assert (r["ctas"], r["mma_issuers"], r["tiles"]) == (4, 2, 20)
    assert r["mma_cycles_per_tile"] == 1100.0
    assert r["mma_wait_accumulator"] == round(200 / 22_000, 4)
    assert r["mma_wait_operands"] == round(4_800 / 22_000, 4)
    assert r["mma_cta_spread"] == round(12_000 / 11_000, 4)
    assert r["producer_wait_stage"] == 0.1 and r["producer_wait_lockstep"] == 0.05
    assert r["epilogue_wait_accumulator"] == 0.25
    assert r["flops_per_sm_cycle"] == 5000.0             # 2.2e8 / (22_000 cycles x 2 CTAs)
