"""Host-side checks of the C ABI: the library loads, exports what the header
declares, sizes its workspace linearly in N, and rejects bad arguments before
any launch.  None of these calls reaches a kernel: each bad argument is
caught by the host checks, which run before the device is touched."""
import ctypes
import os
import re

import pytest

import output_head_kl_b200 as K

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from output_head_kl_b200 import build
    build.build()
    return K.lib()


def test_exports_every_declared_symbol(lib):
    header = open(os.path.join(ROOT, "include", "kdkl.h")).read()
    names = sorted(set(re.findall(r"\b(kdkl_[a-z_]+)\s*\(", header)))
    assert {"kdkl_forward", "kdkl_backward", "kdkl_workspace_bytes", "kdkl_read_device_flags",
            "kdkl_status_string", "kdkl_last_error"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code, name in K.STATUS_NAMES.items():
        assert K.kdkl_status_string(code) == name


def test_workspace_linear_in_N_without_NxV_term(lib):
    d, V, Kc = 4096, 128256, 100
    chunk = 8192
    sizes = [K.kdkl_workspace_bytes(n, d, V, Kc, chunk) for n in (16384, 32768, 65536, 131072)]
    # the chunk buffer is fixed; the remainder grows linearly with N
    diffs = [b - a for a, b in zip(sizes, sizes[1:])]
    per_tok = [diffs[0] / 16384, diffs[1] / 32768, diffs[2] / 65536]
    assert max(per_tok) - min(per_tok) < 1.0
    assert per_tok[0] < 2000          # a few hundred bytes per token, nothing like V * 2
    assert sizes[0] >= chunk * V * 2


def test_workspace_rejects_bad_shapes(lib):
    assert K.kdkl_workspace_bytes(10, 12, 100, 5, 0) == 0        # d % 8
    assert K.kdkl_workspace_bytes(10, 16, 100, 0, 0) == 0        # K < 1
    assert K.kdkl_workspace_bytes(10, 16, 100, 257, 0) == 0      # K > 256
    assert K.kdkl_workspace_bytes(10, 16, 4, 5, 0) == 0          # K > V
    assert K.kdkl_workspace_bytes(-1, 16, 100, 5, 0) == 0
    assert K.kdkl_workspace_bytes(0, 16, 100, 5, 0) > 0


def _fwd(lib, **kw):
    args = dict(hidden=0x10000, W=0x20000, idx=0x30000, logit=0x40000, mask=0x50000, N=256, d=256, V=4096, K=16,
                tau=1.0, loss=0x60000, lse=0x70000, ws=0x80000, ws_bytes=1 << 40)
    args.update(kw)
    return lib.kdkl_forward(args["hidden"], args["W"], args["idx"], args["logit"], args["mask"], args["N"],
                            args["d"], args["V"], args["K"], args["tau"], args["loss"], args["lse"], args["ws"],
                            args["ws_bytes"], None)


def test_forward_argument_checks(lib):
    assert _fwd(lib, hidden=None) == 1
    assert _fwd(lib, ws=None) == 1
    assert _fwd(lib, loss=None) == 1
    assert _fwd(lib, d=12) == 2
    assert _fwd(lib, K=300) == 2
    assert _fwd(lib, tau=0.0) == 2
    assert _fwd(lib, tau=float("nan")) == 2
    assert _fwd(lib, N=-5) == 2
    assert _fwd(lib, hidden=0x10008) == 3
    assert _fwd(lib, ws=0x80010) == 3
    assert _fwd(lib, lse=0x70002) == 3
    assert _fwd(lib, ws_bytes=100) == 5
    assert "workspace" in K.kdkl_last_error()


def test_backward_argument_checks(lib):
    def bwd(**kw):
        a = dict(dH=0x90000, dW=0xA0000, lse=0x70000, chunk=0, ws_bytes=1 << 40)
        a.update(kw)
        return lib.kdkl_backward(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 256, 256, 4096, 16, 1.0, a["lse"],
                                 None, a["dH"], a["dW"], a["chunk"], 0x80000, a["ws_bytes"], None)
    assert bwd(dH=None) == 1
    assert bwd(dW=0xA0004) == 3
    assert bwd(chunk=-1) == 2
    assert bwd(ws_bytes=4096) == 5


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(K, "_lib", None)
    monkeypatch.setattr(K, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError, match="not built"):
        K.lib()


def _dh_waves(N, d, bn, chunk, groups=74, rows=256):
    """Waves of the dHidden GEMM over all chunks: ceil(row tiles x column tiles / CTA pairs) per chunk."""
    nt = -(-d // bn)
    total = 0
    for c0 in range(0, N, chunk):
        nc = min(chunk, N - c0)
        total += -(-(-(-nc // rows) * nt) // groups)
    return total


def test_backward_plan_on_a_148_sm_device(lib):
    # 8B-class head: 32 row tiles x 16 column tiles = 512 tiles = 6.9 waves of 74 pairs per chunk
    assert K.kdkl_backward_plan(32768, 4096, 128256, 100, sm_count=148) == (256, 8192)
    # d = 2880: 12 column tiles of 256; 30 row tiles per chunk give 360 dHidden tiles = 4.9 waves of
    # 74 pairs, where 32 row tiles give 384 tiles = 5.2, i.e. 6 waves (86 against 96 in all)
    assert K.kdkl_backward_plan(131072, 2880, 201088, 100, sm_count=148) == (256, 7680)
    assert _dh_waves(131072, 2880, 256, 7680) == 86 and _dh_waves(131072, 2880, 256, 8192) == 96
    # N below the chunk capacity: one chunk of N rounded up to 128 rows
    assert K.kdkl_backward_plan(300, 200, 1001, 7, sm_count=148)[1] == 384


def test_backward_plan_arguments(lib):
    # an explicit chunk is kept (rounded up to 128 rows, at most N rounded up)
    assert K.kdkl_backward_plan(32768, 4096, 128256, 100, chunk_tokens=1000, sm_count=148)[1] == 1024
    assert K.kdkl_backward_plan(300, 200, 1001, 7, chunk_tokens=5000, sm_count=148)[1] == 384
    # a forced tile width is kept; the chunk is planned for it
    for bn in (256, 240, 224, 192, 160, 128):
        assert K.kdkl_backward_plan(65536, 2880, 201088, 100, options=K.kdkl_options(bwd_tile_n=bn),
                                    sm_count=148)[0] == bn
    tn, ch = ctypes.c_int32(), ctypes.c_int64()
    assert lib.kdkl_backward_plan(100, 64, 100, 10, 0, None, 148, None, ctypes.byref(ch)) == 1
    assert lib.kdkl_backward_plan(100, 60, 100, 10, 0, None, 148, ctypes.byref(tn), ctypes.byref(ch)) == 2
    assert lib.kdkl_backward_plan(100, 64, 100, 10, -1, None, 148, ctypes.byref(tn), ctypes.byref(ch)) == 2
    bad = K.kdkl_options(bwd_tile_n=200)
    assert lib.kdkl_backward_plan(100, 64, 100, 10, 0, ctypes.byref(bad), 148, ctypes.byref(tn),
                                  ctypes.byref(ch)) == 4


@pytest.mark.parametrize("sms", [148, 132, 2])
def test_backward_plan_is_valid_everywhere(lib, sms):
    for N in (1, 127, 256, 1000, 8192, 8193, 50000, 262144):
        for d in (8, 200, 480, 896, 2048, 2880, 3584, 4096, 8192):
            for V in (128, 32768, 201088):
                bn, ch = K.kdkl_backward_plan(N, d, V, min(100, V), sm_count=sms)
                assert bn in (256, 240, 224, 192, 160, 128)
                n_up = -(-N // 128) * 128
                assert ch % 128 == 0 and 128 <= ch <= min(8192, n_up)
                assert K.kdkl_workspace_bytes(N, d, V, min(100, V)) >= K.kdkl_workspace_bytes(N, d, V, min(100, V), ch)


def test_teacher_topk_vocabulary_limit(lib):
    # each vocabulary split of the producer spans at most 255 tiles of 256 columns (16-bit heap
    # indices), with at most floor(1024 / K) splits
    assert K.kdkl_teacher_topk_workspace_bytes(4096, 4096, 522240, 128) > 0
    assert K.kdkl_teacher_topk_workspace_bytes(4096, 4096, 522241, 128) == 0
    assert K.kdkl_teacher_topk_workspace_bytes(4096, 4096, 652800, 100) > 0
    assert K.kdkl_teacher_topk_workspace_bytes(4096, 4096, 652801, 100) == 0
    assert K.kdkl_teacher_topk_workspace_bytes(4096, 4096, 201088, 128) > 0


def test_forward_backward_argument_checks(lib):
    N, d, V, Kc = 256, 256, 4096, 16
    need = K.kdkl_forward_backward_workspace_bytes(N, d, V, Kc)
    # the fused step's workspace is the loss workspace plus the chunk's fp32 logits
    assert need >= K.kdkl_workspace_bytes(N, d, V, Kc) + 256 * V * 4
    assert K.kdkl_forward_backward_workspace_bytes(N, 12, V, Kc) == 0          # d % 8

    def fb(**kw):
        a = dict(loss=0x60000, lse=0x70000, dH=0x90000, dW=0xA0000, chunk=0, ws_bytes=need)
        a.update(kw)
        return lib.kdkl_forward_backward(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, N, d, V, Kc, 1.0, None, None,
                                         a["loss"], a["lse"], a["dH"], a["dW"], a["chunk"], 0x80000, a["ws_bytes"],
                                         None)
    assert fb(loss=None) == 1
    assert fb(dW=0xA0004) == 3
    assert fb(chunk=-1) == 2
    assert fb(ws_bytes=need - 1) == 5 and "workspace" in K.kdkl_last_error()


def test_count_valid_argument_checks(lib):
    N, V, Kc = 256, 4096, 16
    need = K.kdkl_workspace_bytes(N, 8, V, Kc)

    def cv(**kw):
        a = dict(idx=0x30000, logit=0x40000, mask=0x50000, N=N, V=V, K=Kc, tau=1.0, ws=0x80000, ws_bytes=need)
        a.update(kw)
        return lib.kdkl_count_valid(a["idx"], a["logit"], a["mask"], a["N"], a["V"], a["K"], a["tau"], None, a["ws"],
                                    a["ws_bytes"], None)
    assert cv(idx=None) == 1 and cv(mask=None) == 1 and cv(ws=None) == 1
    assert cv(K=0) == 2 and cv(K=V + 1) == 2 and cv(tau=-1.0) == 2 and cv(N=-1) == 2
    assert cv(idx=0x30002) == 3 and cv(ws=0x80040) == 3
    assert cv(ws_bytes=need // 2) == 5 and "workspace" in K.kdkl_last_error()
    # the workspace layout does not depend on d, so the count's workspace serves the forward and backward
    assert need == K.kdkl_workspace_bytes(N, 4096, V, Kc)
