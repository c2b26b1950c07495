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
