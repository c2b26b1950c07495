"""Python binding of the kdkl C ABI (``include/kdkl.h``): argument marshalling only.

Every step of the loss runs in the CUDA library ``_lib/libkdkl.so``; this module
turns torch tensors into pointers and status codes into exceptions.  There is
no fallback: if the library is missing, importing a function that needs it
raises.

Names mirror the C entry points: ``kdkl_workspace_bytes``, ``kdkl_forward``,
``kdkl_backward``, ``kdkl_forward_ex``, ``kdkl_backward_ex`` (with ``kdkl_options``),
``kdkl_forward_noalloc``, ``kdkl_teacher_topk``, ``kdkl_count_valid``, ``kdkl_read_device_flags``, ``kdkl_timing_enable``,
``kdkl_timing_read``, ``kdkl_status_string``, ``kdkl_last_error``; with the profiling build loaded,
``kdkl_profile_role_cycles_read`` / ``kdkl_profile_role_cycles_clear`` (``include/kdkl_profile.h``).
``fused_kl_forward_backward`` is a convenience wrapper
that allocates the outputs and the workspace with torch (the library itself
never allocates).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libkdkl.so")
# The same library with in-kernel index checks (KDKL_DEV_BOUNDS); see build.py.
DEBUG_LIB_PATH = os.path.join(_HERE, "_lib", "libkdkl_debug.so")
# The same library with per-role cycle counters in the GEMM kernels; see build.py.
PROFILE_LIB_PATH = os.path.join(_HERE, "_lib", "libkdkl_prof.so")

KDKL_OK = 0
STATUS_NAMES = {0: "KDKL_OK", 1: "KDKL_ERR_NULL", 2: "KDKL_ERR_SHAPE", 3: "KDKL_ERR_ALIGN",
                4: "KDKL_ERR_UNSUPPORTED", 5: "KDKL_ERR_WORKSPACE", 6: "KDKL_ERR_CUDA"}
DEV_IDX_RANGE, DEV_IDX_DUP, DEV_NONFINITE, DEV_TIMEOUT, DEV_BOUNDS = 1, 2, 4, 8, 16

_lib = None


class KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_uint64), ("total_ms", ctypes.c_double)]


CACHE_I32_F32, CACHE_U16_BF16 = 0, 1


class Options(ctypes.Structure):
    """kdkl_options: cache format and loss-design variant (see include/kdkl.h)."""
    _fields_ = [("cache_format", ctypes.c_int32), ("student_tau", ctypes.c_float), ("kd_weight", ctypes.c_float),
                ("kd_scale_tau_sq", ctypes.c_int32), ("ce_weight", ctypes.c_float), ("labels", ctypes.c_void_p),
                ("n_valid_global", ctypes.c_void_p), ("bwd_tile_n", ctypes.c_int32)]


def kdkl_options(cache_format=CACHE_I32_F32, student_tau=1.0, kd_weight=1.0, kd_scale_tau_sq=False,
                 ce_weight=0.0, labels=None, n_valid_global=None, bwd_tile_n=0) -> Options:
    o = Options()
    lib().kdkl_options_init(ctypes.byref(o))
    o.cache_format = int(cache_format)
    o.student_tau = float(student_tau)
    o.kd_weight = float(kd_weight)
    o.kd_scale_tau_sq = 1 if kd_scale_tau_sq else 0
    o.ce_weight = float(ce_weight)
    o.labels = _ptr(labels)
    o.n_valid_global = _ptr(n_valid_global)
    o.bwd_tile_n = int(bwd_tile_n)
    # the struct holds raw device addresses: keep the tensors alive as long as it lives
    o._keep = (labels, n_valid_global)
    return o


class KDKLError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {detail}")
        self.status = status


def lib() -> ctypes.CDLL:
    """Loads the in-tree CUDA library (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"kdkl CUDA library not built: {LIB_PATH} is missing "
                           "(run `python -m output_head_kl_b200.build`)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, f32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    L.kdkl_workspace_bytes.argtypes = [i64, i32, i32, i32, i64]
    L.kdkl_workspace_bytes.restype = sz
    L.kdkl_forward.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, i32, f32, vp, vp, vp, sz, vp]
    L.kdkl_forward.restype = ctypes.c_int
    L.kdkl_backward.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, i32, f32, vp, vp, vp, vp, i64, vp, sz, vp]
    L.kdkl_backward.restype = ctypes.c_int
    L.kdkl_read_device_flags.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
    L.kdkl_read_device_flags.restype = ctypes.c_int
    L.kdkl_status_string.argtypes = [ctypes.c_int]
    L.kdkl_status_string.restype = ctypes.c_char_p
    L.kdkl_last_error.argtypes = []
    L.kdkl_last_error.restype = ctypes.c_char_p
    L.kdkl_options_init.argtypes = [ctypes.POINTER(Options)]
    L.kdkl_options_init.restype = None
    L.kdkl_forward_ex.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, i32, f32, ctypes.POINTER(Options), vp, vp, vp,
                                  sz, vp]
    L.kdkl_forward_ex.restype = ctypes.c_int
    L.kdkl_backward_ex.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, i32, f32, ctypes.POINTER(Options), vp, vp, vp,
                                   vp, i64, vp, sz, vp]
    L.kdkl_backward_ex.restype = ctypes.c_int
    L.kdkl_forward_backward_workspace_bytes.argtypes = [i64, i32, i32, i32, i64]
    L.kdkl_forward_backward_workspace_bytes.restype = sz
    L.kdkl_forward_backward.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, i32, f32, ctypes.POINTER(Options), vp, vp,
                                        vp, vp, vp, i64, vp, sz, vp]
    L.kdkl_forward_backward.restype = ctypes.c_int
    L.kdkl_teacher_topk_workspace_bytes.argtypes = [i64, i32, i32, i32]
    L.kdkl_teacher_topk_workspace_bytes.restype = sz
    L.kdkl_teacher_topk.argtypes = [vp, vp, i64, i32, i32, i32, vp, vp, vp, sz, vp]
    L.kdkl_teacher_topk.restype = ctypes.c_int
    L.kdkl_n_valid_device.argtypes = [vp]
    L.kdkl_n_valid_device.restype = ctypes.c_void_p
    L.kdkl_count_valid.argtypes = [vp, vp, vp, i64, i32, i32, f32, ctypes.POINTER(Options), vp, sz, vp]
    L.kdkl_count_valid.restype = ctypes.c_int
    L.kdkl_selftest_wait_timeout.argtypes = [vp, ctypes.c_uint64, vp]
    L.kdkl_selftest_wait_timeout.restype = ctypes.c_int
    L.kdkl_timing_enable.argtypes = [ctypes.c_int]
    L.kdkl_timing_enable.restype = ctypes.c_int
    L.kdkl_timing_read.argtypes = [ctypes.POINTER(KernelTime), ctypes.c_int, ctypes.c_int]
    L.kdkl_timing_read.restype = ctypes.c_int
    L.kdkl_backward_plan.argtypes = [i64, i32, i32, i32, i64, ctypes.POINTER(Options), i32,
                                     ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int64)]
    L.kdkl_backward_plan.restype = ctypes.c_int
    if hasattr(L, "kdkl_profile_read_role_cycles"):
        L.kdkl_profile_role_cycles_shape.argtypes = [ctypes.POINTER(ctypes.c_int32)] * 3
        L.kdkl_profile_role_cycles_shape.restype = ctypes.c_int
        L.kdkl_profile_read_role_cycles.argtypes = [vp, sz]
        L.kdkl_profile_read_role_cycles.restype = ctypes.c_int
        L.kdkl_profile_clear_role_cycles.argtypes = [vp]
        L.kdkl_profile_clear_role_cycles.restype = ctypes.c_int
    _lib = L
    return L


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != KDKL_OK:
        raise KDKLError(status, where, kdkl_last_error())


def kdkl_status_string(status: int) -> str:
    return lib().kdkl_status_string(status).decode()


def kdkl_last_error() -> str:
    return lib().kdkl_last_error().decode()


def kdkl_workspace_bytes(N: int, d: int, V: int, K: int, chunk_tokens: int = 0) -> int:
    return int(lib().kdkl_workspace_bytes(N, d, V, K, chunk_tokens))


def kdkl_backward_plan(N: int, d: int, V: int, K: int, chunk_tokens: int = 0, options: Options | None = None,
                       sm_count: int = 0) -> tuple[int, int]:
    """(tile_n, chunk_tokens) the backward uses for these sizes; sm_count 0 = the current device."""
    tn = ctypes.c_int32()
    ch = ctypes.c_int64()
    st = lib().kdkl_backward_plan(int(N), int(d), int(V), int(K), int(chunk_tokens),
                                  ctypes.byref(options) if options is not None else None, int(sm_count),
                                  ctypes.byref(tn), ctypes.byref(ch))
    _check(st, "kdkl_backward_plan")
    return tn.value, ch.value


def kdkl_forward(hidden, W, topk_idx, topk_logit, mask, tau, loss, lse, workspace, *, N=None, d=None, V=None,
                 K=None, workspace_bytes=None, stream=None, check=True) -> int:
    """Calls kdkl_forward.  Tensors (or raw device pointers with explicit sizes)."""
    N = hidden.shape[0] if N is None else N
    d = hidden.shape[1] if d is None else d
    V = W.shape[0] if V is None else V
    K = topk_idx.shape[1] if K is None else K
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    st = lib().kdkl_forward(_ptr(hidden), _ptr(W), _ptr(topk_idx), _ptr(topk_logit), _ptr(mask), int(N), int(d),
                            int(V), int(K), float(tau), _ptr(loss), _ptr(lse), _ptr(workspace), int(wsb),
                            _stream(stream))
    if check:
        _check(st, "kdkl_forward")
    return st


def kdkl_backward(hidden, W, topk_idx, topk_logit, mask, tau, lse, grad_loss, dHidden, dW, workspace, *,
                  chunk_tokens=0, N=None, d=None, V=None, K=None, workspace_bytes=None, stream=None,
                  check=True) -> int:
    """Calls kdkl_backward (grad_loss may be None for g = 1)."""
    N = hidden.shape[0] if N is None else N
    d = hidden.shape[1] if d is None else d
    V = W.shape[0] if V is None else V
    K = topk_idx.shape[1] if K is None else K
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    st = lib().kdkl_backward(_ptr(hidden), _ptr(W), _ptr(topk_idx), _ptr(topk_logit), _ptr(mask), int(N), int(d),
                             int(V), int(K), float(tau), _ptr(lse), _ptr(grad_loss), _ptr(dHidden), _ptr(dW),
                             int(chunk_tokens), _ptr(workspace), int(wsb), _stream(stream))
    if check:
        _check(st, "kdkl_backward")
    return st


def kdkl_forward_ex(hidden, W, topk_idx, topk_logit, mask, tau, loss, lse, workspace, options=None, *, N=None,
                    d=None, V=None, K=None, workspace_bytes=None, stream=None, check=True) -> int:
    """Calls kdkl_forward_ex (options: an ``Options`` from ``kdkl_options(...)`` or None)."""
    N = hidden.shape[0] if N is None else N
    d = hidden.shape[1] if d is None else d
    V = W.shape[0] if V is None else V
    K = topk_idx.shape[1] if K is None else K
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    opt = ctypes.byref(options) if options is not None else None
    st = lib().kdkl_forward_ex(_ptr(hidden), _ptr(W), _ptr(topk_idx), _ptr(topk_logit), _ptr(mask), int(N), int(d),
                               int(V), int(K), float(tau), opt, _ptr(loss), _ptr(lse), _ptr(workspace), int(wsb),
                               _stream(stream))
    if check:
        _check(st, "kdkl_forward_ex")
    return st


def kdkl_backward_ex(hidden, W, topk_idx, topk_logit, mask, tau, lse, grad_loss, dHidden, dW, workspace,
                     options=None, *, chunk_tokens=0, N=None, d=None, V=None, K=None, workspace_bytes=None,
                     stream=None, check=True) -> int:
    """Calls kdkl_backward_ex (same options as the forward)."""
    N = hidden.shape[0] if N is None else N
    d = hidden.shape[1] if d is None else d
    V = W.shape[0] if V is None else V
    K = topk_idx.shape[1] if K is None else K
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    opt = ctypes.byref(options) if options is not None else None
    st = lib().kdkl_backward_ex(_ptr(hidden), _ptr(W), _ptr(topk_idx), _ptr(topk_logit), _ptr(mask), int(N),
                                int(d), int(V), int(K), float(tau), opt, _ptr(lse), _ptr(grad_loss), _ptr(dHidden),
                                _ptr(dW), int(chunk_tokens), _ptr(workspace), int(wsb), _stream(stream))
    if check:
        _check(st, "kdkl_backward_ex")
    return st


def kdkl_forward_backward_workspace_bytes(N: int, d: int, V: int, K: int, chunk_tokens: int = 0) -> int:
    return int(lib().kdkl_forward_backward_workspace_bytes(N, d, V, K, chunk_tokens))


def kdkl_forward_backward(hidden, W, topk_idx, topk_logit, mask, tau, loss, lse, dHidden, dW, workspace,
                          options=None, *, grad_loss=None, chunk_tokens=0, N=None, d=None, V=None, K=None,
                          workspace_bytes=None, stream=None, check=True) -> int:
    """Calls kdkl_forward_backward: loss, lse, dHidden and dW in one call, each logit chunk computed once."""
    N = hidden.shape[0] if N is None else N
    d = hidden.shape[1] if d is None else d
    V = W.shape[0] if V is None else V
    K = topk_idx.shape[1] if K is None else K
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    opt = ctypes.byref(options) if options is not None else None
    st = lib().kdkl_forward_backward(_ptr(hidden), _ptr(W), _ptr(topk_idx), _ptr(topk_logit), _ptr(mask), int(N),
                                     int(d), int(V), int(K), float(tau), opt, _ptr(grad_loss), _ptr(loss), _ptr(lse),
                                     _ptr(dHidden), _ptr(dW), int(chunk_tokens), _ptr(workspace), int(wsb),
                                     _stream(stream))
    if check:
        _check(st, "kdkl_forward_backward")
    return st


def kdkl_teacher_topk_workspace_bytes(N: int, d: int, V: int, K: int) -> int:
    return int(lib().kdkl_teacher_topk_workspace_bytes(N, d, V, K))


def kdkl_teacher_topk(hidden, W, K, topk_idx, topk_logit, workspace, *, N=None, d=None, V=None,
                      workspace_bytes=None, stream=None, check=True) -> int:
    """Calls kdkl_teacher_topk: the K largest logits of hidden W^T per row, with indices."""
    N = hidden.shape[0] if N is None else N
    d = hidden.shape[1] if d is None else d
    V = W.shape[0] if V is None else V
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    st = lib().kdkl_teacher_topk(_ptr(hidden), _ptr(W), int(N), int(d), int(V), int(K), _ptr(topk_idx),
                                 _ptr(topk_logit), _ptr(workspace), int(wsb), _stream(stream))
    if check:
        _check(st, "kdkl_teacher_topk")
    return st


def kdkl_forward_noalloc(hidden, W, topk_idx, topk_logit, mask, tau, loss, lse, *, N=None, d=None, V=None,
                         K=None, stream=None, check=True) -> int:
    """Calls kdkl_forward_noalloc: the forward without a caller workspace (built-in 32 MiB scratch)."""
    L = lib()
    fn = L.kdkl_forward_noalloc
    vp = ctypes.c_void_p
    fn.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                   ctypes.c_float, vp, vp, vp]
    fn.restype = ctypes.c_int
    N = hidden.shape[0] if N is None else N
    d = hidden.shape[1] if d is None else d
    V = W.shape[0] if V is None else V
    K = topk_idx.shape[1] if K is None else K
    st = fn(_ptr(hidden), _ptr(W), _ptr(topk_idx), _ptr(topk_logit), _ptr(mask), int(N), int(d), int(V), int(K),
            float(tau), _ptr(loss), _ptr(lse), _stream(stream))
    if check:
        _check(st, "kdkl_forward_noalloc")
    return st


def kdkl_n_valid_device(workspace) -> int:
    """Device address of the workspace's N_valid count (uint32)."""
    return int(lib().kdkl_n_valid_device(_ptr(workspace)))


def n_valid_view(workspace):
    """A one-element int32 view of the workspace tensor (uint8) at the address
    kdkl_n_valid_device returns (the count fits 31 bits: N is at most 2^31 - 256)."""
    import torch
    off = kdkl_n_valid_device(workspace) - workspace.data_ptr()
    if not 0 <= off <= workspace.numel() * workspace.element_size() - 4 or off % 4:
        raise RuntimeError(f"kdkl_n_valid_device gave an offset {off} outside the workspace")
    return workspace.view(torch.uint8)[off:off + 4].view(torch.int32)


def kdkl_count_valid(topk_idx, topk_logit, mask, tau, V, workspace, options=None, *, N=None, K=None,
                     workspace_bytes=None, stream=None, check=True) -> int:
    """Calls kdkl_count_valid: this shard's valid-token count, left at kdkl_n_valid_device(workspace)."""
    N = topk_idx.shape[0] if N is None else N
    K = topk_idx.shape[1] if K is None else K
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    opt = ctypes.byref(options) if options is not None else None
    st = lib().kdkl_count_valid(_ptr(topk_idx), _ptr(topk_logit), _ptr(mask), int(N), int(V), int(K), float(tau),
                                opt, _ptr(workspace), int(wsb), _stream(stream))
    if check:
        _check(st, "kdkl_count_valid")
    return st


def kdkl_read_device_flags(workspace, stream=None) -> int:
    out = ctypes.c_uint32(0)
    _check(lib().kdkl_read_device_flags(_ptr(workspace), _stream(stream), ctypes.byref(out)),
           "kdkl_read_device_flags")
    return int(out.value)


def kdkl_selftest_wait_timeout(workspace, limit_ns: int, stream=None) -> None:
    """Runs the bounded-wait self-test (see include/kdkl.h); read the flags afterwards."""
    _check(lib().kdkl_selftest_wait_timeout(_ptr(workspace), int(limit_ns), _stream(stream)),
           "kdkl_selftest_wait_timeout")


def kdkl_timing_enable(enable: bool = True) -> None:
    _check(lib().kdkl_timing_enable(1 if enable else 0), "kdkl_timing_enable")


def kdkl_timing_read(reset: bool = False) -> dict:
    """{kernel name: (launches, total ms)} accumulated since the last reset."""
    arr = (KernelTime * 16)()
    n = lib().kdkl_timing_read(arr, 16, 1 if reset else 0)
    return {arr[i].name.decode(): (int(arr[i].launches), float(arr[i].total_ms)) for i in range(n)}


def fused_kl_forward_backward(hidden, W, topk_idx, topk_logit, mask, tau, *, grad_loss=None, chunk_tokens=0,
                              workspace=None, stream=None):
    """Forward + backward with torch-allocated outputs.

    Returns (loss[1] f32, lse[N] f32, dHidden[N, d] bf16, dW[V, d] f32, workspace).
    """
    import torch
    N, d = hidden.shape
    V = W.shape[0]
    K = topk_idx.shape[1]
    dev = hidden.device
    if workspace is None:
        workspace = torch.empty(kdkl_workspace_bytes(N, d, V, K, chunk_tokens), dtype=torch.uint8, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    lse = torch.empty(N, dtype=torch.float32, device=dev)
    dH = torch.empty(N, d, dtype=torch.bfloat16, device=dev)
    dW = torch.empty(V, d, dtype=torch.float32, device=dev)
    kdkl_forward(hidden, W, topk_idx, topk_logit, mask, tau, loss, lse, workspace, stream=stream)
    kdkl_backward(hidden, W, topk_idx, topk_logit, mask, tau, lse, grad_loss, dH, dW, workspace,
                  chunk_tokens=chunk_tokens, stream=stream)
    return loss, lse, dH, dW, workspace


def _profile_lib() -> ctypes.CDLL:
    L = lib()
    if not hasattr(L, "kdkl_profile_read_role_cycles"):
        raise RuntimeError("the loaded kdkl library is not the profiling build: set LIB_PATH = PROFILE_LIB_PATH "
                           "before the first call")
    return L


def kdkl_profile_role_cycles_read():
    """The profiling build's role cycle counters, a numpy uint64 array [kind, cta, slot]
    (see include/kdkl_profile.h); synchronises the device."""
    import numpy as np
    L = _profile_lib()
    k, c, s = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(L.kdkl_profile_role_cycles_shape(ctypes.byref(k), ctypes.byref(c), ctypes.byref(s)),
           "kdkl_profile_role_cycles_shape")
    out = np.zeros((k.value, c.value, s.value), dtype=np.uint64)
    _check(L.kdkl_profile_read_role_cycles(out.ctypes.data, out.nbytes), "kdkl_profile_read_role_cycles")
    return out


def kdkl_profile_role_cycles_clear(stream=None) -> None:
    """Zeroes the profiling build's role cycle counters on `stream`."""
    _check(_profile_lib().kdkl_profile_clear_role_cycles(_stream(stream)), "kdkl_profile_clear_role_cycles")
