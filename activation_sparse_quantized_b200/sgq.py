"""Thin ctypes binding to libsgq.so (include/sgq.h). Argument marshalling only.

Each ``sgq_*`` function here has the name and argument order of the C entry
point; torch tensors are passed as device pointers (``data_ptr()``), the
stream defaults to torch's current stream, and a nonzero return code raises
``SgqError``. Every step of the computation runs in the CUDA library; there
is no fallback. If ``libsgq.so`` is missing the first call raises.

``alloc_*`` helpers only allocate correctly sized torch tensors (device
memory is plumbing, not part of the path).
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsgq.so")

SGQ_ACT_SILU = 0
SGQ_ACT_RELU = 1
SGQ_STATUS_NONFINITE_W = 1
SGQ_STATUS_BAD_INDEX = 2
SGQ_STATUS_BAD_COUNT = 4
SGQ_STATUS_TIMEOUT = 8
SGQ_MAX_BATCH = 16
SGQ_NOALLOC_MAX_N = 65536

EXPORTS = (
    "sgq_packed_sizes", "sgq_pack", "sgq_select", "sgq_gemv_workspace_bytes", "sgq_gemv",
    "sgq_gemv_thresh", "sgq_gemv_dense", "sgq_glu", "sgq_status_string", "sgq_last_cuda_error",
    "sgq_layout_version", "sgq_gemv_thresh_noalloc", "sgq_gemv_glu", "sgq_gemv_glu_thresh",
    "sgq_gemv_glu_dense", "sgq_select_mask", "sgq_gemv_mask", "sgq_packed_sizes_nm",
    "sgq_pack_nm", "sgq_gemv_nm", "sgq_gemv_nm_thresh", "sgq_gemv_acc", "sgq_gemv_thresh_acc",
    "sgq_ffn_workspace_bytes", "sgq_ffn", "sgq_read_status", "sgq_debug_gemv_withhold",
    "sgq_gemv_thresh_batch", "sgq_gemv_glu_thresh_batch",
)


class SgqError(RuntimeError):
    def __init__(self, fn, code, lib):
        msg = lib.sgq_status_string(code).decode()
        if code == -8:
            msg += f" (cudaError {lib.sgq_last_cuda_error()})"
        super().__init__(f"{fn}: {msg} [{code}]")
        self.code = code


_lib = None
_lock = threading.Lock()


def _open(path):
    if not os.path.exists(path):
        raise RuntimeError(
            f"libsgq.so not found at {path}: build it with "
            "`python -m activation_sparse_quantized_b200.build` (there is no CPU fallback)")
    return _declare(ctypes.CDLL(path))


def load(path: str = LIB_PATH):
    """Load libsgq.so (raises if it has not been built)."""
    global _lib
    if path != LIB_PATH:
        return _open(path)
    with _lock:
        if _lib is None:
            _lib = _open(path)
    return _lib


def _declare(lib):
    P, I, Z, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    sig = {
        "sgq_packed_sizes": ([I, I, I, ctypes.POINTER(Z), ctypes.POINTER(Z)], I),
        "sgq_pack": ([P, I, I, I, P, P, P, P], I),
        "sgq_select": ([P, I, I, P, P, P, P], I),
        "sgq_gemv_workspace_bytes": ([I, I, I], Z),
        "sgq_gemv": ([P, P, I, I, I, P, I, P, P, P, P, P, Z, P, P], I),
        "sgq_debug_gemv_withhold": ([P, P, I, I, I, P, I, P, P, P, P, P, Z, P, P], I),
        "sgq_gemv_thresh": ([P, P, I, I, I, P, F, P, P, P, Z, P, P], I),
        "sgq_gemv_thresh_batch": ([P, P, I, I, I, P, I, P, P, P, P, Z, P, P], I),
        "sgq_gemv_glu_thresh_batch": ([P, P, I, I, I, P, I, P, I, P, P, P, Z, P, P], I),
        "sgq_gemv_dense": ([P, P, I, I, I, P, I, P, P, P, Z, P, P], I),
        "sgq_gemv_thresh_noalloc": ([P, P, I, I, I, P, F, P, P, P, P], I),
        "sgq_glu": ([P, P, P, I, I, I, P], I),
        "sgq_gemv_glu": ([P, P, I, I, I, P, I, P, P, I, P, P, P, Z, P, P], I),
        "sgq_gemv_glu_thresh": ([P, P, I, I, I, P, F, I, P, P, P, Z, P, P], I),
        "sgq_gemv_glu_dense": ([P, P, I, I, I, P, I, I, P, P, P, Z, P, P], I),
        "sgq_select_mask": ([P, I, I, P, P, P, P], I),
        "sgq_gemv_mask": ([P, P, I, I, I, P, I, P, P, P, P, Z, P, P], I),
        "sgq_packed_sizes_nm": ([I, I, I, ctypes.POINTER(Z), ctypes.POINTER(Z),
                                 ctypes.POINTER(Z)], I),
        "sgq_pack_nm": ([P, I, I, I, P, P, P, P, P], I),
        "sgq_gemv_nm": ([P, P, P, I, I, I, P, P, P, P, P, P, Z, P, P], I),
        "sgq_gemv_nm_thresh": ([P, P, P, I, I, I, P, F, P, P, P, Z, P, P], I),
        "sgq_gemv_acc": ([P, P, I, I, I, P, I, P, P, P, P, P], I),
        "sgq_gemv_thresh_acc": ([P, P, I, I, I, P, F, P, P, P], I),
        "sgq_ffn_workspace_bytes": ([I, I], Z),
        "sgq_read_status": ([P, P, I, P], I),
        "sgq_ffn": ([P, P, P, P, I, I, I, P, F, I, F, P, P, P, P, Z, P, P], I),
        "sgq_status_string": ([I], ctypes.c_char_p),
        "sgq_last_cuda_error": ([], I),
        "sgq_layout_version": ([], I),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn, rc):
    if rc != 0:
        raise SgqError(fn, rc, load())


# --------------------------------------------------------------------------
# The C entry points, one to one.
# --------------------------------------------------------------------------

def sgq_read_status(status, clear=True, stream=None) -> int:
    """The SGQ_STATUS_* bits of a device status word (synchronises the stream
    to return the value; the C call itself only enqueues the copy)."""
    out = ctypes.c_int32(0)
    _check("sgq_read_status", load().sgq_read_status(_ptr(status), ctypes.byref(out),
                                                     1 if clear else 0, _stream(stream)))
    (stream or torch.cuda.current_stream()).synchronize()
    return out.value


def sgq_layout_version() -> int:
    return load().sgq_layout_version()


def sgq_packed_sizes(N: int, K: int, group: int):
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check("sgq_packed_sizes", load().sgq_packed_sizes(N, K, group, ctypes.byref(a), ctypes.byref(b)))
    return a.value, b.value


def sgq_pack(W, N, K, group, qweight, sz, status=None, stream=None):
    _check("sgq_pack", load().sgq_pack(_ptr(W), N, K, group, _ptr(qweight), _ptr(sz),
                                       _ptr(status), _stream(stream)))


def sgq_select(x, B, K, t_host, idx, count, stream=None):
    t = (ctypes.c_float * B)(*[float(v) for v in t_host])
    _check("sgq_select", load().sgq_select(_ptr(x), B, K, t, _ptr(idx), _ptr(count),
                                           _stream(stream)))


def sgq_select_mask(x, B, K, t_host, mask, count=None, stream=None):
    t = (ctypes.c_float * B)(*[float(v) for v in t_host])
    _check("sgq_select_mask", load().sgq_select_mask(_ptr(x), B, K, t, _ptr(mask), _ptr(count),
                                                     _stream(stream)))


def sgq_gemv_mask(qweight, sz, N, K, group, x, B, mask, y, y_f32, workspace, status=None,
                  stream=None):
    _check("sgq_gemv_mask", load().sgq_gemv_mask(
        _ptr(qweight), _ptr(sz), N, K, group, _ptr(x), B, _ptr(mask), _ptr(y), _ptr(y_f32),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
        _stream(stream)))


def sgq_packed_sizes_nm(N: int, K: int, group: int):
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check("sgq_packed_sizes_nm", load().sgq_packed_sizes_nm(
        N, K, group, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)))
    return a.value, b.value, c.value


def sgq_pack_nm(W, N, K, group, qweight, keep, sz, status=None, stream=None):
    _check("sgq_pack_nm", load().sgq_pack_nm(_ptr(W), N, K, group, _ptr(qweight), _ptr(keep),
                                             _ptr(sz), _ptr(status), _stream(stream)))


def sgq_gemv_nm(qweight, keep, sz, N, K, group, x, idx, count, y, y_f32, workspace, status=None,
                stream=None):
    _check("sgq_gemv_nm", load().sgq_gemv_nm(
        _ptr(qweight), _ptr(keep), _ptr(sz), N, K, group, _ptr(x), _ptr(idx), _ptr(count),
        _ptr(y), _ptr(y_f32), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(status), _stream(stream)))


def sgq_gemv_nm_thresh(qweight, keep, sz, N, K, group, x, t, y, y_f32, workspace, status=None,
                       stream=None):
    _check("sgq_gemv_nm_thresh", load().sgq_gemv_nm_thresh(
        _ptr(qweight), _ptr(keep), _ptr(sz), N, K, group, _ptr(x), float(t), _ptr(y),
        _ptr(y_f32), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(status), _stream(stream)))


def sgq_gemv_acc(qweight, sz, N, K, group, x, B, idx, count, y_acc, status=None, stream=None):
    """y_acc (fp32 [B][N]) += the sparse GEMV; one kernel, no workspace."""
    _check("sgq_gemv_acc", load().sgq_gemv_acc(
        _ptr(qweight), _ptr(sz), N, K, group, _ptr(x), B, _ptr(idx), _ptr(count), _ptr(y_acc),
        _ptr(status), _stream(stream)))


def sgq_gemv_thresh_acc(qweight, sz, N, K, group, x, t, y_acc, status=None, stream=None):
    _check("sgq_gemv_thresh_acc", load().sgq_gemv_thresh_acc(
        _ptr(qweight), _ptr(sz), N, K, group, _ptr(x), float(t), _ptr(y_acc), _ptr(status),
        _stream(stream)))


def sgq_gemv_workspace_bytes(N: int, K: int, B: int) -> int:
    return load().sgq_gemv_workspace_bytes(N, K, B)


def sgq_gemv(qweight, sz, N, K, group, x, B, idx, count, y, y_f32, workspace, status=None,
             stream=None):
    _check("sgq_gemv", load().sgq_gemv(
        _ptr(qweight), _ptr(sz), N, K, group, _ptr(x), B, _ptr(idx), _ptr(count), _ptr(y),
        _ptr(y_f32), _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
        _stream(stream)))


def sgq_debug_gemv_withhold(qweight, sz, N, K, group, x, B, idx, count, y, y_f32, workspace,
                            status, stream=None):
    """Test hook: sgq_gemv (B = 9..16) whose last group run is never released,
    so the kernel's bounded waits run out and set SGQ_STATUS_TIMEOUT."""
    _check("sgq_debug_gemv_withhold", load().sgq_debug_gemv_withhold(
        _ptr(qweight), _ptr(sz), N, K, group, _ptr(x), B, _ptr(idx), _ptr(count), _ptr(y),
        _ptr(y_f32), _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
        _stream(stream)))


def sgq_gemv_thresh(qweight, sz, N, K, group, x, t, y, y_f32, workspace, status=None,
                    stream=None):
    _check("sgq_gemv_thresh", load().sgq_gemv_thresh(
        _ptr(qweight), _ptr(sz), N, K, group, _ptr(x), float(t), _ptr(y), _ptr(y_f32),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
        _stream(stream)))


def sgq_gemv_thresh_batch(qweight, sz, N, K, group, x, B, t_host, y, y_f32, workspace,
                          status=None, stream=None):
    t = (ctypes.c_float * B)(*[float(v) for v in t_host])
    _check("sgq_gemv_thresh_batch", load().sgq_gemv_thresh_batch(
        _ptr(qweight), _ptr(sz), N, K, group, _ptr(x), B, t, _ptr(y), _ptr(y_f32),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
        _stream(stream)))


def sgq_gemv_thresh_noalloc(qweight, sz, N, K, group, x, t, y, y_f32, status=None, stream=None):
    """sgq_gemv_thresh with the library's fixed scratch instead of a workspace
    (for callers that cannot allocate); N <= SGQ_NOALLOC_MAX_N."""
    _check("sgq_gemv_thresh_noalloc", load().sgq_gemv_thresh_noalloc(
        _ptr(qweight), _ptr(sz), N, K, group, _ptr(x), float(t), _ptr(y), _ptr(y_f32),
        _ptr(status), _stream(stream)))


def sgq_gemv_dense(qweight, sz, N, K, group, x, B, y, y_f32, workspace, status=None,
                   stream=None):
    _check("sgq_gemv_dense", load().sgq_gemv_dense(
        _ptr(qweight), _ptr(sz), N, K, group, _ptr(x), B, _ptr(y), _ptr(y_f32), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream)))


def sgq_gemv_glu(qweight, sz, I, K, group, x, B, idx, count, act, h, h_f32, workspace,
                 status=None, stream=None):
    """Fused gate + up + act over the stacked [W_g; W_u] weights (packed with N = 2I)."""
    _check("sgq_gemv_glu", load().sgq_gemv_glu(
        _ptr(qweight), _ptr(sz), I, K, group, _ptr(x), B, _ptr(idx), _ptr(count), act, _ptr(h),
        _ptr(h_f32), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(status), _stream(stream)))


def sgq_gemv_glu_thresh(qweight, sz, I, K, group, x, t, act, h, h_f32, workspace, status=None,
                        stream=None):
    _check("sgq_gemv_glu_thresh", load().sgq_gemv_glu_thresh(
        _ptr(qweight), _ptr(sz), I, K, group, _ptr(x), float(t), act, _ptr(h), _ptr(h_f32),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
        _stream(stream)))


def sgq_gemv_glu_thresh_batch(qweight, sz, I, K, group, x, B, t_host, act, h, h_f32, workspace,
                              status=None, stream=None):
    t = (ctypes.c_float * B)(*[float(v) for v in t_host])
    _check("sgq_gemv_glu_thresh_batch", load().sgq_gemv_glu_thresh_batch(
        _ptr(qweight), _ptr(sz), I, K, group, _ptr(x), B, t, act, _ptr(h), _ptr(h_f32),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
        _stream(stream)))


def sgq_gemv_glu_dense(qweight, sz, I, K, group, x, B, act, h, h_f32, workspace, status=None,
                       stream=None):
    _check("sgq_gemv_glu_dense", load().sgq_gemv_glu_dense(
        _ptr(qweight), _ptr(sz), I, K, group, _ptr(x), B, act, _ptr(h), _ptr(h_f32),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
        _stream(stream)))


def sgq_ffn_workspace_bytes(H: int, I: int) -> int:
    return load().sgq_ffn_workspace_bytes(H, I)


def sgq_ffn(qweight_gu, sz_gu, qweight_d, sz_d, H, I, group, x, t_in, act, t_h, y, y_f32,
            h_out, workspace, status=None, stream=None):
    """The batch-1 decode FFN in three kernels (gate/up GEMV, down GEMV with the
    GLU and the selection of h in its prologue, epilogue)."""
    _check("sgq_ffn", load().sgq_ffn(
        _ptr(qweight_gu), _ptr(sz_gu), _ptr(qweight_d), _ptr(sz_d), H, I, group, _ptr(x),
        float(t_in), act, float(t_h), _ptr(y), _ptr(y_f32), _ptr(h_out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream)))


def alloc_ffn_workspace(H, I, device="cuda"):
    return torch.zeros(sgq_ffn_workspace_bytes(H, I) // 4, dtype=torch.int32, device=device)


def sgq_glu(gate, up, h, B, I, act, stream=None):
    _check("sgq_glu", load().sgq_glu(_ptr(gate), _ptr(up), _ptr(h), B, I, act, _stream(stream)))


# --------------------------------------------------------------------------
# Allocation helpers (torch device memory; plumbing only).
# --------------------------------------------------------------------------

def alloc_packed(N, K, group, device="cuda"):
    qb, sb = sgq_packed_sizes(N, K, group)
    return (torch.empty(qb, dtype=torch.uint8, device=device),
            torch.empty(sb // 4, dtype=torch.int32, device=device))


def alloc_workspace(N, K, B, device="cuda"):
    nbytes = sgq_gemv_workspace_bytes(N, K, B)
    return torch.zeros(nbytes // 4, dtype=torch.int32, device=device)


def alloc_packed_nm(N, K, group, device="cuda"):
    """(qweight u8, keep u8, sz int32) buffers of the 2:4 layout."""
    qb, kb, sb = sgq_packed_sizes_nm(N, K, group)
    return (torch.empty(qb, dtype=torch.uint8, device=device),
            torch.empty(kb, dtype=torch.uint8, device=device),
            torch.empty(sb // 4, dtype=torch.int32, device=device))


def alloc_mask(K, device="cuda"):
    """uint32 words for a K-channel bitmask (int32 tensor; bits are what matter)."""
    return torch.zeros((K + 31) // 32, dtype=torch.int32, device=device)


def alloc_select(K, device="cuda"):
    return (torch.empty(K, dtype=torch.int32, device=device),
            torch.zeros(1, dtype=torch.int32, device=device))
