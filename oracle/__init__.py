"""The CPU oracle: a plain fp64 C restatement of the activation-sparse int4 GEMV.

TEST INFRASTRUCTURE ONLY. Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference legs of ``bench.py`` may import this package. The
CUDA library never calls it and shares no code with it.

The C source (``sgq_oracle.c``) cites, for each function, the page section it
follows:

* "Enabling Dynamic Sparsity in Quantized LLM Inference", Abstract
  (group-wise low-bit quantization, dynamic activation sparsity, a GEMV on the
  quantized layout, runtime gathering of the sparse indices);
* "SVD Contextual Sparsity Predictors for Fast LLM Inference", Abstract
  (ReGLU FFNs whose zero neurons are skipped).

This module only marshals numpy arrays to the C functions.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sgq_oracle.c")
_HDR = os.path.join(_HERE, "sgq_oracle.h")
LIB_PATH = os.path.join(_HERE, "libsgq_oracle.so")

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-fopenmp"]

_lib = None
_lock = threading.Lock()


def build(force: bool = False, src: str = _SRC, out: str = LIB_PATH) -> str:
    """Compile the oracle with gcc (no GPU needed). Returns the library path."""
    stale = (not os.path.exists(out)) or any(
        os.path.getmtime(p) > os.path.getmtime(out) for p in (src, _HDR))
    if force or stale:
        cmd = ["gcc", *CFLAGS, "-I", _HERE, src, "-o", out + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(out + ".tmp", out)
    return out


def _u16p(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16))


def _u8p(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))


def _i32p(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _f64p(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f32p(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def load(path: str | None = None):
    """Load (building first if needed) and return the ctypes library."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _declare(ctypes.CDLL(build()))
    return _lib


def _declare(lib):
    P = ctypes.c_void_p
    i = ctypes.c_int
    lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_half_to_double.restype = ctypes.c_double
    lib.oracle_double_to_half.argtypes = [ctypes.c_double]
    lib.oracle_double_to_half.restype = ctypes.c_uint16
    lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_double.restype = ctypes.c_double
    lib.oracle_double_to_bf16.argtypes = [ctypes.c_double]
    lib.oracle_double_to_bf16.restype = ctypes.c_uint16
    lib.oracle_quantize.argtypes = [P, i, i, i, P, P, P]
    lib.oracle_pack_layout.argtypes = [P, P, P, i, i, i, P, P]
    lib.oracle_select.argtypes = [P, i, i, P, P, P]
    lib.oracle_gemv.argtypes = [P, P, P, i, i, i, P, i, P, i, P, P, P]
    lib.oracle_gemv_dense.argtypes = [P, P, P, i, i, i, P, i, P, P, P]
    lib.oracle_gemv_threads.argtypes = [P, P, P, i, i, i, P, i, P, i, P, P, P, i]
    lib.oracle_glu.argtypes = [P, P, ctypes.c_int64, i, P, P]
    lib.oracle_act_mul.argtypes = [P, P, ctypes.c_int64, i, P, P]
    lib.oracle_select_mask.argtypes = [P, i, i, P, P, P]
    lib.oracle_nm_keep.argtypes = [P, i, i, i, P, P]
    lib.oracle_pack_layout_nm.argtypes = [P, P, P, P, P, i, i, i, P, P, P]
    for f in ("oracle_quantize", "oracle_pack_layout", "oracle_select",
              "oracle_gemv", "oracle_gemv_threads", "oracle_gemv_dense", "oracle_glu", "oracle_act_mul", "oracle_select_mask", "oracle_nm_keep",
              "oracle_pack_layout_nm"):
        getattr(lib, f).restype = ctypes.c_int
    return lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


class OracleError(RuntimeError):
    pass


def _check(rc, what):
    if rc != 0:
        raise OracleError(f"{what} returned {rc}")


# --- number formats -------------------------------------------------------

def half_to_double(bits, lib=None):
    lib = lib or load()
    return np.array([lib.oracle_half_to_double(int(b)) for b in np.ravel(bits)])


def double_to_half(vals, lib=None):
    lib = lib or load()
    return np.array([lib.oracle_double_to_half(float(v)) for v in np.ravel(vals)], dtype=np.uint16)


def bf16_to_double(bits, lib=None):
    lib = lib or load()
    return np.array([lib.oracle_bf16_to_double(int(b)) for b in np.ravel(bits)])


def double_to_bf16(vals, lib=None):
    lib = lib or load()
    return np.array([lib.oracle_double_to_bf16(float(v)) for v in np.ravel(vals)], dtype=np.uint16)


# --- the path ---------------------------------------------------------------

def quantize(W_bits, g, lib=None):
    """W_bits: uint16 fp16 bit patterns [N, K]. Returns (q [N,K] u8, s, z [N,K/g] u16)."""
    lib = lib or load()
    W = _c(W_bits, np.uint16)
    N, K = W.shape
    q = np.empty((N, K), np.uint8)
    s = np.empty((N, K // g), np.uint16)
    z = np.empty((N, K // g), np.uint16)
    _check(lib.oracle_quantize(W.ctypes.data, N, K, g, q.ctypes.data, s.ctypes.data,
                               z.ctypes.data), "oracle_quantize")
    return q, s, z


def quantize_rc(W_bits, g, lib=None):
    """Return code of oracle_quantize (for the error-path tests)."""
    lib = lib or load()
    W = _c(W_bits, np.uint16)
    N, K = W.shape
    q = np.empty((N, K), np.uint8)
    s = np.empty((N, max(K // g, 1)), np.uint16)
    z = np.empty((N, max(K // g, 1)), np.uint16)
    return lib.oracle_quantize(W.ctypes.data, N, K, g, q.ctypes.data, s.ctypes.data, z.ctypes.data)


def pack_layout(q, s, z, g, lib=None):
    """Returns (qweight [K, N/2] u8, sz [K/g, N, 2] u16) in layout version 1."""
    lib = lib or load()
    q = _c(q, np.uint8)
    s = _c(s, np.uint16)
    z = _c(z, np.uint16)
    N, K = q.shape
    qw = np.empty((K, N // 2), np.uint8)
    sz = np.empty((K // g, N, 2), np.uint16)
    _check(lib.oracle_pack_layout(q.ctypes.data, s.ctypes.data, z.ctypes.data, N, K, g,
                                  qw.ctypes.data, sz.ctypes.data), "oracle_pack_layout")
    return qw, sz


def select(x_bits, t, lib=None):
    """x_bits: uint16 bf16 [B, K]; t: B floats. Returns the int32 active list."""
    lib = lib or load()
    x = _c(np.atleast_2d(x_bits), np.uint16)
    B, K = x.shape
    tt = _c(np.broadcast_to(np.asarray(t, np.float32), (B,)), np.float32)
    idx = np.empty(K, np.int32)
    cnt = np.zeros(1, np.int32)
    _check(lib.oracle_select(x.ctypes.data, B, K, tt.ctypes.data, idx.ctypes.data,
                             cnt.ctypes.data), "oracle_select")
    return idx[: int(cnt[0])].copy()


def gemv(q, s, z, g, x_bits, idx, lib=None, threads=None):
    """Returns (y f64 [B,N], sumabs f64 [B,N], y_bf16 u16 [B,N]). With
    ``threads`` the outputs are shared over that many OpenMP threads (same
    results bit for bit)."""
    lib = lib or load()
    q = _c(q, np.uint8)
    s = _c(s, np.uint16)
    z = _c(z, np.uint16)
    x = _c(np.atleast_2d(x_bits), np.uint16)
    idx = _c(idx, np.int32)
    N, K = q.shape
    B = x.shape[0]
    y = np.empty((B, N), np.float64)
    sa = np.empty((B, N), np.float64)
    yb = np.empty((B, N), np.uint16)
    args = (q.ctypes.data, s.ctypes.data, z.ctypes.data, N, K, g, x.ctypes.data, B,
            idx.ctypes.data, int(idx.size), y.ctypes.data, sa.ctypes.data, yb.ctypes.data)
    if threads is None:
        _check(lib.oracle_gemv(*args), "oracle_gemv")
    else:
        _check(lib.oracle_gemv_threads(*args, int(threads)), "oracle_gemv_threads")
    return y, sa, yb


def gemv_dense(q, s, z, g, x_bits, lib=None):
    lib = lib or load()
    q = _c(q, np.uint8)
    s = _c(s, np.uint16)
    z = _c(z, np.uint16)
    x = _c(np.atleast_2d(x_bits), np.uint16)
    N, K = q.shape
    B = x.shape[0]
    y = np.empty((B, N), np.float64)
    sa = np.empty((B, N), np.float64)
    yb = np.empty((B, N), np.uint16)
    _check(lib.oracle_gemv_dense(q.ctypes.data, s.ctypes.data, z.ctypes.data, N, K, g,
                                 x.ctypes.data, B, y.ctypes.data, sa.ctypes.data,
                                 yb.ctypes.data), "oracle_gemv_dense")
    return y, sa, yb


def glu(gate_bits, up_bits, act, lib=None):
    """act: 0 = SiLU, 1 = ReLU. Returns (h f64, h_bf16 u16) shaped like gate."""
    lib = lib or load()
    gt = _c(gate_bits, np.uint16)
    up = _c(up_bits, np.uint16)
    assert gt.shape == up.shape
    h = np.empty(gt.shape, np.float64)
    hb = np.empty(gt.shape, np.uint16)
    _check(lib.oracle_glu(gt.ctypes.data, up.ctypes.data, gt.size, act, h.ctypes.data,
                          hb.ctypes.data), "oracle_glu")
    return h, hb


def act_mul(gate, up, act, lib=None):
    """h = act(gate) * up on fp64 inputs (act 0 = SiLU, 1 = ReLU).
    Returns (h f64, h_bf16 u16) shaped like gate."""
    lib = lib or load()
    g = _c(gate, np.float64)
    u = _c(up, np.float64)
    assert g.shape == u.shape
    h = np.empty(g.shape, np.float64)
    hb = np.empty(g.shape, np.uint16)
    _check(lib.oracle_act_mul(g.ctypes.data, u.ctypes.data, g.size, act, h.ctypes.data,
                              hb.ctypes.data), "oracle_act_mul")
    return h, hb


def select_mask(x_bits, t, lib=None):
    """Bitmask of the active set of x [B][K] (bf16 bits): uint32 [(K + 31) / 32]."""
    lib = lib or load()
    x = _c(np.atleast_2d(x_bits), np.uint16)
    B, K = x.shape
    tt = _c(np.broadcast_to(np.asarray(t, np.float32), (B,)), np.float32)
    mask = np.empty((K + 31) // 32, np.uint32)
    cnt = ctypes.c_int32()
    _check(lib.oracle_select_mask(x.ctypes.data, B, K, tt.ctypes.data, mask.ctypes.data,
                                  ctypes.byref(cnt)), "oracle_select_mask")
    return mask, cnt.value


def nm_keep(W_bits, g, lib=None):
    """2:4 choice of W [N, K] (fp16 bits): (keep [K/g, N/4] nibbles, bad [K/g, N/4])."""
    lib = lib or load()
    W = _c(W_bits, np.uint16)
    N, K = W.shape
    keep = np.empty((K // g, N // 4), np.uint8)
    bad = np.empty((K // g, N // 4), np.uint8)
    _check(lib.oracle_nm_keep(W.ctypes.data, N, K, g, keep.ctypes.data, bad.ctypes.data),
           "oracle_nm_keep")
    return keep, bad


def pack_layout_nm(q, s, z, keep, bad, g, lib=None):
    """The 2:4 packed layout: (qweight [K, N/4] u8, keep_packed [K/g, N/8] u8,
    sz [K/g, N/2, 2] u16)."""
    lib = lib or load()
    q = _c(q, np.uint8)
    N, K = q.shape
    s, z = _c(s, np.uint16), _c(z, np.uint16)
    keep, bad = _c(keep, np.uint8), _c(bad, np.uint8)
    qw = np.empty((K, N // 4), np.uint8)
    kp = np.empty((K // g, N // 8), np.uint8)
    sz = np.empty((K // g, N // 2, 2), np.uint16)
    _check(lib.oracle_pack_layout_nm(q.ctypes.data, s.ctypes.data, z.ctypes.data,
                                     keep.ctypes.data, bad.ctypes.data, N, K, g, qw.ctypes.data,
                                     kp.ctypes.data, sz.ctypes.data), "oracle_pack_layout_nm")
    return qw, kp, sz


def gemv_nm(q, s, z, keep, bad, g, x_bits, idx, lib=None):
    """The GEMV over the 2:4-pruned weights: the pruned outputs of each
    (group, block), and every output of a bad block, weigh zero (their scale
    and zero are set to 0 before the plain GEMV). Returns as gemv."""
    N = q.shape[0]
    G = s.shape[1]
    kept = np.zeros((N, G), bool)
    for i in range(4):
        kept[i::4, :] = (((keep >> i) & 1) == 1).T & (bad == 0).T
    s2 = np.where(kept, s, np.uint16(0)).astype(np.uint16)
    z2 = np.where(kept, z, np.uint16(0)).astype(np.uint16)
    return gemv(q, s2, z2, g, x_bits, idx, lib)
