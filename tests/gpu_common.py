"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compute the oracle's expectation on the same seeded inputs.

Tolerance (floating point). The bound on an output is
    |y_gpu - y_ref| <= 1e-3 * sum_k |W_deq[n,k] x[k]|          (sum over the active k)
checked on the fp32 result before rounding (``y_f32``). The bf16 output adds
its own round-to-nearest step, at most 2^-8 of the fp32 value, so bf16 y is
checked against
    1e-3 * sumabs * (1 + 2^-8) + 2^-8 * |y_ref|.
Integer / byte / index outputs (packing, selection) are compared bit for bit.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from activation_sparse_quantized_b200 import sgq
from activation_sparse_quantized_b200 import workloads as wl

DEV = "cuda"
REL_TOL = 1e-3
BF16_HALF_ULP = 2.0 ** -8


def bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of an fp16/bf16 tensor (any device)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_values(b: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16)
    return t.double().numpy()


def gpu_pack(W: torch.Tensor, group: int):
    N, K = W.shape
    qw, sz = sgq.alloc_packed(N, K, group)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    sgq.sgq_pack(W.to(DEV).contiguous(), N, K, group, qw, sz, status)
    return qw, sz, status


def packed_codes_rows(qw: torch.Tensor, N: int, K: int, rows) -> np.ndarray:
    """Codes q[rows][K] read back from the packed layout (for sampled checks)."""
    qb = qw.cpu().numpy().reshape(K, N // 2)
    rows = np.asarray(rows)
    byte = qb[:, rows // 2]
    code = np.where((rows % 2) == 1, byte >> 4, byte & 0x0F)
    return code.T.astype(np.uint8)


def sz_rows(sz: torch.Tensor, N: int, K: int, group: int, rows):
    a = sz.cpu().numpy().view(np.uint16).reshape(K // group, N, 2)
    rows = np.asarray(rows)
    return a[:, rows, 0].T.copy(), a[:, rows, 1].T.copy()


def check_y(y_bf16: torch.Tensor, y_f32: torch.Tensor, y64: np.ndarray, sumabs: np.ndarray,
            what=""):
    yb = bf16_values(bits(y_bf16))
    yf = y_f32.detach().cpu().double().numpy()
    err32 = np.abs(yf - y64)
    tol32 = REL_TOL * sumabs
    bad = err32 > tol32
    assert not bad.any(), (
        f"{what}: {int(bad.sum())} outputs beyond 1e-3*sum|wx|; worst ratio "
        f"{np.max(err32 / np.maximum(tol32, 1e-300)):.3g}")
    tolb = REL_TOL * sumabs * (1 + BF16_HALF_ULP) + BF16_HALF_ULP * np.abs(y64)
    badb = np.abs(yb - y64) > tolb
    assert not badb.any(), f"{what}: {int(badb.sum())} bf16 outputs beyond tolerance"
    return float(np.max(err32 / np.maximum(sumabs, 1e-300)))


def sample_rows(N: int, n: int, seed: int = 0) -> np.ndarray:
    """Outputs to check one by one at full size: both ends, tile edges and a
    random sample."""
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 31, 32, 255, 256, 1023, 1024, N // 2, N - 33, N - 32, N - 1]
    r = set(v for v in fixed if 0 <= v < N)
    r.update(rng.choice(N, size=min(n, N), replace=False).tolist())
    return np.array(sorted(r))


class GpuGemv:
    """A packed weight on the device plus the buffers one GEMV call needs."""

    def __init__(self, W: torch.Tensor, group: int, B: int = 1):
        self.W = W
        self.N, self.K = W.shape
        self.group = group
        self.B = B
        self.qw, self.sz, self.pack_status = gpu_pack(W, group)
        self.ws = sgq.alloc_workspace(self.N, self.K, B)
        self.idx, self.count = sgq.alloc_select(self.K)
        self.status = torch.zeros(1, dtype=torch.int32, device=DEV)

    def outputs(self, B=None):
        B = B or self.B
        y = torch.full((B, self.N), float("nan"), dtype=torch.bfloat16, device=DEV)
        y32 = torch.full((B, self.N), float("nan"), dtype=torch.float32, device=DEV)
        return y, y32

    def select(self, x_d, t):
        B = x_d.shape[0]
        sgq.sgq_select(x_d, B, self.K, t, self.idx, self.count)

    def gemv(self, x_d, idx=None, count=None):
        B = x_d.shape[0]
        y, y32 = self.outputs(B)
        sgq.sgq_gemv(self.qw, self.sz, self.N, self.K, self.group, x_d, B,
                     self.idx if idx is None else idx, self.count if count is None else count,
                     y, y32, self.ws, self.status)
        return y, y32

    def dense(self, x_d):
        B = x_d.shape[0]
        y, y32 = self.outputs(B)
        sgq.sgq_gemv_dense(self.qw, self.sz, self.N, self.K, self.group, x_d, B, y, y32,
                           self.ws, self.status)
        return y, y32

    def thresh(self, x_d, t):
        y, y32 = self.outputs(1)
        sgq.sgq_gemv_thresh(self.qw, self.sz, self.N, self.K, self.group, x_d, t, y, y32,
                            self.ws, self.status)
        return y, y32

    def active(self):
        return self.idx[: int(self.count.item())].cpu().numpy()

    def workspace_is_zero(self):
        return bool((self.ws == 0).all().item())


def oracle_codes(W: torch.Tensor, group: int, rows=None):
    Wb = bits(W)
    if rows is not None:
        Wb = Wb[np.asarray(rows)]
    return oracle.quantize(Wb, group)


def oracle_expect(W, group, x, t, rows=None):
    """(idx, y64, sumabs, y_bf16) of the oracle for the given rows of W."""
    xb = bits(x)
    idx = oracle.select(xb, t)
    q, s, z = oracle_codes(W, group, rows)
    y64, sa, yb = oracle.gemv(q, s, z, group, xb, idx)
    return idx, y64, sa, yb


__all__ = ["wl", "sgq", "oracle"]
