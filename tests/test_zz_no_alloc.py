"""The no-allocation GEMV entry point against the workspace entry point.

Some callers cannot allocate device memory: they run inside a host framework
that owns all GPU memory, or on a path where an allocation may not happen (or
fail) in the middle of a decode step. sgq_gemv_thresh_noalloc serves them: its
split-K scratch is a fixed array inside the library rather than a workspace
the caller allocates. These tests call it through the C ABI twice in a row
(the second call must start from the zeros the first call left behind) and
compare each result with sgq_gemv_thresh on the same inputs, within the
tolerance the other GEMV tests use (1e-3 * sum |w x| on the fp32 result, plus
the bf16 rounding step on y). This file is collected last; it passes on its
own in a fresh process and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from activation_sparse_quantized_b200 import build, sgq
from activation_sparse_quantized_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    torch.cuda.set_device(0)
    return sgq.load()


def test_noalloc_matches_workspace_entry_point_twice(lib):
    shp = wl.LLAMA8B_DOWN
    N, K, g = shp["N"], shp["K"], shp["group"]
    case = wl.gemv_case(**shp, sparsity=0.5, seed=5, act="silu")
    qw, sz = sgq.alloc_packed(N, K, g)
    sgq.sgq_pack(case.W.cuda(), N, K, g, qw, sz)
    x = case.x.cuda()
    t = case.t[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    ws = sgq.alloc_workspace(N, K, 1)
    y_ref = torch.empty(1, N, dtype=torch.bfloat16, device="cuda")
    y32_ref = torch.empty(1, N, dtype=torch.float32, device="cuda")
    rc = lib.sgq_gemv_thresh(_ptr(qw), _ptr(sz), N, K, g, _ptr(x), ctypes.c_float(t),
                             _ptr(y_ref), _ptr(y32_ref), _ptr(ws),
                             ws.numel() * ws.element_size(), None, stream)
    assert rc == 0

    xb = _bits(case.x)
    idx = oracle.select(xb, [t])
    q, s, z = oracle.quantize(_bits(case.W), g)
    _, sumabs, _ = oracle.gemv(q, s, z, g, xb, idx)
    tol32 = 1e-3 * sumabs[0]

    for _ in range(2):
        y = torch.full((1, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        y32 = torch.full((1, N), float("nan"), dtype=torch.float32, device="cuda")
        rc = lib.sgq_gemv_thresh_noalloc(_ptr(qw), _ptr(sz), N, K, g, _ptr(x),
                                         ctypes.c_float(t), _ptr(y), _ptr(y32), None, stream)
        assert rc == 0
        torch.cuda.synchronize()
        a = y32.cpu().double().numpy()[0]
        b = y32_ref.cpu().double().numpy()[0]
        assert np.all(np.abs(a - b) <= tol32)
        ab = y.float().cpu().double().numpy()[0]
        bb = y_ref.float().cpu().double().numpy()[0]
        assert np.all(np.abs(ab - bb) <= tol32 * (1 + 2.0 ** -8) + 2.0 ** -7 * np.abs(bb))


def test_noalloc_rejects_n_above_its_scratch(lib):
    fake = ctypes.c_void_p(1 << 20)
    rc = lib.sgq_gemv_thresh_noalloc(fake, fake, sgq.SGQ_NOALLOC_MAX_N + 32, 4096, 128, fake,
                                     ctypes.c_float(0.5), fake, None, None, None)
    assert rc == -10
    assert b"SGQ_NOALLOC_MAX_N" in lib.sgq_status_string(rc)
