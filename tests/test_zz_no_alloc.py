"""The no-allocation GEMV entry point against the oracle and the workspace
entry point.

Some callers cannot allocate device memory: they run inside a host framework
that owns all GPU memory, or on a path where an allocation may not happen (or
fail) in the middle of a decode step. sgq_gemv_thresh_noalloc serves them: its
split-K scratch is a fixed array inside the library rather than a workspace
the caller allocates. These tests call it through the C ABI on a non-blocking
stream (one that does not synchronise with the legacy default stream), twice in
a row (the second call must not depend on what the first left behind), and
check each result against the oracle within the tolerance the other GEMV
tests use (1e-3 * sum |w x| on the fp32 result, plus the bf16 rounding step on
y) and against sgq_gemv_thresh. One test makes the very first call of a fresh
process on such a stream. This file is collected last; it passes on its own in
a fresh process and after the rest of the suite.
"""
import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from activation_sparse_quantized_b200 import build, sgq
from activation_sparse_quantized_b200 import workloads as wl
from gpu_common import bits, check_y

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    torch.cuda.set_device(0)
    return sgq.load()


def _case():
    shp = wl.LLAMA8B_DOWN
    case = wl.gemv_case(**shp, sparsity=0.5, seed=5, act="silu")
    xb = bits(case.x)
    idx = oracle.select(xb, [case.t[0]])
    q, s, z = oracle.quantize(bits(case.W), shp["group"])
    y64, sumabs, _ = oracle.gemv(q, s, z, shp["group"], xb, idx)
    return shp, case, y64, sumabs


def test_noalloc_matches_oracle_and_workspace_entry_point_twice(lib):
    shp, case, y64, sumabs = _case()
    N, K, g = shp["N"], shp["K"], shp["group"]
    qw, sz = sgq.alloc_packed(N, K, g)
    sgq.sgq_pack(case.W.cuda(), N, K, g, qw, sz)
    x = case.x.cuda()
    t = case.t[0]
    side = torch.cuda.Stream()          # non-blocking: no implicit sync with stream 0
    torch.cuda.synchronize()
    with torch.cuda.stream(side):
        stream = ctypes.c_void_p(side.cuda_stream)
        ws = sgq.alloc_workspace(N, K, 1)
        y_ref = torch.empty(1, N, dtype=torch.bfloat16, device="cuda")
        y32_ref = torch.empty(1, N, dtype=torch.float32, device="cuda")
        rc = lib.sgq_gemv_thresh(_ptr(qw), _ptr(sz), N, K, g, _ptr(x), ctypes.c_float(t),
                                 _ptr(y_ref), _ptr(y32_ref), _ptr(ws),
                                 ws.numel() * ws.element_size(), None, stream)
        assert rc == 0
        outs = []
        for _ in range(2):
            y = torch.full((1, N), float("nan"), dtype=torch.bfloat16, device="cuda")
            y32 = torch.full((1, N), float("nan"), dtype=torch.float32, device="cuda")
            rc = lib.sgq_gemv_thresh_noalloc(_ptr(qw), _ptr(sz), N, K, g, _ptr(x),
                                             ctypes.c_float(t), _ptr(y), _ptr(y32), None,
                                             stream)
            assert rc == 0
            outs.append((y, y32))
    side.synchronize()
    tol32 = 1e-3 * sumabs[0]
    for i, (y, y32) in enumerate(outs):
        check_y(y, y32, y64, sumabs, f"noalloc call {i}")
        a = y32.cpu().double().numpy()[0]
        b = y32_ref.cpu().double().numpy()[0]
        assert np.all(np.abs(a - b) <= tol32), f"call {i} vs sgq_gemv_thresh"


# The first call of a process, on a non-blocking stream: the set-up (address
# look-up) and the clear must be ordered before that call's GEMV.
_FRESH = r"""
import ctypes, sys
import numpy as np, torch
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import oracle
from activation_sparse_quantized_b200 import sgq
from activation_sparse_quantized_b200 import workloads as wl
from gpu_common import bits, check_y
torch.cuda.set_device(0)
lib = sgq.load()
shp = wl.LLAMA8B_DOWN
N, K, g = shp["N"], shp["K"], shp["group"]
case = wl.gemv_case(**shp, sparsity=0.5, seed=9, act="silu")
qw, sz = sgq.alloc_packed(N, K, g)
sgq.sgq_pack(case.W.cuda(), N, K, g, qw, sz)
x = case.x.cuda()
torch.cuda.synchronize()
side = torch.cuda.Stream()
p = lambda t: ctypes.c_void_p(t.data_ptr())
with torch.cuda.stream(side):
    y = torch.full((1, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    y32 = torch.full((1, N), float("nan"), dtype=torch.float32, device="cuda")
    rc = lib.sgq_gemv_thresh_noalloc(p(qw), p(sz), N, K, g, p(x), ctypes.c_float(case.t[0]),
                                     p(y), p(y32), None, ctypes.c_void_p(side.cuda_stream))
    assert rc == 0, rc
side.synchronize()
xb = bits(case.x)
q, s, z = oracle.quantize(bits(case.W), g)
y64, sa, _ = oracle.gemv(q, s, z, g, xb, oracle.select(xb, [case.t[0]]))
check_y(y, y32, y64, sa, "first noalloc call of a process")
print("fresh-process noalloc ok")
"""


def test_noalloc_first_call_of_a_fresh_process_on_a_side_stream(lib):
    code = _FRESH.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    assert "fresh-process noalloc ok" in r.stdout


def test_noalloc_rejects_n_above_its_scratch(lib):
    fake = ctypes.c_void_p(1 << 20)
    rc = lib.sgq_gemv_thresh_noalloc(fake, fake, sgq.SGQ_NOALLOC_MAX_N + 32, 4096, 128, fake,
                                     ctypes.c_float(0.5), fake, None, None, None)
    assert rc == -10
    assert b"SGQ_NOALLOC_MAX_N" in lib.sgq_status_string(rc)
