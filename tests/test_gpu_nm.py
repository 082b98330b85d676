"""Parity of the 2:4 weight-sparse path (sgq_pack_nm, sgq_gemv_nm,
sgq_gemv_nm_thresh) against the oracle: the pruning choice and the packed
layout bit for bit, the GEMV within the GEMV bound (1e-3 * sum|w x| over the
kept weights of the active channels, plus the bf16 rounding)."""
import numpy as np
import pytest
import torch

from gpu_common import DEV, bits, check_y
from activation_sparse_quantized_b200 import sgq
from activation_sparse_quantized_b200 import workloads as wl
import oracle

pytestmark = pytest.mark.gpu


def gpu_pack_nm(W, g):
    N, K = W.shape
    qw, kp, sz = sgq.alloc_packed_nm(N, K, g)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    sgq.sgq_pack_nm(W.to(DEV).contiguous(), N, K, g, qw, kp, sz, status)
    return qw, kp, sz, status


def oracle_nm(W, g, Wq=None):
    """Keep choice from W; codes from Wq (W with non-finite entries zeroed)."""
    Wb = bits(W)
    keep, bad = oracle.nm_keep(Wb, g)
    q, s, z = oracle.quantize(bits(Wq if Wq is not None else W), g)
    return q, s, z, keep, bad


@pytest.mark.parametrize("N,K,g", [(64, 256, 64), (1088, 4160, 32), (4096, 14336, 128)])
def test_pack_nm_bit_exact(N, K, g):
    W = wl.weight(N, K, 400 + g)
    qw, kp, sz, status = gpu_pack_nm(W, g)
    q, s, z, keep, bad = oracle_nm(W, g)
    eqw, ekp, esz = oracle.pack_layout_nm(q, s, z, keep, bad, g)
    assert np.array_equal(qw.cpu().numpy().reshape(K, N // 4), eqw)
    assert np.array_equal(kp.cpu().numpy().reshape(K // g, N // 8), ekp)
    assert np.array_equal(sz.cpu().numpy().view(np.uint16).reshape(K // g, N // 2, 2), esz)
    assert int(status.item()) == 0


def test_pack_nm_ties_and_nonfinite_blocks():
    N, K, g = 128, 256, 64
    W = wl.weight(N, K, 410)
    W[5] = W[4]                       # equal energies
    W[16:20] = W[16]                  # four equal rows
    W[33, 70] = float("nan")          # block 8, group 1
    W[99, 3] = float("inf")           # block 24, group 0
    qw, kp, sz, status = gpu_pack_nm(W, g)
    Wq = W.clone()
    Wq[33, 70] = 0.0
    Wq[99, 3] = 0.0
    q, s, z, keep, bad = oracle_nm(W, g, Wq)
    assert bad.sum() == 2 and bad[1, 8] == 1 and bad[0, 24] == 1
    eqw, ekp, esz = oracle.pack_layout_nm(q, s, z, keep, bad, g)
    assert np.array_equal(qw.cpu().numpy().reshape(K, N // 4), eqw)
    assert np.array_equal(kp.cpu().numpy().reshape(K // g, N // 8), ekp)
    assert np.array_equal(sz.cpu().numpy().view(np.uint16).reshape(K // g, N // 2, 2), esz)
    assert int(status.item()) & sgq.SGQ_STATUS_NONFINITE_W


def run_nm_case(case, path, what=""):
    W, g = case.W, case.group
    N, K = W.shape
    qw, kp, sz, _ = gpu_pack_nm(W, g)
    x_d = case.x.to(DEV)
    y = torch.full((1, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    y32 = torch.full((1, N), float("nan"), dtype=torch.float32, device=DEV)
    ws = sgq.alloc_workspace(N, K, 1)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    if path == "list":
        idx, cnt = sgq.alloc_select(K)
        sgq.sgq_select(x_d, 1, K, case.t, idx, cnt)
        sgq.sgq_gemv_nm(qw, kp, sz, N, K, g, x_d, idx, cnt, y, y32, ws, status)
    else:
        sgq.sgq_gemv_nm_thresh(qw, kp, sz, N, K, g, x_d, case.t[0], y, y32, ws, status)
    q, s, z, keep, bad = oracle_nm(W, g)
    xb = bits(case.x)
    oidx = oracle.select(xb, case.t)
    y64, sa, _ = oracle.gemv_nm(q, s, z, keep, bad, g, xb, oidx)
    check_y(y, y32, y64, sa, what)
    assert bool((ws == 0).all().item()) and int(status.item()) == 0
    # pruned outputs get contributions too (every block keeps two): nothing is
    # left unwritten
    assert not torch.isnan(y32).any()


@pytest.mark.parametrize("path", ["list", "thresh"])
@pytest.mark.parametrize("sparsity", [0.0, 0.5, 0.9])
def test_gemv_nm_8b_down(path, sparsity):
    case = wl.gemv_case(**wl.LLAMA8B_DOWN, sparsity=sparsity, seed=420)
    run_nm_case(case, path, what=f"2:4 8B down {path} {sparsity}")


@pytest.mark.parametrize("N,K,g", [(64, 256, 64), (1088, 4160, 32), (3136, 8192, 128),
                                   (4096, 4096, 64)])
@pytest.mark.parametrize("path", ["list", "thresh"])
def test_gemv_nm_ragged(N, K, g, path):
    """Partial 2048-output tiles, odd channel slices and group spans."""
    case = wl.gemv_case(N=N, K=K, group=g, sparsity=0.5, seed=421)
    run_nm_case(case, path, what=f"2:4 ragged {N}x{K} g{g} {path}")


def test_gemv_nm_all_masked_gives_positive_zero():
    case = wl.gemv_case(N=1024, K=2048, group=128, sparsity=0.5, seed=422)
    N, K, g = 1024, 2048, 128
    qw, kp, sz, _ = gpu_pack_nm(case.W, g)
    y = torch.full((1, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    y32 = torch.full((1, N), float("nan"), dtype=torch.float32, device=DEV)
    ws = sgq.alloc_workspace(N, K, 1)
    sgq.sgq_gemv_nm_thresh(qw, kp, sz, N, K, g, case.x.to(DEV), float("inf"), y, y32, ws)
    assert (y32 == 0).all() and not torch.signbit(y32).any() and bits(y).max() == 0
