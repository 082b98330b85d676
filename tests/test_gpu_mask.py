"""Parity of the bitmask active set (sgq_select_mask, sgq_gemv_mask) against
the oracle: the mask and its count bit for bit, the GEMV within the GEMV bound
(1e-3 * sum|w x| on the fp32 result, plus the bf16 rounding)."""
import numpy as np
import pytest
import torch

from gpu_common import DEV, bits, check_y, gpu_pack, oracle_codes, sample_rows
from activation_sparse_quantized_b200 import sgq
from activation_sparse_quantized_b200 import workloads as wl
import oracle

pytestmark = pytest.mark.gpu


def gpu_mask(x_d, t):
    B, K = x_d.shape
    m = torch.full(((K + 31) // 32,), -1, dtype=torch.int32, device=DEV)   # garbage first
    c = torch.full((1,), -7, dtype=torch.int32, device=DEV)
    sgq.sgq_select_mask(x_d, B, K, t, m, c)
    return m.cpu().numpy().view(np.uint32), int(c.item())


@pytest.mark.parametrize("K", [8, 256, 8192, 8200, 14336, 25600])
@pytest.mark.parametrize("sparsity", [0.0, 0.5, 0.9, 1.0])
def test_select_mask_bit_exact(K, sparsity):
    x = wl.x_silu_gated(1, K, K + int(sparsity * 10))
    t = [wl.percentile_threshold(x[0], sparsity) if sparsity < 1 else float("inf")]
    m, c = gpu_mask(x.to(DEV), t)
    mo, co = oracle.select_mask(bits(x), t)
    assert np.array_equal(m, mo) and c == co


@pytest.mark.parametrize("B", [2, 3, 8, 16])
def test_select_mask_union_bit_exact(B):
    K = 5120
    x = wl.x_silu_gated(B, K, 40 + B)
    t = [wl.percentile_threshold(x[b], 0.7) for b in range(B)]
    m, c = gpu_mask(x.to(DEV), t)
    mo, co = oracle.select_mask(bits(x), t)
    assert np.array_equal(m, mo) and c == co


def test_select_mask_edge_values():
    vals = torch.tensor([0.0, -0.0, 1.0, -1.0, float("nan"), float("inf"), float("-inf"), 0.5,
                         -0.5, 2.0 ** -130, 3.0, -3.0, 0.0, 0.0, 7.0, -7.0])
    x = vals.repeat(40).reshape(1, -1).to(torch.bfloat16)
    for t in (0.0, 0.5, -1.0, float("inf"), 2.0 ** -131):
        m, c = gpu_mask(x.to(DEV), [t])
        mo, co = oracle.select_mask(bits(x), [t])
        assert np.array_equal(m, mo) and c == co


def run_mask_case(case, rows=None, what=""):
    N, K, g, B = case.W.shape[0], case.W.shape[1], case.group, case.B
    qw, sz, _ = gpu_pack(case.W, g)
    x_d = case.x.to(DEV)
    m = sgq.alloc_mask(K)
    sgq.sgq_select_mask(x_d, B, K, case.t, m)
    y = torch.full((B, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    y32 = torch.full((B, N), float("nan"), dtype=torch.float32, device=DEV)
    ws = sgq.alloc_workspace(N, K, B)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    sgq.sgq_gemv_mask(qw, sz, N, K, g, x_d, B, m, y, y32, ws, status)
    xb = bits(case.x)
    idx = oracle.select(xb, case.t)
    q, s, z = oracle_codes(case.W, g, rows)
    y64, sa, _ = oracle.gemv(q, s, z, g, xb, idx)
    if rows is not None:
        y, y32 = y[:, rows], y32[:, rows]
    check_y(y, y32, y64, sa, what)
    assert bool((ws == 0).all().item()) and int(status.item()) == 0


@pytest.mark.parametrize("sparsity", [0.0, 0.5, 0.9])
def test_gemv_mask_8b_down(sparsity):
    case = wl.gemv_case(**wl.LLAMA8B_DOWN, sparsity=sparsity, seed=60)
    run_mask_case(case, what=f"mask 8B down {sparsity}")


@pytest.mark.parametrize("N,K,g", [(96, 64, 32), (3168, 4160, 64), (512, 8320, 64),
                                   (1056, 8000, 32)])
def test_gemv_mask_ragged(N, K, g):
    """Ragged output tiles and channel slices (K is a multiple of the group,
    hence of 32, so every mask word is whole)."""
    case = wl.gemv_case(N=N, K=K, group=g, sparsity=0.5, seed=61)
    run_mask_case(case, what=f"mask ragged {N}x{K}")


@pytest.mark.parametrize("B", [2, 4, 5, 6, 16])
def test_gemv_mask_qwen_down_batch(B):
    cfg = wl.QWEN32B_FFN
    case = wl.gemv_case(N=cfg["hidden"], K=cfg["inter"], group=cfg["group"], B=B,
                        sparsity=0.5, seed=62, act="silu")
    run_mask_case(case, rows=sample_rows(cfg["hidden"], 256, B), what=f"mask qwen B={B}")


def test_gemv_mask_empty_gives_positive_zero():
    case = wl.gemv_case(**wl.TINY, sparsity=0.5, seed=63)
    N, K, g = case.W.shape[0], case.W.shape[1], case.group
    qw, sz, _ = gpu_pack(case.W, g)
    m = sgq.alloc_mask(K)
    y = torch.full((1, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    y32 = torch.full((1, N), float("nan"), dtype=torch.float32, device=DEV)
    ws = sgq.alloc_workspace(N, K, 1)
    sgq.sgq_gemv_mask(qw, sz, N, K, g, case.x.to(DEV), 1, m, y, y32, ws)
    assert (y32 == 0).all() and not torch.signbit(y32).any() and bits(y).max() == 0


# ---------------------------------------------------------------------------
# accumulating forms (y_acc += the GEMV, one kernel)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("path,B", [("thresh", 1), ("list", 1), ("list", 4)])
def test_gemv_acc_adds_into_fp32_buffer(path, B):
    """y_acc starts at random r0; afterwards y_acc - r0 must be the GEMV within
    its bound plus the fp32 roundings of adding into r0 (at most one per
    split-K share and one for r0 itself: 64 ulps of |r0| + sum|wx| is ample)."""
    case = wl.gemv_case(**wl.LLAMA8B_DOWN, B=B, sparsity=0.5, seed=430)
    N, K, g = case.W.shape[0], case.W.shape[1], case.group
    qw, sz, _ = gpu_pack(case.W, g)
    x_d = case.x.to(DEV)
    r0 = torch.randn(B, N, generator=torch.Generator().manual_seed(431)) * 3
    y_acc = r0.clone().to(DEV)
    if path == "thresh":
        sgq.sgq_gemv_thresh_acc(qw, sz, N, K, g, x_d, case.t[0], y_acc)
    else:
        idx, cnt = sgq.alloc_select(K)
        sgq.sgq_select(x_d, B, K, case.t, idx, cnt)
        sgq.sgq_gemv_acc(qw, sz, N, K, g, x_d, B, idx, cnt, y_acc)
    xb = bits(case.x)
    oidx = oracle.select(xb, case.t)
    q, s, z = oracle_codes(case.W, g)
    y64, sa, _ = oracle.gemv(q, s, z, g, xb, oidx)
    got = y_acc.cpu().double().numpy() - r0.double().numpy()
    tol = 1e-3 * sa + 64 * 2.0 ** -24 * (np.abs(r0.double().numpy()) + sa)
    assert np.all(np.abs(got - y64) <= tol)
