"""Parity of the fused batch threshold GEMV (sgq_gemv_thresh_batch and
sgq_gemv_glu_thresh_batch) against the oracle.

At batch B the active set is the union over the rows of {k : |x[b][k]| > t_b}
("Enabling Dynamic Sparsity in Quantized LLM Inference", Abstract: the active
indices are gathered at run time); every row then multiplies over that one set
unmasked. The fused entry points find the union inside the GEMV (each CTA
thresholds all B rows of its channel slice), so the expectation is the
oracle's select over the rows followed by its GEMV over that list, checked
with the suite's tolerance (1e-3 * sum |w x| on the fp32 result, plus the bf16
rounding of y). B = 2 and 5 run on the CUDA-core kernel, B = 9, 12 and 16 on
the tensor-core kernel.
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_common import DEV, GpuGemv, bits, check_y, oracle_codes, sample_rows
from test_gpu_ffn_fused import GpuGlu, check_h, fused_expect
from activation_sparse_quantized_b200 import sgq
from activation_sparse_quantized_b200 import workloads as wl
import oracle

pytestmark = pytest.mark.gpu


def _thresh_batch(g, x_d, t):
    B = x_d.shape[0]
    y, y32 = g.outputs(B)
    sgq.sgq_gemv_thresh_batch(g.qw, g.sz, g.N, g.K, g.group, x_d, B, t, y, y32, g.ws,
                              g.status)
    return y, y32


@pytest.mark.parametrize("B", [2, 5, 9, 16])
@pytest.mark.parametrize("N,K,g", [(3168, 4160, 64), (96, 64, 32)])
def test_thresh_batch_matches_select_then_gemv(N, K, g, B):
    """Several tiles and a ragged tail (N = 3 x 1024 + 96), per-row 50%
    thresholds that differ between rows."""
    case = wl.gemv_case(N, K, g, B=B, sparsity=0.5, seed=40 + B, act="silu")
    gg = GpuGemv(case.W, g, B)
    x = case.x.to(DEV)
    y, y32 = _thresh_batch(gg, x, case.t)
    torch.cuda.synchronize()
    idx = oracle.select(bits(case.x), case.t)
    q, s, z = oracle_codes(case.W, g)
    y64, sa, _ = oracle.gemv(q, s, z, g, bits(case.x), idx)
    check_y(y, y32, y64, sa, f"thresh_batch B={B}")
    assert gg.workspace_is_zero()
    assert sgq.sgq_read_status(gg.status) == 0
    # the same union through the list path (sgq_select + sgq_gemv) agrees too
    gg.select(x, case.t)
    assert np.array_equal(gg.active(), idx)
    yl, yl32 = gg.gemv(x)
    torch.cuda.synchronize()
    check_y(yl, yl32, y64, sa, f"list B={B}")


@pytest.mark.parametrize("B", [3, 12])
def test_thresh_batch_one_row_selects_everything(B):
    """t < 0 on one row makes the union every channel: the dense GEMV."""
    N, K, g = 1056, 1024, 128
    case = wl.gemv_case(N, K, g, B=B, sparsity=0.9, seed=7, act="gaussian")
    t = list(case.t)
    t[B // 2] = -1.0
    gg = GpuGemv(case.W, g, B)
    y, y32 = _thresh_batch(gg, case.x.to(DEV), t)
    torch.cuda.synchronize()
    q, s, z = oracle_codes(case.W, g)
    y64, sa, _ = oracle.gemv_dense(q, s, z, g, bits(case.x))
    check_y(y, y32, y64, sa, f"union = all, B={B}")


@pytest.mark.parametrize("B", [3, 12])
def test_thresh_batch_all_masked_gives_positive_zero(B):
    N, K, g = 2080, 512, 64
    case = wl.gemv_case(N, K, g, B=B, sparsity=0.5, seed=8)
    gg = GpuGemv(case.W, g, B)
    y, y32 = gg.outputs(B)
    y.fill_(float("nan"))
    sgq.sgq_gemv_thresh_batch(gg.qw, gg.sz, N, K, g, case.x.to(DEV), B, [1e30] * B, y, y32,
                              gg.ws, gg.status)
    torch.cuda.synchronize()
    assert np.all(bits(y) == 0), "all-masked rows must give +0"
    assert gg.workspace_is_zero()


@pytest.mark.parametrize("B", [4, 10])
def test_thresh_batch_edge_values(B):
    """NaN is never active and +-0 is not above t >= 0: channels whose rows
    hold only such values are left out, and the others follow the rule."""
    N, K, g = 1024, 256, 32
    case = wl.gemv_case(N, K, g, B=B, sparsity=0.5, seed=9, act="gaussian")
    x = case.x.clone()
    x[:, 3] = float("nan")             # NaN in every row: inactive
    x[:, 17] = 0.0
    x[1:, 18] = -0.0                   # +-0 everywhere: inactive at t >= 0
    x[0, 18] = 0.0
    t = [max(v, 0.0) for v in case.t]
    gg = GpuGemv(case.W, g, B)
    y, y32 = _thresh_batch(gg, x.to(DEV), t)
    torch.cuda.synchronize()
    idx = oracle.select(bits(x), t)
    assert 3 not in idx and 17 not in idx and 18 not in idx
    q, s, z = oracle_codes(case.W, g)
    y64, sa, _ = oracle.gemv(q, s, z, g, bits(x), idx)
    check_y(y, y32, y64, sa, f"edge values B={B}")


@pytest.mark.parametrize("B", [2, 5, 16])
def test_thresh_batch_qwen_down_sampled(B):
    """The Qwen3-32B down_proj shape (K = 25600, N = 5120, g128) in the launch
    configuration the benchmark uses, checked on sampled outputs."""
    shp = dict(N=5120, K=25600, group=128)
    case = wl.gemv_case(**shp, B=B, sparsity=0.5, seed=60 + B, act="silu")
    gg = GpuGemv(case.W, shp["group"], B)
    y, y32 = _thresh_batch(gg, case.x.to(DEV), case.t)
    torch.cuda.synchronize()
    rows = sample_rows(shp["N"], 48, seed=B)
    idx = oracle.select(bits(case.x), case.t)
    q, s, z = oracle_codes(case.W, shp["group"], rows)
    y64, sa, _ = oracle.gemv(q, s, z, shp["group"], bits(case.x), idx)
    check_y(y[:, rows], y32[:, rows], y64, sa, f"qwen down B={B}")
    assert gg.workspace_is_zero()


@pytest.mark.parametrize("B", [2, 5, 8, 16])
def test_glu_thresh_batch_qwen_gate_up_sampled(B):
    """The Qwen3-32B stacked gate/up shape (K = 5120, I = 25600: 50 output
    tiles, equal per-SM shares that span tile boundaries) through the fused
    GLU form at batch B, checked on sampled outputs of h."""
    I, K, g = 25600, 5120, 128
    Wg, Wu = wl.weight(I, K, 80), wl.weight(I, K, 81)
    x = wl.x_silu_gated(B, K, 82 + B)
    t = [wl.percentile_threshold(x[b], 0.5) for b in range(B)]
    gl = GpuGlu(Wg, Wu, g, B)
    h, h32 = gl.outputs(B)
    sgq.sgq_gemv_glu_thresh_batch(gl.qw, gl.sz, I, K, g, x.to(DEV), B, t, sgq.SGQ_ACT_SILU, h,
                                  h32, gl.ws, gl.status)
    torch.cuda.synchronize()
    rows = sample_rows(I, 40, seed=B)
    _, h64, a64, u64, sag, sau = fused_expect(Wg, Wu, g, x, t, sgq.SGQ_ACT_SILU, rows=rows)
    check_h(h, h32, h64, a64, u64, sag, sau, sgq.SGQ_ACT_SILU, rows=rows,
            what=f"qwen gate/up B={B}")
    assert bool((gl.ws == 0).all().item())
    assert sgq.sgq_read_status(gl.status) == 0


@pytest.mark.parametrize("B", [2, 5, 16])
@pytest.mark.parametrize("act", [sgq.SGQ_ACT_SILU, sgq.SGQ_ACT_RELU])
def test_glu_thresh_batch(B, act):
    """The fused gate/up GLU at batch B with the rows' union found in the GEMV."""
    I, K, g = 1056, 1024, 64
    Wg, Wu = wl.weight(I, K, 70), wl.weight(I, K, 71)
    x = wl.x_silu_gated(B, K, 72 + B)
    t = [wl.percentile_threshold(x[b], 0.5) for b in range(B)]
    gl = GpuGlu(Wg, Wu, g, B)
    h, h32 = gl.outputs(B)
    sgq.sgq_gemv_glu_thresh_batch(gl.qw, gl.sz, I, K, g, x.to(DEV), B, t, act, h, h32, gl.ws,
                                  gl.status)
    torch.cuda.synchronize()
    _, h64, a64, u64, sag, sau = fused_expect(Wg, Wu, g, x, t, act)
    check_h(h, h32, h64, a64, u64, sag, sau, act, what=f"glu_thresh_batch B={B}")
    assert bool((gl.ws == 0).all().item())


def test_thresh_batch_rejects_bad_arguments():
    gg = GpuGemv(wl.weight(64, 64, 1), 32, 2)
    x = wl.x_gaussian(2, 64, 2).to(DEV)
    y, y32 = gg.outputs(2)
    lib = sgq.load()
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    tt = (ctypes.c_float * 2)(0.5, 0.5)
    nb = gg.ws.numel() * gg.ws.element_size()
    assert lib.sgq_gemv_thresh_batch(P(gg.qw), P(gg.sz), 64, 64, 32, P(x), 17, tt, P(y), None,
                                     P(gg.ws), nb, None, None) == -5
    assert lib.sgq_gemv_thresh_batch(P(gg.qw), P(gg.sz), 64, 64, 32, P(x), 2, None, P(y), None,
                                     P(gg.ws), nb, None, None) == -1
