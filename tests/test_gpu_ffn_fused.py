"""Parity of the fused gate + up + GLU GEMV (sgq_gemv_glu / _thresh / _dense)
against the oracle.

The GPU computes gate and up as fp32 sums over the stacked [W_g; W_u] weight
and h = act(gate) * up from them; the oracle computes gate64 and up64 with its
fp64 GEMV and h64 = act(gate64) * up64 in fp64. With the GEMV bound
e = 1e-3 * sum|w x| on each sum, and L the Lipschitz constant of act (1 for
ReLU; SiLU's derivative never exceeds 1.0998, so 1.1), the fp32 h obeys

    |h32 - h64| <= L e_g (|up64| + e_u) + |act(gate64)| e_u
                   + 2^-20 (|act(gate64)| + L e_g)(|up64| + e_u)

(the last term: exp, divide and multiply in fp32, a few ulps), and the bf16 h
adds its rounding, 2^-8 |h64| (with 1% slack on the fp32 term).
"""
import numpy as np
import pytest
import torch

from gpu_common import DEV, bf16_values, bits, check_y, gpu_pack, oracle_codes, sample_rows
from activation_sparse_quantized_b200 import sgq
from activation_sparse_quantized_b200 import workloads as wl
import oracle

pytestmark = pytest.mark.gpu

SILU, RELU = sgq.SGQ_ACT_SILU, sgq.SGQ_ACT_RELU
LIP = {SILU: 1.1, RELU: 1.0}


class GpuGlu:
    """Stacked [W_g; W_u] packed on the device (N = 2I) plus call buffers."""

    def __init__(self, Wg, Wu, group, B=1):
        assert Wg.shape == Wu.shape
        self.I, self.K = Wg.shape
        self.Wg, self.Wu, self.group, self.B = Wg, Wu, group, B
        self.qw, self.sz, _ = gpu_pack(torch.cat([Wg, Wu], 0), group)
        self.ws = sgq.alloc_workspace(2 * self.I, self.K, B)
        self.idx, self.count = sgq.alloc_select(self.K)
        self.status = torch.zeros(1, dtype=torch.int32, device=DEV)

    def outputs(self, B):
        h = torch.full((B, self.I), float("nan"), dtype=torch.bfloat16, device=DEV)
        h32 = torch.full((B, self.I), float("nan"), dtype=torch.float32, device=DEV)
        return h, h32

    def run(self, path, x_d, t, act):
        B = x_d.shape[0]
        h, h32 = self.outputs(B)
        if path == "list":
            sgq.sgq_select(x_d, B, self.K, t, self.idx, self.count)
            sgq.sgq_gemv_glu(self.qw, self.sz, self.I, self.K, self.group, x_d, B, self.idx,
                             self.count, act, h, h32, self.ws, self.status)
        elif path == "thresh":
            sgq.sgq_gemv_glu_thresh(self.qw, self.sz, self.I, self.K, self.group, x_d, t[0],
                                    act, h, h32, self.ws, self.status)
        else:
            sgq.sgq_gemv_glu_dense(self.qw, self.sz, self.I, self.K, self.group, x_d, B, act,
                                   h, h32, self.ws, self.status)
        return h, h32


def fused_expect(Wg, Wu, group, x, t, act, rows=None, dense=False):
    """Oracle h64 (and gate64, up64, sum|wx| of each) for the given outputs."""
    xb = bits(x)
    idx = np.arange(x.shape[1], dtype=np.int32) if dense else oracle.select(xb, t)
    qg, sg, zg = oracle_codes(Wg, group, rows)
    qu, su, zu = oracle_codes(Wu, group, rows)
    g64, sag, _ = oracle.gemv(qg, sg, zg, group, xb, idx)
    u64, sau, _ = oracle.gemv(qu, su, zu, group, xb, idx)
    h64, _ = oracle.act_mul(g64, u64, act)
    a64, _ = oracle.act_mul(g64, np.ones_like(g64), act)
    return idx, h64, a64, u64, sag, sau


def check_h(h, h32, h64, a64, u64, sag, sau, act, rows=None, what=""):
    hb = bf16_values(bits(h))
    hf = h32.detach().cpu().double().numpy()
    if rows is not None:
        hb, hf = hb[:, rows], hf[:, rows]
    L = LIP[act]
    eg, eu = 1e-3 * sag, 1e-3 * sau
    tol32 = (L * eg * (np.abs(u64) + eu) + np.abs(a64) * eu
             + 2.0 ** -20 * (np.abs(a64) + L * eg) * (np.abs(u64) + eu) + 1e-37)
    err = np.abs(hf - h64)
    bad = err > tol32
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} fp32 h beyond bound; "
                           f"worst ratio {np.max(err / tol32):.3g}")
    tolb = tol32 * 1.01 + 2.0 ** -8 * np.abs(h64)
    badb = np.abs(hb - h64) > tolb
    assert not badb.any(), f"{what}: {int(badb.sum())} bf16 h beyond bound"
    return float(np.max(err / tol32))


def weights(I, K, seed):
    return wl.weight(I, K, seed), wl.weight(I, K, seed + 1)


@pytest.mark.parametrize("act", [SILU, RELU])
@pytest.mark.parametrize("path", ["list", "thresh", "dense"])
def test_glu_fused_tiny(act, path):
    I, K, g = 256, 512, 64
    Wg, Wu = weights(I, K, 300 + act)
    x = wl.x_gaussian(1, K, 310)
    t = [wl.percentile_threshold(x[0], 0.5)]
    gg = GpuGlu(Wg, Wu, g)
    h, h32 = gg.run(path, x.to(DEV), t, act)
    idx, h64, a64, u64, sag, sau = fused_expect(Wg, Wu, g, x, t, act, dense=(path == "dense"))
    if path == "list":
        assert np.array_equal(gg.idx[: int(gg.count.item())].cpu().numpy(), idx)
    check_h(h, h32, h64, a64, u64, sag, sau, act, what=f"tiny {path}")
    assert bool((gg.ws == 0).all().item())


@pytest.mark.parametrize("I,K,g", [(1040, 4160, 32), (1040, 4160, 64), (48, 64, 32),
                                   (3088, 1024, 128)])
@pytest.mark.parametrize("path", ["list", "thresh"])
def test_glu_fused_ragged(I, K, g, path):
    """Stacked widths that leave ragged output tiles, odd group counts."""
    Wg, Wu = weights(I, K, 320)
    x = wl.x_silu_gated(1, K, 321)
    t = [wl.percentile_threshold(x[0], 0.5)]
    gg = GpuGlu(Wg, Wu, g)
    h, h32 = gg.run(path, x.to(DEV), t, SILU)
    _, h64, a64, u64, sag, sau = fused_expect(Wg, Wu, g, x, t, SILU)
    check_h(h, h32, h64, a64, u64, sag, sau, SILU, what=f"ragged {I}x{K} g{g} {path}")
    assert bool((gg.ws == 0).all().item())


@pytest.mark.parametrize("path", ["list", "thresh"])
@pytest.mark.parametrize("sparsity", [0.0, 0.5, 0.9])
def test_glu_fused_8b_gate_up(path, sparsity):
    """Llama-3-8B gate/up (4096 -> 14336 each) at the decode-layer sparsities;
    every output checked."""
    shp = wl.LLAMA8B_LAYER["gate"]
    I, K, g = shp["N"], shp["K"], shp["group"]
    Wg, Wu = weights(I, K, 330)
    x = wl.x_gaussian(1, K, 331)
    t = [wl.percentile_threshold(x[0], sparsity) if sparsity > 0 else -1.0]
    gg = GpuGlu(Wg, Wu, g)
    h, h32 = gg.run(path, x.to(DEV), t, SILU)
    _, h64, a64, u64, sag, sau = fused_expect(Wg, Wu, g, x, t, SILU)
    check_h(h, h32, h64, a64, u64, sag, sau, SILU, what=f"8B gate/up {path} {sparsity}")


def test_glu_fused_reglu_chain():
    """ReGLU FFN (hidden 4096, intermediate 11008): dense gate/up with ReLU
    gating, then the down projection skips h's zeros (threshold 0, select
    fused). h is checked on sampled outputs; the down output against the
    oracle run on the GPU's own bf16 h."""
    cfg = wl.REGLU_FFN
    H, I, g = cfg["hidden"], cfg["inter"], cfg["group"]
    Wg, Wu = weights(I, H, 340)
    Wd = wl.weight(H, I, 342)
    x = wl.x_gaussian(1, H, 343)
    gg = GpuGlu(Wg, Wu, g)
    h, h32 = gg.run("dense", x.to(DEV), [-1.0], RELU)
    rows = sample_rows(I, 512, 3)
    _, h64, a64, u64, sag, sau = fused_expect(Wg, Wu, g, x, [-1.0], RELU, rows=rows, dense=True)
    check_h(h, h32, h64, a64, u64, sag, sau, RELU, rows=rows, what="reglu h")
    hbits = bits(h)
    zero_frac = float(np.mean((hbits & 0x7FFF) == 0))
    assert 0.4 < zero_frac < 0.6, zero_frac      # random W_g: about half negative
    # the down projection over the nonzeros of h
    qd, sd, _ = gpu_pack(Wd, g)
    y = torch.full((1, H), float("nan"), dtype=torch.bfloat16, device=DEV)
    y32 = torch.full((1, H), float("nan"), dtype=torch.float32, device=DEV)
    ws = sgq.alloc_workspace(H, I, 1)
    sgq.sgq_gemv_thresh(qd, sd, H, I, g, h, 0.0, y, y32, ws)
    idx = oracle.select(hbits, [0.0])
    assert idx.size == int(np.sum((hbits & 0x7FFF) != 0))
    q, s, z = oracle_codes(Wd, g)
    y64, sa, _ = oracle.gemv(q, s, z, g, hbits, idx)
    check_y(y, y32, y64, sa, "reglu down")


@pytest.mark.parametrize("B", [1, 4, 16])
def test_glu_fused_qwen_batch(B):
    """Qwen3-32B gate/up (5120 -> 25600) at batch B over the union of the rows'
    50% active sets (sampled outputs)."""
    cfg = wl.QWEN32B_FFN
    H, I, g = cfg["hidden"], cfg["inter"], cfg["group"]
    Wg, Wu = weights(I, H, 350)
    x = wl.x_silu_gated(B, H, 351)
    t = [wl.percentile_threshold(x[b], 0.5) for b in range(B)]
    gg = GpuGlu(Wg, Wu, g, B)
    h, h32 = gg.run("list", x.to(DEV), t, SILU)
    rows = sample_rows(I, 256, B)
    _, h64, a64, u64, sag, sau = fused_expect(Wg, Wu, g, x, t, SILU, rows=rows)
    check_h(h, h32, h64, a64, u64, sag, sau, SILU, rows=rows, what=f"qwen gate/up B={B}")
    assert bool((gg.ws == 0).all().item())


def test_glu_fused_all_masked_gives_zero():
    """No active channel: gate = up = 0, so h = act(0) * 0 = +0 everywhere."""
    I, K, g = 512, 1024, 64
    Wg, Wu = weights(I, K, 360)
    x = wl.x_gaussian(1, K, 361)
    gg = GpuGlu(Wg, Wu, g)
    for path in ("list", "thresh"):
        for act in (SILU, RELU):
            h, h32 = gg.run(path, x.to(DEV), [float("inf")], act)
            assert (h32 == 0).all() and bits(h).max() == 0


def test_qkv_stacked_single_gemv():
    """Llama-3-8B q/k/v (4096 -> 4096 / 1024 / 1024) stacked as one weight:
    one threshold-GEMV gives y = q | k | v, each part within the GEMV bound of
    the oracle's own projection, every output checked."""
    L = wl.LLAMA8B_LAYER
    K, g = L["q"]["K"], L["q"]["group"]
    Ws = [wl.weight(L[n]["N"], K, 370 + j) for j, n in enumerate(("q", "k", "v"))]
    W = torch.cat(Ws, 0)
    x = wl.x_gaussian(1, K, 373)
    t = [wl.percentile_threshold(x[0], 0.5)]
    qw, sz, _ = gpu_pack(W, g)
    N = W.shape[0]
    y = torch.full((1, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    y32 = torch.full((1, N), float("nan"), dtype=torch.float32, device=DEV)
    ws = sgq.alloc_workspace(N, K, 1)
    sgq.sgq_gemv_thresh(qw, sz, N, K, g, x.to(DEV), t[0], y, y32, ws)
    xb = bits(x)
    idx = oracle.select(xb, t)
    o = 0
    for Wp, name in zip(Ws, ("q", "k", "v")):
        n = Wp.shape[0]
        q, s, z = oracle_codes(Wp, g)
        y64, sa, _ = oracle.gemv(q, s, z, g, xb, idx)
        check_y(y[:, o:o + n], y32[:, o:o + n], y64, sa, f"stacked {name}")
        o += n


# ---------------------------------------------------------------------------
# sgq_ffn: the decode FFN in three kernels (h formed and selected in the down
# projection's prologue)
# ---------------------------------------------------------------------------

def run_ffn_case(H, I, g, act, t_in_sparsity, t_h_sparsity, seed):
    Wg, Wu = weights(I, H, seed)
    Wd = wl.weight(H, I, seed + 2)
    x = wl.x_gaussian(1, H, seed + 3)
    t_in = wl.percentile_threshold(x[0], t_in_sparsity) if t_in_sparsity > 0 else -1.0
    qgu, sgu, _ = gpu_pack(torch.cat([Wg, Wu], 0), g)
    qd, sd, _ = gpu_pack(Wd, g)
    # oracle h (fp64) for the threshold of h and the h check
    _, h64, a64, u64, sag, sau = fused_expect(Wg, Wu, g, x, [t_in], act)
    hb64 = np.abs(h64[0])
    t_h = 0.0 if t_h_sparsity == 0 else float(np.quantile(hb64, t_h_sparsity))
    ws = sgq.alloc_ffn_workspace(H, I)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    q, s, z = oracle_codes(Wd, g)
    for call in range(2):                      # the workspace must come back to zero
        y = torch.full((1, H), float("nan"), dtype=torch.bfloat16, device=DEV)
        y32 = torch.full((1, H), float("nan"), dtype=torch.float32, device=DEV)
        h = torch.full((1, I), float("nan"), dtype=torch.bfloat16, device=DEV)
        sgq.sgq_ffn(qgu, sgu, qd, sd, H, I, g, x.to(DEV), t_in, act, t_h, y, y32, h, ws, status)
        hbits = bits(h)
        # h against the oracle's fp64 h (the GLU bound, bf16 part)
        hv = bf16_values(hbits)
        L = LIP[act]
        eg, eu = 1e-3 * sag, 1e-3 * sau
        tol = (L * eg * (np.abs(u64) + eu) + np.abs(a64) * eu
               + 2.0 ** -20 * (np.abs(a64) + L * eg) * (np.abs(u64) + eu)) * 1.01 \
            + 2.0 ** -8 * np.abs(h64) + 1e-37
        assert np.all(np.abs(hv - h64) <= tol), f"ffn h call {call}"
        # y against the oracle's down GEMV over the GPU's own h and t_h
        idx = oracle.select(hbits, [t_h])
        y64, sa, _ = oracle.gemv(q, s, z, g, hbits, idx)
        check_y(y, y32, y64, sa, f"ffn y call {call}")
        assert bool((ws == 0).all().item()) and int(status.item()) == 0
    return idx.size / I


def test_ffn_three_kernels_llama8b_silu():
    shp = wl.LLAMA8B_LAYER["gate"]
    frac = run_ffn_case(shp["K"], shp["N"], shp["group"], SILU, 0.5, 0.5, 380)
    assert 0.45 < frac < 0.55


def test_ffn_three_kernels_reglu_zeros():
    """ReGLU: dense input, ReLU gating, t_h = 0: the down projection reads
    exactly the nonzero neurons."""
    cfg = wl.REGLU_FFN
    frac = run_ffn_case(cfg["hidden"], cfg["inter"], cfg["group"], RELU, 0.0, 0.0, 390)
    assert 0.4 < frac < 0.6


@pytest.mark.parametrize("H,I,g", [(512, 1056, 32), (1024, 3136, 64)])
def test_ffn_three_kernels_ragged(H, I, g):
    run_ffn_case(H, I, g, SILU, 0.5, 0.7, 400)


@pytest.mark.parametrize("B,act", [(2, RELU), (4, SILU)])
def test_glu_fused_dense_batch(B, act):
    """Dense gate/up at B > 1 (two batch rows per warp) with the GLU epilogue."""
    I, K, g = 2048, 2048, 128
    Wg, Wu = weights(I, K, 450)
    x = wl.x_gaussian(B, K, 451)
    gg = GpuGlu(Wg, Wu, g, B)
    h, h32 = gg.run("dense", x.to(DEV), [-1.0] * B, act)
    _, h64, a64, u64, sag, sau = fused_expect(Wg, Wu, g, x, [-1.0] * B, act, dense=True)
    check_h(h, h32, h64, a64, u64, sag, sau, act, what=f"dense GLU B={B}")
    assert bool((gg.ws == 0).all().item())
