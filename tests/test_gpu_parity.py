"""Parity of the CUDA path (called through the C ABI) with the CPU oracle on a
B200: packing and selection bit for bit, GEMV outputs within the tolerance
stated in gpu_common, on the shapes and distributions of the workloads plus
ragged and degenerate cases."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import (DEV, GpuGemv, bf16_values, bits, check_y, gpu_pack, oracle_codes,
                        oracle_expect, packed_codes_rows, sample_rows, sz_rows)
from activation_sparse_quantized_b200 import sgq
from activation_sparse_quantized_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from activation_sparse_quantized_b200 import build
    build.build()
    sgq.load()
    torch.cuda.set_device(0)


# ---------------------------------------------------------------------------
# sgq_pack: bit-exact against the oracle's quantizer + layout
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("N,K,g,seed", [
    (512, 256, 64, 0),        # tiny config
    (96, 64, 32, 1),          # one partial tile
    (3168, 4160, 64, 2),      # ragged: 3 tiles + 96 outputs
    (1024, 4096, 128, 3),
])
def test_pack_bit_exact(N, K, g, seed):
    W = wl.weight(N, K, seed)
    qw, sz, st = gpu_pack(W, g)
    q, s, z = oracle_codes(W, g)
    qw_o, sz_o = oracle.pack_layout(q, s, z, g)
    torch.cuda.synchronize()
    assert np.array_equal(qw.cpu().numpy().reshape(K, N // 2), qw_o)
    assert np.array_equal(sz.cpu().numpy().view(np.uint16).reshape(K // g, N, 2), sz_o)
    assert st.item() == 0


def test_pack_bit_exact_full_8b_down():
    N, K, g = wl.LLAMA8B_DOWN["N"], wl.LLAMA8B_DOWN["K"], wl.LLAMA8B_DOWN["group"]
    W = wl.weight(N, K, 0)
    qw, sz, st = gpu_pack(W, g)
    q, s, z = oracle_codes(W, g)
    qw_o, sz_o = oracle.pack_layout(q, s, z, g)
    assert np.array_equal(qw.cpu().numpy().reshape(K, N // 2), qw_o)
    assert np.array_equal(sz.cpu().numpy().view(np.uint16).reshape(K // g, N, 2), sz_o)


def test_pack_special_groups():
    """Zero groups, one-signed groups, exact ties, fp16 extremes and subnormals."""
    N, K, g = 64, 128, 32
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    W[0, :32] = 0
    W[1, :32] = np.abs(W[1, :32])
    W[2, :32] = -np.abs(W[2, :32])
    W[3, :32] = np.array([-0.4375, 0.0625, 0.5, 1.4375] * 8, np.float16)   # ties
    W[4, :32] = np.float16(65504.0)
    W[5, :32] = np.float16(-65504.0)
    W[6, :32] = (rng.standard_normal(32) * 1e-6).astype(np.float16)         # subnormals
    W[7, 32:64] = np.float16(6e-8)
    W[8] = np.linspace(-1, 1, K).astype(np.float16)
    Wt = torch.from_numpy(W)
    qw, sz, st = gpu_pack(Wt, g)
    q, s, z = oracle_codes(Wt, g)
    qw_o, sz_o = oracle.pack_layout(q, s, z, g)
    assert np.array_equal(qw.cpu().numpy().reshape(K, N // 2), qw_o)
    assert np.array_equal(sz.cpu().numpy().view(np.uint16).reshape(K // g, N, 2), sz_o)
    assert st.item() == 0


def test_pack_flags_nonfinite():
    W = wl.weight(64, 128, 7)
    W[5, 17] = float("nan")
    W[9, 100] = float("inf")
    _, _, st = gpu_pack(W, 64)
    assert st.item() & sgq.SGQ_STATUS_NONFINITE_W


# ---------------------------------------------------------------------------
# sgq_select: bit-exact against the oracle
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("K", [8, 256, 2048, 2056, 8192, 8200, 14336, 25600, 65536])
@pytest.mark.parametrize("sparsity", [0.0, 0.3, 0.5, 0.7, 0.9, 1.0])
def test_select_bit_exact(K, sparsity):
    x = wl.x_silu_gated(1, K, 11)
    t = [wl.percentile_threshold(x[0], sparsity)]
    idx, cnt = sgq.alloc_select(K)
    sgq.sgq_select(x.to(DEV), 1, K, t, idx, cnt)
    ref = oracle.select(bits(x), t)
    n = int(cnt.item())
    assert n == ref.size
    assert np.array_equal(idx[:n].cpu().numpy(), ref)


def test_select_edge_values():
    vals = torch.tensor([0.0, -0.0, 1.0, -1.0, float("nan"), float("inf"), float("-inf"), 0.5,
                         -0.5, 2.0 ** -130, 3.0, -3.0, 0.0, 0.0, 7.0, -7.0],
                        dtype=torch.float32).to(torch.bfloat16)[None, :]
    idx, cnt = sgq.alloc_select(16)
    for t in (0.0, 0.5, -1.0, float("inf"), 2.0 ** -131):
        sgq.sgq_select(vals.to(DEV), 1, 16, [t], idx, cnt)
        ref = oracle.select(bits(vals), [t])
        n = int(cnt.item())
        assert np.array_equal(idx[:n].cpu().numpy(), ref), t


@pytest.mark.parametrize("B", [2, 3, 4, 8, 16])
def test_select_union_bit_exact(B):
    K = 5120
    x = wl.x_silu_gated(B, K, 13)
    t = [wl.percentile_threshold(x[b], 0.5) for b in range(B)]
    idx, cnt = sgq.alloc_select(K)
    sgq.sgq_select(x.to(DEV), B, K, t, idx, cnt)
    ref = oracle.select(bits(x), t)
    n = int(cnt.item())
    assert np.array_equal(idx[:n].cpu().numpy(), ref)


def test_select_relu_zeros():
    x = wl.x_relu_shifted(1, 11008, 3)
    idx, cnt = sgq.alloc_select(11008)
    sgq.sgq_select(x.to(DEV), 1, 11008, [0.0], idx, cnt)
    ref = oracle.select(bits(x), [0.0])
    n = int(cnt.item())
    assert np.array_equal(idx[:n].cpu().numpy(), ref)
    assert 0.08 < n / 11008 < 0.16


# ---------------------------------------------------------------------------
# sgq_gemv: tolerance against the oracle
# ---------------------------------------------------------------------------

def run_list_case(case, rows=None, what=""):
    g = GpuGemv(case.W, case.group, case.B)
    x_d = case.x.to(DEV)
    g.select(x_d, case.t)
    y, y32 = g.gemv(x_d)
    idx, y64, sa, _ = oracle_expect(case.W, case.group, case.x, case.t, rows)
    torch.cuda.synchronize()
    assert np.array_equal(g.active(), idx)
    if rows is not None:
        y, y32 = y[:, rows], y32[:, rows]
    ratio = check_y(y, y32, y64, sa, what)
    assert g.workspace_is_zero()
    assert g.status.item() == 0
    return ratio


@pytest.mark.parametrize("sparsity", [0.0, 0.5, 0.9])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_gemv_tiny(sparsity, seed):
    case = wl.gemv_case(**wl.TINY, sparsity=sparsity, seed=seed)
    run_list_case(case, what="tiny")


@pytest.mark.parametrize("N,K,g", [(96, 64, 32), (3168, 4160, 64), (3168, 4160, 32),
                                   (32, 128, 128), (2080, 384, 128)])
def test_gemv_ragged(N, K, g):
    case = wl.gemv_case(N, K, g, sparsity=0.5, seed=4)
    run_list_case(case, what=f"ragged {N}x{K}")


@pytest.mark.parametrize("sparsity", wl.SPARSITY_SWEEP)
def test_gemv_8b_down_sweep(sparsity):
    case = wl.gemv_case(**wl.LLAMA8B_DOWN, sparsity=sparsity, seed=0, act="silu")
    run_list_case(case, what=f"8B down {sparsity}")


@pytest.mark.parametrize("proj", list(wl.LLAMA8B_LAYER))
def test_gemv_8b_layer(proj):
    shp = wl.LLAMA8B_LAYER[proj]
    act = "silu" if proj == "down" else "gaussian"
    case = wl.gemv_case(**shp, sparsity=0.5, seed=10, act=act)
    rows = sample_rows(shp["N"], 1024, 1) if shp["N"] > 8192 else None
    run_list_case(case, rows=rows, what=proj)


def test_gemv_reglu_down_shifted_relu():
    case = wl.gemv_case(N=4096, K=11008, group=128, sparsity=0.0, seed=3, act="relu_shifted")
    run_list_case(case, what="reglu down")


@pytest.mark.parametrize("B", wl.QWEN_BATCHES)
def test_gemv_qwen_down_batch(B):
    h, I = wl.QWEN32B_FFN["hidden"], wl.QWEN32B_FFN["inter"]
    case = wl.gemv_case(N=h, K=I, group=128, B=B, sparsity=0.5, seed=20 + B, act="silu")
    run_list_case(case, rows=sample_rows(h, 256, B), what=f"qwen down B={B}")


@pytest.mark.parametrize("B", [1, 4, 5, 16])
def test_gemv_qwen_up_batch(B):
    h, I = wl.QWEN32B_FFN["hidden"], wl.QWEN32B_FFN["inter"]
    case = wl.gemv_case(N=I, K=h, group=128, B=B, sparsity=0.5, seed=40 + B)
    run_list_case(case, rows=sample_rows(I, 256, B), what=f"qwen up B={B}")


@pytest.mark.parametrize("B", [2, 3, 4, 5, 6, 7, 8, 9, 16])
def test_gemv_batch_ragged(B):
    case = wl.gemv_case(N=3168, K=4160, group=64, B=B, sparsity=0.6, seed=50 + B)
    run_list_case(case, what=f"ragged B={B}")


def test_gemv_batch_rows_match_single():
    """Row b of a batched call equals the single-row GEMV of x_b on the union list."""
    case = wl.gemv_case(N=2048, K=4096, group=128, B=4, sparsity=0.5, seed=60)
    g = GpuGemv(case.W, 128, 4)
    x_d = case.x.to(DEV)
    g.select(x_d, case.t)
    _, y32 = g.gemv(x_d)
    idx, y64, sa, _ = oracle_expect(case.W, 128, case.x, case.t)
    for b in range(4):
        _, yb32 = g.gemv(x_d[b:b + 1].contiguous())
        err = np.abs(yb32.cpu().double().numpy()[0] - y32.cpu().double().numpy()[b])
        assert np.all(err <= 2e-3 * sa[b])


def test_gemv_dense_matches_oracle_and_full_list():
    case = wl.gemv_case(**wl.LLAMA8B_DOWN, sparsity=0.0, seed=1, act="silu")
    g = GpuGemv(case.W, 128)
    x_d = case.x.to(DEV)
    y, y32 = g.dense(x_d)
    q, s, z = oracle_codes(case.W, 128)
    y64, sa, _ = oracle.gemv_dense(q, s, z, 128, bits(case.x))
    check_y(y, y32, y64, sa, "dense")
    assert g.workspace_is_zero()


@pytest.mark.parametrize("B", [2, 4, 5, 8, 12])
def test_gemv_dense_batch(B):
    case = wl.gemv_case(N=1024, K=4096, group=128, B=B, sparsity=0.0, seed=70)
    g = GpuGemv(case.W, 128, B)
    y, y32 = g.dense(case.x.to(DEV))
    q, s, z = oracle_codes(case.W, 128)
    y64, sa, _ = oracle.gemv_dense(q, s, z, 128, bits(case.x))
    check_y(y, y32, y64, sa, f"dense B={B}")


@pytest.mark.parametrize("B,g", [(5, 64), (9, 32), (12, 128), (16, 64)])
def test_gemv_batch_unsorted_list_with_repeats(B, g):
    """A caller's index list in no order, with repeated channels, at batch
    sizes of the tensor-core kernel: the list is cut into runs of one group
    wherever the group changes, and a repeated channel counts once per entry,
    as in the oracle's sum over the list. N = 2080 leaves a ragged tile."""
    N, K = 2080, 4096
    case = wl.gemv_case(N=N, K=K, group=g, B=B, sparsity=0.0, seed=90 + B)
    rng = np.random.default_rng(B)
    idx = rng.permutation(K)[: K // 2]
    idx = np.concatenate([idx, idx[:200]]).astype(np.int32)
    rng.shuffle(idx)
    gg = GpuGemv(case.W, g, B)
    idx_d = torch.tensor(idx, dtype=torch.int32, device=DEV)
    cnt = torch.tensor([idx.size], dtype=torch.int32, device=DEV)
    y, y32 = gg.gemv(case.x.to(DEV), idx_d, cnt)
    q, s, z = oracle_codes(case.W, g)
    y64, sa, _ = oracle.gemv(q, s, z, g, bits(case.x), idx)
    torch.cuda.synchronize()
    check_y(y, y32, y64, sa, f"unsorted list B={B} g={g}")
    assert gg.workspace_is_zero()
    assert gg.status.item() == 0


@pytest.mark.parametrize("B,order", [(1, "sorted"), (3, "sorted"), (1, "unsorted"), (5, "unsorted")])
def test_gemv_list_equal_shares_over_tiles(B, order):
    """40 tiles (N = 40928, the last one ragged): whole splits per tile would
    leave SMs idle, so the CUDA-core kernel gives each SM an equal share of
    the (tile, list entry) space, some shares spanning two tiles."""
    N, K, g = 40928, 2048, 64
    case = wl.gemv_case(N=N, K=K, group=g, B=B, sparsity=0.5, seed=120 + B)
    gg = GpuGemv(case.W, g, B)
    x_d = case.x.to(DEV)
    if order == "sorted":
        gg.select(x_d, case.t)
        idx = gg.active()
        y, y32 = gg.gemv(x_d)
    else:
        rng = np.random.default_rng(B)
        idx = rng.permutation(K)[: K // 3]
        idx = np.concatenate([idx, idx[:50]]).astype(np.int32)
        rng.shuffle(idx)
        idx_d = torch.tensor(idx, dtype=torch.int32, device=DEV)
        cnt = torch.tensor([idx.size], dtype=torch.int32, device=DEV)
        y, y32 = gg.gemv(x_d, idx_d, cnt)
    rows = sample_rows(N, 512, B)
    q, s, z = oracle_codes(case.W, g, rows)
    y64, sa, _ = oracle.gemv(q, s, z, g, bits(case.x), idx)
    torch.cuda.synchronize()
    check_y(y[:, rows], y32[:, rows], y64, sa, f"equal shares B={B} {order}")
    assert gg.workspace_is_zero()
    assert gg.status.item() == 0


@pytest.mark.parametrize("sparsity", [0.0, 0.5, 0.9])
def test_gemv_thresh_matches_oracle(sparsity):
    case = wl.gemv_case(**wl.LLAMA8B_DOWN, sparsity=sparsity, seed=2, act="silu")
    g = GpuGemv(case.W, 128)
    y, y32 = g.thresh(case.x.to(DEV), case.t[0])
    _, y64, sa, _ = oracle_expect(case.W, 128, case.x, case.t)
    check_y(y, y32, y64, sa, "thresh")
    assert g.workspace_is_zero()


@pytest.mark.parametrize("N,K,g", [(512, 256, 64), (3168, 4160, 32), (96, 64, 32)])
def test_gemv_thresh_ragged(N, K, g):
    case = wl.gemv_case(N, K, g, sparsity=0.5, seed=8)
    gg = GpuGemv(case.W, g)
    y, y32 = gg.thresh(case.x.to(DEV), case.t[0])
    _, y64, sa, _ = oracle_expect(case.W, g, case.x, case.t)
    check_y(y, y32, y64, sa, "thresh ragged")


@pytest.mark.parametrize("B", [1, 3, 4, 5, 6, 8, 12])
def test_gemv_exact_integer_case_bitwise(B):
    """Power-of-two scales and small-integer x: every partial sum on both sides
    is exact, so fp32 y equals the oracle's fp64 y and bf16 y matches bitwise
    (B = 3, 4: the CUDA-core batch kernel; B = 5, 6, 8, 12: the tensor-core
    kernel, whose products, row sums and fp32 sums are exact here too)."""
    rng = np.random.default_rng(80 + B)
    N, K, g = 2048, 1024, 64
    G = K // g
    q = rng.integers(0, 16, (N, K))
    q[:, 0::g], q[:, 1::g] = 0, 15
    s = 2.0 ** rng.integers(-3, 3, (N, G))
    z = rng.integers(0, 16, (N, G))
    W = torch.from_numpy((np.repeat(s, g, 1) * (q - np.repeat(z, g, 1))).astype(np.float16))
    x = torch.from_numpy(rng.integers(-8, 9, (B, K)).astype(np.float32)).to(torch.bfloat16)
    gg = GpuGemv(W, g, B)
    x_d = x.to(DEV)
    gg.select(x_d, [0.0] * B)
    y, y32 = gg.gemv(x_d)
    _, y64, _, yb = oracle_expect(W, g, x, [0.0] * B)
    assert np.array_equal(y32.cpu().double().numpy(), y64)
    assert np.array_equal(bits(y), yb)


@pytest.mark.parametrize("B", [1, 5, 12])
def test_gemv_power_of_two_scaling(B):
    case = wl.gemv_case(N=2048, K=4096, group=128, B=B, sparsity=0.5, seed=81, act="silu")
    g = GpuGemv(case.W, 128, B)
    x_d = case.x.to(DEV)
    g.select(x_d, case.t)
    _, y0 = g.gemv(x_d)
    _, _, sa, _ = oracle_expect(case.W, 128, case.x, case.t)
    for j in (-20, 7):
        x2 = (case.x.float() * 2.0 ** j).to(torch.bfloat16).to(DEV)
        g.select(x2, [t * 2.0 ** j for t in case.t])
        _, y2 = g.gemv(x2)
        err = np.abs(y2.cpu().double().numpy() * 2.0 ** -j - y0.cpu().double().numpy())
        assert np.all(err <= 2e-3 * sa)


def test_gemv_all_masked_gives_positive_zero():
    case = wl.gemv_case(**wl.TINY, sparsity=0.5, seed=9)
    g = GpuGemv(case.W, case.group)
    x_d = case.x.to(DEV)
    g.select(x_d, [float("inf")])
    assert int(g.count.item()) == 0
    y, y32 = g.gemv(x_d)             # y prefilled with NaN
    assert bits(y).max() == 0 and not torch.signbit(y32).any()
    assert (y32 == 0).all()
    assert g.workspace_is_zero()


@pytest.mark.parametrize("B", [5, 12, 16])
def test_gemv_batch_all_masked_gives_positive_zero(B):
    """The tensor-core kernel with no active channel: no run, no MMA; y = +0
    and the workspace stays zero."""
    case = wl.gemv_case(N=2048, K=1024, group=128, B=B, sparsity=0.5, seed=9)
    g = GpuGemv(case.W, 128, B)
    x_d = case.x.to(DEV)
    g.select(x_d, [float("inf")] * B)
    assert int(g.count.item()) == 0
    y, y32 = g.gemv(x_d)
    assert bits(y).max() == 0 and not torch.signbit(y32).any()
    assert (y32 == 0).all()
    assert g.workspace_is_zero()
    assert g.status.item() == 0


@pytest.mark.parametrize("N,K,g,B", [(96, 32, 32, 10), (992, 64, 32, 16), (1056, 128, 64, 9),
                                     (96, 64, 32, 5), (1056, 128, 64, 6)])
def test_gemv_batch_tiny_shapes(N, K, g, B):
    """The tensor-core kernel on one group, one partial tile, or a tile of
    1024 plus 32 outputs, dense and at 50% sparsity."""
    for sp in (0.0, 0.5):
        case = wl.gemv_case(N=N, K=K, group=g, B=B, sparsity=sp, seed=N + K + B)
        run_list_case(case, what=f"tiny N={N} K={K} g={g} B={B} sparsity={sp}")


def test_gemv_nan_channel_never_active():
    case = wl.gemv_case(**wl.TINY, sparsity=0.0, seed=12)
    x = case.x.clone()
    x[0, 17] = float("nan")
    g = GpuGemv(case.W, case.group)
    x_d = x.to(DEV)
    g.select(x_d, [-1.0])
    y, y32 = g.gemv(x_d)
    idx, y64, sa, _ = oracle_expect(case.W, case.group, x, [-1.0])
    assert 17 not in idx and np.array_equal(g.active(), idx)
    check_y(y, y32, y64, sa, "nan channel")


def test_gemv_bad_index_and_count_are_flagged_and_skipped():
    case = wl.gemv_case(**wl.TINY, sparsity=0.5, seed=13)
    g = GpuGemv(case.W, case.group)
    x_d = case.x.to(DEV)
    xb = bits(case.x)
    good = oracle.select(xb, case.t)
    bad = np.concatenate([good[:10], [case.K + 3], good[10:20], [-1], good[20:]]).astype(np.int32)
    idx = torch.from_numpy(bad).to(DEV)
    cnt = torch.tensor([bad.size], dtype=torch.int32, device=DEV)
    y, y32 = g.gemv(x_d, idx, cnt)
    q, s, z = oracle_codes(case.W, case.group)
    y64, sa, _ = oracle.gemv(q, s, z, case.group, xb, good)
    check_y(y, y32, y64, sa, "bad index")
    assert g.status.item() & sgq.SGQ_STATUS_BAD_INDEX
    g.status.zero_()
    full = torch.arange(case.K, dtype=torch.int32, device=DEV)
    cnt2 = torch.tensor([case.K + 5], dtype=torch.int32, device=DEV)
    y, y32 = g.gemv(x_d, full, cnt2)
    y64, sa, _ = oracle.gemv_dense(q, s, z, case.group, xb)
    check_y(y, y32, y64, sa, "bad count")
    assert g.status.item() & sgq.SGQ_STATUS_BAD_COUNT
    assert g.workspace_is_zero()


def test_gemv_repeated_calls_share_workspace():
    """The workspace returns to zero after every call, so consecutive calls of
    different shapes can share it."""
    big = wl.gemv_case(N=4096, K=4096, group=128, sparsity=0.5, seed=90)
    small = wl.gemv_case(N=1024, K=4096, group=128, sparsity=0.3, seed=91)
    gb, gs = GpuGemv(big.W, 128), GpuGemv(small.W, 128)
    gs.ws = gb.ws
    for _ in range(3):
        for c, gg in ((big, gb), (small, gs)):
            x_d = c.x.to(DEV)
            gg.select(x_d, c.t)
            y, y32 = gg.gemv(x_d)
            _, y64, sa, _ = oracle_expect(c.W, 128, c.x, c.t)
            check_y(y, y32, y64, sa, "shared ws")
    assert gb.workspace_is_zero()


# ---------------------------------------------------------------------------
# sgq_glu
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("B,I", [(1, 11008), (4, 25600), (1, 8)])
def test_glu_relu_bit_exact(B, I):
    gen = torch.Generator().manual_seed(B * I)
    gt = torch.randn(B, I, generator=gen).to(torch.bfloat16)
    up = torch.randn(B, I, generator=gen).to(torch.bfloat16)
    gt[0, :4] = torch.tensor([0.0, -0.0, float("inf"), -1.0]).to(torch.bfloat16)
    h = torch.empty_like(gt, device=DEV)
    sgq.sgq_glu(gt.to(DEV), up.to(DEV), h, B, I, sgq.SGQ_ACT_RELU)
    _, hb = oracle.glu(bits(gt), bits(up), 1)
    assert np.array_equal(bits(h), hb)


@pytest.mark.parametrize("B,I", [(1, 14336), (16, 25600)])
def test_glu_silu(B, I):
    gen = torch.Generator().manual_seed(B + I)
    gt = (torch.randn(B, I, generator=gen) * 3).to(torch.bfloat16)
    up = torch.randn(B, I, generator=gen).to(torch.bfloat16)
    h = torch.empty_like(gt, device=DEV)
    sgq.sgq_glu(gt.to(DEV), up.to(DEV), h, B, I, sgq.SGQ_ACT_SILU)
    h64, _ = oracle.glu(bits(gt), bits(up), 0)
    hv = bf16_values(bits(h))
    assert np.all(np.abs(hv - h64) <= (2.0 ** -8 + 1e-5) * np.abs(h64))


# ---------------------------------------------------------------------------
# FFN pipelines (select -> gate/up -> glu -> select -> down), end to end
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("act", ["relu", "silu"])
def test_ffn_pipeline_end_to_end(act):
    """Whole FFN on the GPU against the whole FFN in the oracle. The hidden
    vector is rounded to bf16 on both sides, so hidden values may differ by an
    ulp; the bound is one bf16 ulp (2^-7 relative) of the down projection's
    |W||h| plus the GEMV tolerance."""
    hid, inter, g = 1024, 2816, 128
    Wg, Wu, Wd = (wl.weight(inter, hid, 100), wl.weight(inter, hid, 101),
                  wl.weight(hid, inter, 102))
    x = wl.x_gaussian(1, hid, 103)
    t_in = [wl.percentile_threshold(x[0], 0.5)]
    a = sgq.SGQ_ACT_RELU if act == "relu" else sgq.SGQ_ACT_SILU
    # GPU
    gg, gu, gd = GpuGemv(Wg, g), GpuGemv(Wu, g), GpuGemv(Wd, g)
    x_d = x.to(DEV)
    gg.select(x_d, t_in)
    hg, _ = gg.gemv(x_d)
    hu, _ = gu.gemv(x_d, gg.idx, gg.count)
    h = torch.empty_like(hg)
    sgq.sgq_glu(hg, hu, h, 1, inter, a)
    # oracle (its own hidden vector and its own threshold for the down input)
    xb = bits(x)
    idx = oracle.select(xb, t_in)
    qg, sg, zg = oracle_codes(Wg, g)
    qu, su, zu = oracle_codes(Wu, g)
    qd, sd, zd = oracle_codes(Wd, g)
    _, _, gb = oracle.gemv(qg, sg, zg, g, xb, idx)
    _, _, ub = oracle.gemv(qu, su, zu, g, xb, idx)
    h64, hb = oracle.glu(gb, ub, 0 if act == "silu" else 1)
    t_h = [0.0]     # the nonzero hidden channels (ReLU zeros are skipped)
    gd.select(h, t_h)
    y, _ = gd.gemv(h)
    idx_h = oracle.select(hb, t_h)
    y64, sa, _ = oracle.gemv(qd, sd, zd, g, hb, idx_h)
    Wdq = (np.repeat(np.asarray(sd, np.uint16).view(np.float16).astype(np.float64), g, 1)
           * (qd - np.repeat(np.asarray(zd, np.uint16).view(np.float16).astype(np.float64), g, 1)))
    hv = bf16_values(hb)[0]
    spread = np.abs(Wdq) @ np.abs(hv)
    yv = bf16_values(bits(y))[0]
    tol = 1e-3 * sa[0] + 2.0 ** -7 * spread + 2.0 ** -8 * np.abs(y64[0])
    assert np.all(np.abs(yv - y64[0]) <= tol)


@pytest.mark.parametrize("B", [2, 5, 16])
def test_gemv_batch_bad_index_is_skipped(B):
    """Invalid list entries at B > 1 (every batch group reads the same rows):
    skipped for every row, flagged, and the workspace left zero. Per-row
    sparsity 0.9 keeps the union (1 - 0.9^B of K) short of K, so the two planted
    entries do not push the count past K (which would be clamped)."""
    case = wl.gemv_case(N=2048, K=4096, group=128, B=B, sparsity=0.9, seed=440)
    g = GpuGemv(case.W, case.group, B)
    x_d = case.x.to(DEV)
    xb = bits(case.x)
    good = oracle.select(xb, case.t)
    assert good.size + 2 <= case.K
    bad = np.concatenate([good[:7], [-5], good[7:300], [case.K], good[300:]]).astype(np.int32)
    idx = torch.from_numpy(bad).to(DEV)
    cnt = torch.tensor([bad.size], dtype=torch.int32, device=DEV)
    y, y32 = g.gemv(x_d, idx, cnt)
    q, s, z = oracle_codes(case.W, case.group)
    y64, sa, _ = oracle.gemv(q, s, z, case.group, xb, good)
    check_y(y, y32, y64, sa, f"batch {B} bad index")
    assert not (g.status.item() & sgq.SGQ_STATUS_BAD_COUNT)
    assert g.status.item() & sgq.SGQ_STATUS_BAD_INDEX
    assert g.workspace_is_zero()


def test_batch_kernel_wait_limit_sets_timeout_and_context_survives():
    """Fault injection from the host: the tensor-core kernel's issuer withholds
    the release of the last group run, so the waits on it run out (0.2 s);
    the status word carries SGQ_STATUS_TIMEOUT, the call returns, and the
    next ordinary call on the same context and workspace is correct."""
    B = 12
    case = wl.gemv_case(N=2048, K=2048, group=128, B=B, sparsity=0.5, seed=95)
    g = GpuGemv(case.W, 128, B)
    x_d = case.x.to(DEV)
    g.select(x_d, case.t)
    y, y32 = g.outputs(B)
    sgq.sgq_debug_gemv_withhold(g.qw, g.sz, g.N, g.K, 128, x_d, B, g.idx, g.count, y, y32,
                                g.ws, g.status)
    torch.cuda.synchronize()
    assert g.status.item() & sgq.SGQ_STATUS_TIMEOUT
    # the partial sums of the broken call are still in the workspace: clear it
    g.ws.zero_()
    g.status.zero_()
    y, y32 = g.gemv(x_d)
    idx, y64, sa, _ = oracle_expect(case.W, 128, case.x, case.t)
    torch.cuda.synchronize()
    check_y(y, y32, y64, sa, "after a timed-out call")
    assert g.status.item() == 0
    assert g.workspace_is_zero()
    with pytest.raises(sgq.SgqError):
        sgq.sgq_debug_gemv_withhold(g.qw, g.sz, g.N, g.K, 128, x_d, 4, g.idx, g.count, y, y32,
                                    g.ws, g.status)


def test_read_status_returns_and_clears_the_word():
    W = wl.weight(64, 128, 8)
    W[3, 9] = float("nan")
    _, _, st = gpu_pack(W, 64)
    assert sgq.sgq_read_status(st, clear=False) & sgq.SGQ_STATUS_NONFINITE_W
    assert sgq.sgq_read_status(st, clear=True) & sgq.SGQ_STATUS_NONFINITE_W
    assert sgq.sgq_read_status(st) == 0 and int(st.item()) == 0
