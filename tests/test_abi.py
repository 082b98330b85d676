"""The C ABI library: builds for sm_100a, loads, exports every entry point that
include/sgq.h declares, and rejects bad arguments on the host (no GPU needed:
none of these calls reaches a CUDA API)."""
import ctypes
import os
import re
import subprocess

import pytest

from activation_sparse_quantized_b200 import build as sgq_build
from activation_sparse_quantized_b200 import sgq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sgq.h")


@pytest.fixture(scope="module")
def lib():
    sgq_build.build()
    return sgq.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sgq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("sgq_pack", "sgq_select", "sgq_gemv", "sgq_gemv_dense", "sgq_glu",
                     "sgq_gemv_thresh", "sgq_packed_sizes", "sgq_gemv_workspace_bytes"):
        assert required in names
    assert set(names) == set(sgq.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", sgq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (sgq_\w+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_library_is_sm100a_only_and_standalone(lib):
    out = subprocess.run(["nm", "-D", sgq.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    assert "oracle" not in out          # shares nothing with the CPU oracle
    deps = subprocess.run(["ldd", sgq.LIB_PATH], capture_output=True, text=True).stdout
    assert "libtorch" not in deps and "libsgq_oracle" not in deps


def test_layout_version_and_strings(lib):
    assert sgq.sgq_layout_version() == 1
    for code in range(0, -10, -1):
        assert lib.sgq_status_string(code)
    assert b"unknown" in lib.sgq_status_string(-99)


def test_packed_sizes(lib):
    assert sgq.sgq_packed_sizes(4096, 14336, 128) == (14336 * 2048, 112 * 4096 * 4)
    assert sgq.sgq_packed_sizes(512, 256, 64) == (65536, 8192)
    with pytest.raises(sgq.SgqError):
        sgq.sgq_packed_sizes(4100, 14336, 128)      # N % 32
    with pytest.raises(sgq.SgqError):
        sgq.sgq_packed_sizes(4096, 14336, 96)       # group
    with pytest.raises(sgq.SgqError):
        sgq.sgq_packed_sizes(4096, 14300, 128)      # K % group


def test_host_argument_checks(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)          # never dereferenced: every call below fails its checks first
    odd = P((1 << 20) + 8)     # not 16-byte aligned
    f1 = (ctypes.c_float * 1)(0.5)
    assert lib.sgq_select(fake, 0, 256, f1, fake, fake, None) == -5          # batch
    assert lib.sgq_select(fake, 17, 256, f1, fake, fake, None) == -5
    assert lib.sgq_select(fake, 1, 250, f1, fake, fake, None) == -2          # K % 8
    assert lib.sgq_select(None, 1, 256, f1, fake, fake, None) == -1          # null
    assert lib.sgq_select(odd, 1, 256, f1, fake, fake, None) == -4           # align
    ws = lib.sgq_gemv_workspace_bytes(4096, 14336, 1)
    assert ws >= 4096 * 4 and ws % 256 == 0
    assert lib.sgq_gemv_workspace_bytes(4096, 14336, 0) == 0
    args = lambda **kw: [kw.get("qw", fake), kw.get("sz", fake), kw.get("N", 4096),
                         kw.get("K", 14336), kw.get("g", 128), kw.get("x", fake),
                         kw.get("B", 1), kw.get("idx", fake), kw.get("cnt", fake),
                         kw.get("y", fake), None, kw.get("ws", fake), kw.get("wsb", ws), None,
                         None]
    assert lib.sgq_gemv(*args(g=48)) == -3
    assert lib.sgq_gemv(*args(N=4016)) == -2
    assert lib.sgq_gemv(*args(B=0)) == -5
    assert lib.sgq_gemv(*args(B=17)) == -5
    assert lib.sgq_gemv(*args(idx=None)) == -1
    assert lib.sgq_gemv(*args(y=odd)) == -4
    assert lib.sgq_gemv(*args(wsb=ws - 1)) == -6
    # the wait-limit test hook runs only on the tensor-core batch sizes
    wsb = lib.sgq_gemv_workspace_bytes(4096, 14336, 12)
    assert lib.sgq_debug_gemv_withhold(*args(B=4)) == -2
    assert lib.sgq_debug_gemv_withhold(*args(B=17)) == -2
    assert lib.sgq_debug_gemv_withhold(*args(B=12, idx=None, wsb=wsb)) == -1
    assert lib.sgq_debug_gemv_withhold(*args(B=12, wsb=wsb - 1)) == -6
    assert lib.sgq_glu(fake, fake, fake, 1, 12, 0, None) == -2               # not % 8
    assert lib.sgq_glu(fake, fake, fake, 1, 16, 5, None) == -7               # activation
    assert lib.sgq_pack(fake, 4096, 14336, 100, fake, fake, None, None) == -3
    # fused gate + up + GLU: stacked width 2I, act checked first
    wsg = lib.sgq_gemv_workspace_bytes(2 * 14336, 4096, 1)
    glu = lambda **kw: [fake, fake, kw.get("I", 14336), 4096, 128, fake, kw.get("B", 1), fake,
                        fake, kw.get("act", 0), fake, None, fake, kw.get("wsb", wsg), None, None]
    assert lib.sgq_gemv_glu(*glu(act=2)) == -7
    assert lib.sgq_gemv_glu(*glu(I=14344)) == -2                # 2I % 32
    assert lib.sgq_gemv_glu(*glu(I=0)) == -2
    assert lib.sgq_gemv_glu(*glu(B=17)) == -5
    assert lib.sgq_gemv_glu(*glu(wsb=lib.sgq_gemv_workspace_bytes(14336, 4096, 1))) == -6
    F = ctypes.c_float
    assert lib.sgq_gemv_glu_thresh(fake, fake, 14336, 4096, 128, fake, F(0.5), 7, fake, None,
                                   fake, wsg, None, None) == -7
    assert lib.sgq_gemv_glu_dense(fake, fake, 14336, 4096, 96, fake, 1, 0, fake, None, fake,
                                  wsg, None, None) == -3
    assert lib.sgq_read_status(None, None, 0, None) == -1
    # 2:4 layout: N % 64, null keep, sizes
    assert lib.sgq_pack_nm(fake, 4064, 14336, 128, fake, fake, fake, None, None) == -2
    assert lib.sgq_gemv_nm(fake, None, fake, 4096, 14336, 128, fake, fake, fake, fake, None,
                           fake, ws, None, None) == -1
    assert lib.sgq_gemv_nm_thresh(fake, fake, fake, 4000, 14336, 128, fake, F(0.5), fake, None,
                                  fake, ws, None, None) == -2
    assert sgq.sgq_packed_sizes_nm(4096, 14336, 128) == (14336 * 1024, 112 * 512, 112 * 2048 * 4)


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="no CPU fallback|there is no CPU fallback"):
        sgq.load(str(tmp_path / "libsgq.so"))
