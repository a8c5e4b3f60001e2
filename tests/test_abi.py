"""The C ABI library loads, exports every symbol include/halo.h declares, and
rejects invalid arguments on the host before touching the GPU (no CUDA call is
made by any check in this file)."""
import ctypes
import os
import re
import subprocess

import pytest

from hadamard_rotated_precision_halo_b200 import build as halo_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "halo.h")

OK, NULL, SHAPE, BLOCK, ALIGN, DTYPE, WORKSPACE = 0, 1, 2, 3, 4, 5, 6

FAKE = 0x100000  # a 16-byte-aligned address that is never dereferenced by these calls
MISALIGNED = 0x100008


@pytest.fixture(scope="module")
def lib():
    path = halo_build.build()
    import hadamard_rotated_precision_halo_b200 as h

    return h.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(halo_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("halo_hadamard_quantize", "halo_qgemm", "halo_linear_fwd", "halo_linear_bwd",
                     "halo_workspace_size", "halo_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", halo_build.LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (halo_\w+)", out))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_binding_covers_every_export():
    import hadamard_rotated_precision_halo_b200 as h

    assert set(h.EXPORTS) == set(declared_functions())


def test_status_strings(lib):
    for s in range(10):
        assert lib.halo_status_string(s).decode().startswith("HALO")
    assert b"unknown" in lib.halo_status_string(99)


def test_workspace_size(lib):
    m, n, k = 1024, 512, 768
    fwd = lib.halo_workspace_size(m, n, k, 0)
    assert fwd >= m * k + n * k + 4 * (m + n)
    # zero padding of the contraction dimension: K = 700 needs codes for 768 (block 256)
    assert lib.halo_workspace_size(m, n, 700, 0) >= (m + n) * 768 + 4 * (m + n)
    bwd = lib.halo_workspace_size(m, n, k, 1)
    assert bwd >= 2 * m * n + n * k + m * k + 4 * (m + 2 * n + k)
    assert lib.halo_workspace_size(0, n, k, 0) == 0
    assert lib.halo_workspace_size(m, n, k, 7) == 0


def _hq(lib, x=FAKE, rows=256, cols=512, ld_x=512, axis=0, blk=128, qt=0, q=FAKE, ld_q=512, s=FAKE):
    return lib.halo_hadamard_quantize(x, rows, cols, ld_x, axis, blk, qt, q, ld_q, s, None)


def test_hadamard_quantize_host_validation(lib):
    assert _hq(lib, x=None) == NULL
    assert _hq(lib, s=None) == NULL
    assert _hq(lib, qt=5) == DTYPE
    assert _hq(lib, axis=3) == DTYPE
    assert _hq(lib, blk=64) == BLOCK
    assert _hq(lib, axis=1, blk=256) == BLOCK
    assert _hq(lib, cols=500, ld_x=512, ld_q=504) == SHAPE       # codes need the zero-padded length (512)
    assert _hq(lib, rows=0) == SHAPE
    assert _hq(lib, cols=65536, ld_x=65536, ld_q=65536) == SHAPE  # beyond the row-kernel limit
    assert _hq(lib, cols=32770, ld_x=32776, ld_q=32896) == SHAPE  # padded row beyond 32768
    assert _hq(lib, axis=1, cols=500, ld_x=504, ld_q=512) == SHAPE  # dim-0 rotation: cols % 8
    assert _hq(lib, ld_x=256) == SHAPE                            # ld < cols
    assert _hq(lib, x=MISALIGNED) == ALIGN
    assert _hq(lib, ld_x=516, ld_q=516) == ALIGN                  # bf16 row stride not 16 B


def _gemm(lib, a=FAKE, sa=FAKE, am=0, lda=256, b=FAKE, sb=FAKE, bm=0, ldb=256, m=128, n=128, k=256, qt=0,
          c=FAKE, ot=0, ldc=128):
    return lib.halo_qgemm(a, sa, am, lda, b, sb, bm, ldb, m, n, k, qt, c, ot, ldc, None)


def test_qgemm_host_validation(lib):
    assert _gemm(lib, a=None) == NULL
    assert _gemm(lib, c=None) == NULL
    assert _gemm(lib, qt=2) == DTYPE
    assert _gemm(lib, ot=2) == DTYPE
    assert _gemm(lib, am=2) == DTYPE
    assert _gemm(lib, m=0) == SHAPE
    assert _gemm(lib, k=200000, lda=200000, ldb=200000) == SHAPE  # int32 accumulator bound
    assert _gemm(lib, lda=128) == SHAPE
    assert _gemm(lib, lda=264, ldb=264) == ALIGN
    assert _gemm(lib, b=MISALIGNED) == ALIGN
    assert _gemm(lib, ot=1, n=100, ldc=100) == ALIGN  # 200-byte bf16 rows


def test_linear_host_validation(lib):
    ws = lib.halo_workspace_size(256, 256, 512, 0)
    f = lib.halo_linear_fwd
    assert f(None, FAKE, 256, 256, 512, 128, 0, FAKE, 0, FAKE, ws, None) == NULL
    assert f(FAKE, FAKE, 256, 256, 512, 64, 0, FAKE, 0, FAKE, ws, None) == BLOCK
    assert f(FAKE, FAKE, 256, 256, 500, 128, 0, FAKE, 0, FAKE, ws, None) == ALIGN     # 1000-byte rows of X
    assert f(FAKE, FAKE, 256, 256, 32776, 128, 0, FAKE, 0, FAKE, ws, None) == SHAPE   # K padded beyond 32768
    assert f(FAKE, FAKE, 256, 256, 520, 128, 0, FAKE, 0, FAKE, ws, None) == WORKSPACE  # K padded to 640
    assert f(FAKE, FAKE, 256, 256, 512, 128, 0, FAKE, 0, None, ws, None) == WORKSPACE
    assert f(FAKE, FAKE, 256, 256, 512, 128, 0, FAKE, 0, FAKE, ws - 1, None) == WORKSPACE
    assert f(FAKE, FAKE, 256, 256, 512, 128, 9, FAKE, 0, FAKE, ws, None) == DTYPE
    wsb = lib.halo_workspace_size(256, 256, 512, 1)
    b = lib.halo_linear_bwd
    assert b(FAKE, FAKE, FAKE, 256, 256, 512, 128, 0, None, 0, None, 0, FAKE, wsb, None) == NULL
    assert b(FAKE, None, FAKE, 256, 256, 512, 128, 0, None, 0, FAKE, 0, FAKE, wsb, None) == NULL  # dW needs X
    assert b(FAKE, FAKE, FAKE, 256, 256, 512, 256, 0, FAKE, 0, FAKE, 0, FAKE, wsb, None) == BLOCK
    assert b(FAKE, FAKE, FAKE, 256, 200, 512, 128, 0, None, 0, FAKE, 0, FAKE, wsb, None) == SHAPE  # dW: N % 16
    assert b(FAKE, FAKE, FAKE, 256, 300, 512, 128, 0, FAKE, 0, None, 0, FAKE, wsb, None) == WORKSPACE  # N pads to 384
    assert b(FAKE, FAKE, FAKE, 256, 256, 512, 128, 0, FAKE, 0, FAKE, 0, FAKE, wsb - 1, None) == WORKSPACE


def test_linear_fwd_noalloc_host_validation(lib):
    """Every argument check of the scratch-free forward runs before it looks up
    its device or the static array (here, with no GPU, that look-up would fail
    with a CUDA status instead)."""
    f = lib.halo_linear_fwd_noalloc
    assert f(None, FAKE, 256, 256, 512, 128, 0, FAKE, 0, None) == NULL
    assert f(FAKE, FAKE, 256, 256, 512, 64, 0, FAKE, 0, None) == BLOCK
    assert f(FAKE, FAKE, 256, 256, 512, 128, 9, FAKE, 0, None) == DTYPE
    assert f(FAKE, FAKE, 256, 256, 32776, 128, 0, FAKE, 0, None) == SHAPE
    assert f(MISALIGNED, FAKE, 256, 256, 512, 128, 0, FAKE, 0, None) == ALIGN
    assert f(FAKE, MISALIGNED, 256, 256, 512, 128, 0, FAKE, 0, None) == ALIGN
    assert f(FAKE, FAKE, 256, 256, 512, 128, 0, MISALIGNED, 0, None) == ALIGN
    assert f(FAKE, FAKE, 256, 6, 512, 128, 0, FAKE, 1, None) == ALIGN     # 12-byte bf16 output rows
    assert f(FAKE, FAKE, 256, 256, 500, 128, 0, FAKE, 0, None) == ALIGN   # 1000-byte rows of X
    assert f(FAKE, FAKE, 8192, 8192, 4096, 128, 0, FAKE, 0, None) == WORKSPACE  # beyond the static scratch


def test_split_dim0_host_validation(lib):
    c = lib.halo_hadamard_colmax
    assert c(None, 256, 64, 64, 128, FAKE, None) == NULL
    assert c(FAKE, 256, 64, 64, 128, None, None) == NULL
    assert c(FAKE, 256, 64, 64, 256, FAKE, None) == BLOCK       # dimension 0 takes 128-blocks only
    assert c(FAKE, 256, 60, 64, 128, FAKE, None) == SHAPE       # cols % 8
    assert c(FAKE, 256, 64, 60, 128, FAKE, None) == SHAPE       # ld_x < cols
    assert c(MISALIGNED, 256, 64, 64, 128, FAKE, None) == ALIGN
    assert c(FAKE, 256, 64, 64, 128, MISALIGNED, None) == ALIGN
    q = lib.halo_hadamard_quantize_colmax
    assert q(FAKE, 256, 64, 64, 128, 0, None, FAKE, 64, FAKE, None) == NULL
    assert q(FAKE, 256, 64, 64, 128, 0, FAKE, None, 64, FAKE, None) == NULL
    assert q(FAKE, 256, 64, 64, 128, 7, FAKE, FAKE, 64, FAKE, None) == DTYPE
    assert q(FAKE, 256, 64, 64, 128, 0, MISALIGNED, FAKE, 64, FAKE, None) == ALIGN
    assert q(FAKE, 256, 64, 64, 128, 0, FAKE, FAKE, 72, FAKE, None) == ALIGN  # ld_q % 16


def test_hadamard_quantize_ex_host_validation(lib):
    f = lib.halo_hadamard_quantize_ex
    # plain arguments are checked as for halo_hadamard_quantize
    assert f(None, 256, 512, 512, 0, 128, 0, None, None, 0, FAKE, 512, FAKE, None) == NULL
    assert f(FAKE, 256, 512, 512, 0, 64, 0, None, None, 0, FAKE, 512, FAKE, None) == BLOCK
    # signs and random bits: alignment and stride
    assert f(FAKE, 256, 512, 512, 0, 128, 0, MISALIGNED, None, 0, FAKE, 512, FAKE, None) == ALIGN
    assert f(FAKE, 256, 512, 512, 0, 128, 0, None, MISALIGNED, 512, FAKE, 512, FAKE, None) == ALIGN
    assert f(FAKE, 256, 512, 512, 0, 128, 0, None, FAKE, 500, FAKE, 512, FAKE, None) == SHAPE  # ld < cols
    assert f(FAKE, 256, 512, 512, 0, 128, 0, None, FAKE, 516, FAKE, 512, FAKE, None) == ALIGN  # 1032-byte rows


def test_hadamard_quantize_dual_host_validation(lib):
    f = lib.halo_hadamard_quantize_dual
    ok = (FAKE, 256, 512, 512, 128, FAKE, 512, FAKE, FAKE, 512, FAKE, None)
    def call(**kw):
        a = list(ok)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return f(*a)
    assert call(a0=None) == NULL
    assert call(a5=None) == NULL        # INT8 codes
    assert call(a10=None) == NULL       # E4M3 scales
    assert call(a4=64) == BLOCK
    assert call(a2=500, a3=512, a6=504) == SHAPE   # INT8 codes shorter than the padded row (512)
    assert call(a8=MISALIGNED) == ALIGN
    assert call(a9=520) == ALIGN        # E4M3 row stride not a multiple of 16


def test_grouped_host_validation(lib):
    q = lib.halo_hadamard_quantize_grouped
    assert q(FAKE, 256, 512, 512, 0, 128, 32, 0, FAKE, 512, FAKE, None) == BLOCK     # group not 64 / 128
    assert q(FAKE, 256, 512, 512, 0, 64, 64, 0, FAKE, 512, FAKE, None) == BLOCK      # rotation block
    assert q(None, 256, 512, 512, 0, 128, 64, 0, FAKE, 512, FAKE, None) == NULL
    assert q(FAKE, 256, 512, 512, 0, 128, 64, 0, FAKE, 504, FAKE, None) == SHAPE     # codes shorter than the row
    g = lib.halo_qgemm_grouped
    assert g(FAKE, FAKE, 0, 256, FAKE, FAKE, 0, 256, 128, 128, 256, 96, 0, FAKE, 0, 128, None) == BLOCK
    assert g(FAKE, FAKE, 0, 256, FAKE, FAKE, 0, 256, 128, 128, 192, 64, 0, FAKE, 0, 128, None) == SHAPE  # K % 128
    assert g(FAKE, None, 0, 256, FAKE, FAKE, 0, 256, 128, 128, 256, 64, 0, FAKE, 0, 128, None) == NULL
    assert lib.halo_workspace_size_grouped(256, 256, 512, 32, 0) == 0
    ws = lib.halo_workspace_size_grouped(256, 256, 512, 64, 0)
    assert ws >= 2 * 256 * 512 + 2 * 4 * 256 * 8
    f = lib.halo_linear_fwd_grouped
    assert f(FAKE, FAKE, 256, 256, 512, 128, 32, 0, FAKE, 0, FAKE, ws, None) == BLOCK
    assert f(FAKE, FAKE, 256, 256, 512, 128, 64, 0, FAKE, 0, FAKE, ws - 1, None) == WORKSPACE
    b = lib.halo_linear_bwd_grouped
    wsb = lib.halo_workspace_size_grouped(256, 256, 512, 64, 1)
    assert b(FAKE, FAKE, FAKE, 256, 256, 512, 128, 48, 0, FAKE, 0, FAKE, 0, FAKE, wsb, None) == BLOCK
    assert b(FAKE, FAKE, FAKE, 256, 256, 512, 128, 64, 0, FAKE, 0, FAKE, 0, FAKE, wsb - 1, None) == WORKSPACE


def test_selftest_wait_timeout_validation(lib):
    assert lib.halo_selftest_wait_timeout(0, None) == SHAPE
    assert lib.halo_selftest_wait_timeout(3_000_000_000, None) == SHAPE
