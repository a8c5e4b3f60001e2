"""Out-of-bounds write checks (in place of a memory sanitizer): every output is
a view into a larger buffer filled with a guard pattern -- guard rows above and
below, guard columns past each row -- and the guards must be untouched after
the call.  Shapes have ragged tails (rows, columns, zero padding) so that every
kernel's edge handling is exercised."""
import pytest
import torch

import hadamard_rotated_precision_halo_b200 as halo
from hadamard_rotated_precision_halo_b200 import inputs

pytestmark = pytest.mark.gpu

GUARD_U8 = 0xA5


def _guarded(rows, cols, dtype, extra_cols):
    """A [rows, cols] view with a row stride of cols + extra_cols elements inside
    a buffer with one guard row above and below."""
    ld = cols + extra_cols
    if dtype in (torch.int8, torch.uint8, torch.float8_e4m3fn):
        buf = torch.full((rows + 2, ld), GUARD_U8, dtype=torch.uint8, device="cuda")
        view = buf[1:rows + 1, :cols]
        if dtype != torch.uint8:
            view = view.view(dtype)
    else:
        buf = torch.full((rows + 2, ld), float("nan"), dtype=dtype, device="cuda")
        view = buf[1:rows + 1, :cols]
    return buf, view


def _check(buf, rows, cols):
    torch.cuda.synchronize()
    b = buf.view(torch.uint8) if buf.dtype != torch.uint8 else buf
    esz = buf.element_size()
    ref = torch.full_like(buf, GUARD_U8 if buf.dtype == torch.uint8 else float("nan")).view(torch.uint8)
    assert torch.equal(b[0], ref[0]), "guard row above written"
    assert torch.equal(b[rows + 1], ref[rows + 1]), "guard row below written"
    assert torch.equal(b[1:rows + 1, cols * esz:], ref[1:rows + 1, cols * esz:]), "guard columns written"


def _guarded_vec(n):
    buf = torch.full((n + 64,), float("nan"), dtype=torch.float32, device="cuda")
    return buf, buf[32:32 + n]


def _check_vec(buf, n):
    torch.cuda.synchronize()
    b = buf.view(torch.int32)
    nan = torch.full((32,), float("nan"), dtype=torch.float32, device="cuda").view(torch.int32)
    assert torch.equal(b[:32], nan) and torch.equal(b[32 + n:], nan), "scale guards written"


@pytest.mark.parametrize("qtype", [halo.HALO_Q_INT8, halo.HALO_Q_E4M3])
@pytest.mark.parametrize("axis,rows,cols,blk", [(halo.HALO_AXIS_COLS, 300, 1000, 128),
                                                (halo.HALO_AXIS_COLS, 37, 640, 256),
                                                (halo.HALO_AXIS_ROWS, 1000, 48, 128),
                                                (halo.HALO_AXIS_ROWS, 8320, 32, 128),
                                                (halo.HALO_AXIS_ROWS, 4096, 208, 128),
                                                (halo.HALO_AXIS_COLS, 700, 8192, 128),
                                                (halo.HALO_AXIS_COLS, 500, 28672, 128)])
def test_rotate_quantize_writes_only_its_outputs(qtype, axis, rows, cols, blk):
    x = inputs.activations(rows, cols, seed=rows + cols, device="cuda")
    qr, qc = halo.codes_shape(rows, cols, axis, blk)
    dt = torch.int8 if qtype == halo.HALO_Q_INT8 else torch.float8_e4m3fn
    qbuf, q = _guarded(qr, qc, dt, extra_cols=48)
    ns = rows if axis == halo.HALO_AXIS_COLS else cols
    sbuf, s = _guarded_vec(ns)
    halo.halo_hadamard_quantize(x, axis, blk, qtype, q_out=q, scales_out=s)
    _check(qbuf, qr, qc)
    _check_vec(sbuf, ns)


def test_dual_and_grouped_write_only_their_outputs():
    rows, cols = 300, 1000
    x = inputs.activations(rows, cols, seed=9, device="cuda")
    cp = halo.padded_length(cols, 128)
    b8, q8 = _guarded(rows, cp, torch.int8, 32)
    bf, qf = _guarded(rows, cp, torch.float8_e4m3fn, 16)
    s8b, s8 = _guarded_vec(rows)
    sfb, sf = _guarded_vec(rows)
    halo.halo_hadamard_quantize_dual(x, 128, q8, s8, qf, sf)
    _check(b8, rows, cp)
    _check(bf, rows, cp)
    _check_vec(s8b, rows)
    _check_vec(sfb, rows)
    bg, qg = _guarded(rows, cp, torch.int8, 32)
    sgb, sg = _guarded(rows, cp // 64, torch.float32, 0)  # group scales are dense
    halo.halo_hadamard_quantize_grouped(x, halo.HALO_AXIS_COLS, 128, 64, halo.HALO_Q_INT8, q_out=qg, scales_out=sg)
    _check(bg, rows, cp)
    _check(sgb, rows, cp // 64)
    xr = inputs.activations(1000, 48, seed=10, device="cuda")
    bc, qc = _guarded(1024, 48, torch.int8, 16)
    scb, sc = _guarded(1024 // 64, 48, torch.float32, 0)
    halo.halo_hadamard_quantize_grouped(xr, halo.HALO_AXIS_ROWS, 128, 64, halo.HALO_Q_INT8, q_out=qc, scales_out=sc)
    _check(bc, 1024, 48)
    _check(scb, 1024 // 64, 48)


@pytest.mark.parametrize("otype", [halo.HALO_OUT_FP32, halo.HALO_OUT_BF16])
@pytest.mark.parametrize("m,n,k", [(300, 520, 640), (16, 24, 256), (640, 272, 1024)])
def test_gemms_write_only_their_outputs(otype, m, n, k):
    g = torch.Generator(device="cuda").manual_seed(m + n)
    a = torch.randint(-127, 128, (m, k), device="cuda", generator=g, dtype=torch.int8)
    b = torch.randint(-127, 128, (n, k), device="cuda", generator=g, dtype=torch.int8)
    sa = torch.rand(m, device="cuda", generator=g)
    sb = torch.rand(n, device="cuda", generator=g)
    dt = torch.float32 if otype == halo.HALO_OUT_FP32 else torch.bfloat16
    cbuf, c = _guarded(m, n, dt, extra_cols=8)
    halo.halo_qgemm(a, sa, 0, b, sb, 0, m, n, k, halo.HALO_Q_INT8, otype, c=c)
    _check(cbuf, m, n)
    ga = torch.rand((m, k // 64), device="cuda", generator=g)
    gb = torch.rand((n, k // 64), device="cuda", generator=g)
    cbuf2, c2 = _guarded(m, n, dt, extra_cols=8)
    halo.halo_qgemm_grouped(a, ga, 0, b, gb, 0, m, n, k, 64, halo.HALO_Q_INT8, otype, c=c2)
    _check(cbuf2, m, n)


def test_linear_layers_write_only_their_outputs():
    m, n, k = 200, 144, 1008  # M, N and K all zero-padded somewhere (K % 16 and N % 16 for the backward)
    x = inputs.activations(m, k, seed=11, device="cuda")
    w = inputs.weights(n, k, seed=12, device="cuda")
    dy = inputs.grads(m, n + 8, seed=13, device="cuda")[:, :n].contiguous()
    # the linear layers write dense outputs: guard rows only
    ybuf, y = _guarded(m, n, torch.bfloat16, 0)
    halo.halo_linear_fwd(x, w, 128, halo.HALO_Q_INT8, halo.HALO_OUT_BF16, y=y)
    _check(ybuf, m, n)
    dxbuf, dx = _guarded(m, k, torch.bfloat16, 0)
    dwbuf, dw = _guarded(n, k, torch.float32, 0)
    halo.halo_linear_bwd(dy, x, w, 128, halo.HALO_Q_INT8, halo.HALO_OUT_BF16, halo.HALO_OUT_FP32, dx=dx, dw=dw)
    _check(dxbuf, m, k)
    _check(dwbuf, n, k)
