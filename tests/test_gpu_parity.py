"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on seeded inputs.

Small cases span several tiles and ragged tails and are compared element by
element; the full Llama-shaped cases run in the benchmark's launch
configuration and are compared on sampled rows / columns that the oracle
computes one by one (each row or column of a rotated-quantised operand depends
on that row or column alone).
"""
import numpy as np
import pytest
import torch

import hadamard_rotated_precision_halo_b200 as halo
import oracle
from hadamard_rotated_precision_halo_b200 import inputs
from tests._parity import check_codes, check_codes_stochastic, check_output, oracle_operand

pytestmark = pytest.mark.gpu

INT8, E4M3 = halo.HALO_Q_INT8, halo.HALO_Q_E4M3
FP32, BF16 = halo.HALO_OUT_FP32, halo.HALO_OUT_BF16
COLS, ROWS = halo.HALO_AXIS_COLS, halo.HALO_AXIS_ROWS


@pytest.fixture(autouse=True)
def no_device_error():
    yield
    st, site = halo.halo_device_error()
    assert st == halo.HALO_OK, f"kernel bounded wait ran out at site {site:#x}"


def _cuda(t):
    return t.to("cuda")


# ------------------------------------------------------------------ rotate + quantise
@pytest.mark.parametrize("qtype", [INT8, E4M3])
@pytest.mark.parametrize("rows,cols,blk", [(300, 640, 128), (130, 512, 256), (1, 128, 128), (64, 256, 256),
                                           (37, 11008, 128), (5, 28672, 128),
                                           # rows per row group >= 3 (stage refills), codes in the consumed stage
                                           (2000, 8192, 128), (600, 24576, 128),
                                           # rows split over two-CTA clusters, >= 3 rows per cluster
                                           (700, 28672, 128), (2, 25600, 128),
                                           # row groups of 4, 5 (code tiles) and 6 warps (codes in the stage)
                                           (4, 16384, 128), (3, 20480, 128), (3, 24576, 128)])
def test_rotq_rows_parity(qtype, rows, cols, blk):
    x = inputs.activations(rows, cols, seed=rows * 7 + cols, device="cpu")
    x[min(3, rows - 1)] = 0  # an all-zero row: scale 0, codes 0
    q, s = halo.halo_hadamard_quantize(_cuda(x), COLS, blk, qtype)
    torch.cuda.synchronize()
    codes, scales, t = oracle_operand(x, 1, blk, qtype)
    check_codes(q, s, codes, scales, t, qtype, blk=blk, axis=1)


@pytest.mark.parametrize("qtype", [INT8, E4M3])
@pytest.mark.parametrize("rows,cols", [(1024, 208), (384, 96), (2048, 64), (128, 16), (4096, 48), (1152, 48),
                                       (8320, 32), (28672, 64),
                                       # clusters of 16 CTAs (128 and 256 blocks of 128 rows)
                                       (16384, 96), (32768, 64),
                                       # several strips per cluster: every reused buffer goes round
                                       (4096, 8192), (16384, 1056), (28672, 1024)])
def test_rotq_cols_parity(qtype, rows, cols):
    x = inputs.activations(rows, cols, seed=rows + 3 * cols, device="cpu")
    x[:, min(5, cols - 1)] = 0  # an all-zero column
    q, s = halo.halo_hadamard_quantize(_cuda(x), ROWS, 128, qtype)
    torch.cuda.synchronize()
    codes, scales, t = oracle_operand(x, 0, 128, qtype)
    check_codes(q, s, codes, scales, t, qtype, blk=128, axis=0)


def test_rotq_rows_strided_input():
    base = inputs.activations(96, 768, seed=11, device="cpu")
    x = base[:, :512]  # row stride 768 elements
    xd = _cuda(base)[:, :512]
    q, s = halo.halo_hadamard_quantize(xd, COLS, 128, INT8)
    torch.cuda.synchronize()
    codes, scales, t = oracle_operand(x.contiguous(), 1, 128, INT8)
    check_codes(q, s, codes, scales, t, INT8, blk=128, axis=1)


# ------------------------------------------------------------------------------ GEMM
def _rand_codes(rows, cols, qtype, seed):
    g = torch.Generator().manual_seed(seed)
    if qtype == INT8:
        return torch.randint(-127, 128, (rows, cols), generator=g, dtype=torch.int8)
    b = torch.randint(0, 256, (rows, cols), generator=g, dtype=torch.int16).to(torch.uint8)
    b[(b & 0x7F) == 0x7F] = 0x38  # no NaN codes
    return b.view(torch.float8_e4m3fn)


def _stored(codes_logical: torch.Tensor, major: int) -> torch.Tensor:
    """Storage of a logical [rows, K] operand: K-major as is, MN-major transposed."""
    return codes_logical if major == halo.HALO_MAJOR_K else codes_logical.t().contiguous()


@pytest.mark.parametrize("a_major,b_major", [(0, 0), (1, 1), (0, 1), (1, 0)])
@pytest.mark.parametrize("m,n,k", [(300, 520, 640), (128, 256, 128), (16, 16, 208), (640, 272, 1024)])
def test_qgemm_int8_bit_exact(a_major, b_major, m, n, k):
    if a_major == 1 and m % 16 or b_major == 1 and n % 16:
        pytest.skip("MN-major storage needs a 16-byte row stride")
    a = _rand_codes(m, k, INT8, seed=m + k)
    b = _rand_codes(n, k, INT8, seed=n * 3 + k)
    ones_m = torch.ones(m, dtype=torch.float32, device="cuda")
    ones_n = torch.ones(n, dtype=torch.float32, device="cuda")
    c = halo.halo_qgemm(_cuda(_stored(a, a_major)), ones_m, a_major, _cuda(_stored(b, b_major)), ones_n, b_major,
                        m, n, k, INT8, FP32)
    torch.cuda.synchronize()
    acc = oracle.gemm_i8(a.numpy(), b.numpy())
    # with unit scales the output is exactly float32(acc): bit-exact int32 accumulation
    np.testing.assert_array_equal(c.cpu().numpy(), acc.astype(np.float32))


@pytest.mark.parametrize("qtype", [INT8, E4M3])
@pytest.mark.parametrize("a_major,b_major", [(0, 0), (1, 1), (0, 1)])
def test_qgemm_long_k_two_passes_sampled(qtype, a_major, b_major):
    """2048 x 4096 x 16384: 128 tiles of 256 x 256 over 74 SM pairs, so the
    second pass over the grid walks K backwards (K >= 16384).  INT8 with unit
    scales must still equal float32 of the exact integer sum; E4M3 within fp32
    accumulation.  Sampled rows (both passes) and columns."""
    m, n, k = 2048, 4096, 16384
    a = _rand_codes(m, k, qtype, seed=81)
    b = _rand_codes(n, k, qtype, seed=82)
    ones_m = torch.ones(m, dtype=torch.float32, device="cuda")
    ones_n = torch.ones(n, dtype=torch.float32, device="cuda")
    c = halo.halo_qgemm(_cuda(_stored(a, a_major)), ones_m, a_major, _cuda(_stored(b, b_major)), ones_n, b_major,
                        m, n, k, qtype, FP32)
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(83)
    rows = torch.cat([torch.tensor([0, 255, 256, m - 1]), torch.randint(0, m, (28,), generator=g)])
    cols = torch.cat([torch.tensor([0, 255, 256, n - 1]), torch.randint(0, n, (28,), generator=g)])
    got = c.cpu()[rows][:, cols].numpy()
    if qtype == INT8:
        acc = oracle.gemm_i8(a[rows].numpy(), b[cols].numpy())
        np.testing.assert_array_equal(got, acc.astype(np.float32))
    else:
        ref = oracle.gemm_e4m3(a[rows].view(torch.uint8).numpy(), b[cols].view(torch.uint8).numpy())
        err = np.abs(got.astype(np.float64) - ref).max() / np.abs(ref).max()
        assert err < 1e-5, err
    st, site = halo.halo_device_error()
    assert st == halo.HALO_OK, f"bounded wait ran out at site {site:#x}"


@pytest.mark.parametrize("a_major,b_major", [(0, 0), (1, 1)])
@pytest.mark.parametrize("otype", [FP32, BF16])
def test_qgemm_e4m3_with_scales(a_major, b_major, otype):
    m, n, k = 272, 528, 768
    a = _rand_codes(m, k, E4M3, seed=5)
    b = _rand_codes(n, k, E4M3, seed=6)
    g = torch.Generator().manual_seed(7)
    sa = torch.rand(m, generator=g) + 0.5
    sb = torch.rand(n, generator=g) * 1e-3 + 1e-4
    c = halo.halo_qgemm(_cuda(_stored(a, a_major)), _cuda(sa), a_major, _cuda(_stored(b, b_major)), _cuda(sb),
                        b_major, m, n, k, E4M3, otype)
    torch.cuda.synchronize()
    ref = oracle.dequant(oracle.gemm_e4m3(a.view(torch.uint8).numpy(), b.view(torch.uint8).numpy()), sa.numpy(),
                         sb.numpy())
    err = check_output(c, ref)
    if otype == FP32:
        assert err < 1e-5  # fp32 accumulation of exact E4M3 products


def test_qgemm_int8_scales_epilogue():
    m, n, k = 256, 512, 512
    a = _rand_codes(m, k, INT8, seed=1)
    b = _rand_codes(n, k, INT8, seed=2)
    g = torch.Generator().manual_seed(3)
    sa = torch.rand(m, generator=g) * 0.01
    sb = torch.rand(n, generator=g) * 0.01
    c = halo.halo_qgemm(_cuda(a), _cuda(sa), 0, _cuda(b), _cuda(sb), 0, m, n, k, INT8, FP32)
    torch.cuda.synchronize()
    ref = oracle.dequant(oracle.gemm_i8(a.numpy(), b.numpy()).astype(np.float64), sa.numpy(), sb.numpy())
    err = check_output(c, ref)
    assert err < 1e-6


# ---------------------------------------------------------------------- linear layer
def test_linear_fwd_tiny_config():
    """X[64,256], W[128,256] ~ N(0,1), seed 0; one 256-block on K; INT8; Y fp32."""
    x = inputs.plain(64, 256, seed=0, device="cpu")
    w = inputs.plain(128, 256, seed=1, device="cpu")
    y = halo.halo_linear_fwd(_cuda(x), _cuda(w), 256, INT8, FP32)
    qx, sx = halo.halo_hadamard_quantize(_cuda(x), COLS, 256, INT8)
    qw, sw = halo.halo_hadamard_quantize(_cuda(w), COLS, 256, INT8)
    torch.cuda.synchronize()
    cx, osx, tx = oracle_operand(x, 1, 256, INT8)
    cw, osw, tw = oracle_operand(w, 1, 256, INT8)
    check_codes(qx, sx, cx, osx, tx, INT8, blk=256, axis=1)
    check_codes(qw, sw, cw, osw, tw, INT8, blk=256, axis=1)
    ref = oracle.linear_fwd(x, w, 256, INT8)
    check_output(y, ref)


@pytest.mark.parametrize("qtype", [INT8, E4M3])
@pytest.mark.parametrize("otype", [FP32, BF16])
def test_linear_fwd_parity(qtype, otype):
    m, n, k = 384, 320, 640
    x = inputs.activations(m, k, seed=21, device="cpu")
    w = inputs.weights(n, k, seed=22, device="cpu")
    y = halo.halo_linear_fwd(_cuda(x), _cuda(w), 128, qtype, otype)
    torch.cuda.synchronize()
    check_output(y, oracle.linear_fwd(x, w, 128, qtype))


@pytest.mark.parametrize("qtype", [INT8, E4M3])
def test_linear_bwd_parity(qtype):
    m, n, k = 512, 384, 640
    dy = inputs.grads(m, n, seed=31, device="cpu")
    x = inputs.activations(m, k, seed=32, device="cpu")
    w = inputs.weights(n, k, seed=33, device="cpu")
    dx, dw = halo.halo_linear_bwd(_cuda(dy), _cuda(x), _cuda(w), 128, qtype, BF16, FP32)
    torch.cuda.synchronize()
    check_output(dx, oracle.linear_bwd_dx(dy, w, 128, qtype))
    check_output(dw, oracle.linear_bwd_dw(dy, x, 128, qtype))


def test_linear_bwd_single_products():
    m, n, k = 256, 256, 384
    dy = inputs.grads(m, n, seed=41, device="cpu")
    x = inputs.activations(m, k, seed=42, device="cpu")
    w = inputs.weights(n, k, seed=43, device="cpu")
    dx, _ = halo.halo_linear_bwd(_cuda(dy), None, _cuda(w), 128, INT8, FP32, FP32, want_dw=False)
    _, dw = halo.halo_linear_bwd(_cuda(dy), _cuda(x), None, 128, INT8, FP32, FP32, want_dx=False)
    torch.cuda.synchronize()
    check_output(dx, oracle.linear_bwd_dx(dy, w, 128, INT8))
    check_output(dw, oracle.linear_bwd_dw(dy, x, 128, INT8))


# --------------------------------------------------------------- full Llama-shaped cases
def _sampled_gemm_ref(a_rows_bf16, a_along, b_rows_bf16, b_along, blk, qtype):
    """Oracle values C[i, j] for a sample of A's and B's logical rows.

    a_rows_bf16: the sampled part of A's storage -- rows of A when a_along == 1
    (rotate along its contiguous dim), columns of A^T's storage (as a [K, r]
    matrix) when a_along == 0.  Same for B."""
    ca, sa, _ = oracle_operand(a_rows_bf16, a_along, blk, qtype)
    cb, sb, _ = oracle_operand(b_rows_bf16, b_along, blk, qtype)
    if a_along == 0:
        ca = np.ascontiguousarray(ca.T)
    if b_along == 0:
        cb = np.ascontiguousarray(cb.T)
    acc = oracle.gemm_i8(ca, cb).astype(np.float64) if qtype == INT8 else oracle.gemm_e4m3(ca, cb)
    return oracle.dequant(acc, sa, sb)


def _sample(n, count, seed):
    g = np.random.default_rng(seed)
    idx = np.sort(g.choice(n, size=min(count, n), replace=False))
    idx[-1] = n - 1  # always include the last (ragged-tail) index
    return idx


@pytest.mark.parametrize("qtype", [INT8, E4M3])
def test_full_rotate_quantize_16384x4096(qtype):
    x = inputs.activations(16384, 4096, seed=1, device="cuda")
    q, s = halo.halo_hadamard_quantize(x, COLS, 128, qtype)
    torch.cuda.synchronize()
    rows = _sample(16384, 256, 1)
    xs = x[torch.from_numpy(rows).cuda()].cpu()
    codes, scales, t = oracle_operand(xs, 1, 128, qtype)
    sel = torch.from_numpy(rows).cuda()
    check_codes(q[sel], s[sel], codes, scales, t, qtype, blk=128, axis=1)


@pytest.mark.parametrize("qtype", [INT8, E4M3])
def test_full_forward_8192x4096x4096(qtype):
    m, n, k = 8192, 4096, 4096
    x = inputs.activations(m, k, seed=2, device="cuda")
    w = inputs.weights(n, k, seed=3, device="cuda")
    y = halo.halo_linear_fwd(x, w, 128, qtype, BF16)
    torch.cuda.synchronize()
    ri, ci = _sample(m, 48, 4), _sample(n, 64, 5)
    ref = _sampled_gemm_ref(x[torch.from_numpy(ri).cuda()].cpu(), 1, w[torch.from_numpy(ci).cuda()].cpu(), 1, 128,
                            qtype)
    check_output(y[torch.from_numpy(ri).cuda()][:, torch.from_numpy(ci).cuda()], ref)


def test_full_backward_8192x11008x4096():
    m, n, k = 8192, 4096, 11008
    dy = inputs.grads(m, n, seed=5, device="cuda")
    w = inputs.weights(n, k, seed=6, device="cuda")
    x = inputs.activations(m, k, seed=7, device="cuda")
    dx, dw = halo.halo_linear_bwd(dy, x, w, 128, INT8, BF16, FP32)
    torch.cuda.synchronize()
    # dX[M, K] = dY W: A rows = dY rows (rotated along N), B rows = W columns (rotated along dim 0 of W)
    ri, ci = _sample(m, 32, 8), _sample(k, 48, 9)
    ri_t, ci_t = torch.from_numpy(ri).cuda(), torch.from_numpy(ci).cuda()
    ref = _sampled_gemm_ref(dy[ri_t].cpu(), 1, w[:, ci_t].cpu(), 0, 128, INT8)
    check_output(dx[ri_t][:, ci_t], ref)
    # dW[N, K] = dY^T X: A rows = dY columns, B rows = X columns, both rotated along M
    ni, ki = _sample(n, 32, 10), _sample(k, 48, 11)
    ni_t, ki_t = torch.from_numpy(ni).cuda(), torch.from_numpy(ki).cuda()
    ref = _sampled_gemm_ref(dy[:, ni_t].cpu(), 0, x[:, ki_t].cpu(), 0, 128, INT8)
    check_output(dw[ni_t][:, ki_t], ref)


@pytest.mark.parametrize("qtype", [INT8, E4M3])
def test_full_llama70b_layer_step_as_benchmarked(qtype):
    """The Llama-70B layer step (4096 tokens; q, k, v, o, gate, up, down; forward,
    dX and dW) run exactly as bench.py times it -- the same launches, with the
    attention and MLP inputs rotated once and shared -- and every one of the 21
    outputs checked on sampled rows x columns against the oracle."""
    import bench

    step = bench.LayerStep(inputs.LLAMA70B_LAYER, seed=4, device=torch.device("cuda"), qtype=qtype)
    step.run()
    torch.cuda.synchronize()
    for gi, (kind, name, a, a_axis, b, b_axis, m, n, k, c) in enumerate(step.gemms()):
        ri, cj = _sample(m, 8, 100 + gi), _sample(n, 16, 200 + gi)
        ri_t, cj_t = torch.from_numpy(ri).cuda(), torch.from_numpy(cj).cuda()
        # logical rows of A (B) are rows of its storage when rotated along the
        # contiguous dim, columns of its storage when rotated along dim 0
        a_s = a[ri_t] if a_axis == COLS else a[:, ri_t]
        b_s = b[cj_t] if b_axis == COLS else b[:, cj_t]
        ref = _sampled_gemm_ref(a_s.cpu(), 1 if a_axis == COLS else 0, b_s.cpu(), 1 if b_axis == COLS else 0, 128,
                                qtype)
        check_output(c[ri_t][:, cj_t], ref)
    del step
    torch.cuda.empty_cache()


# --------------------------------------------------------------------- variants
def _signs_t(n, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randint(0, 2, (n,), generator=g, dtype=torch.int8) * 2 - 1).to(torch.int8)


def _rand_bits(rows, cols, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(0, 65536, (rows, cols), generator=g, dtype=torch.int32).to(torch.uint16)


@pytest.mark.parametrize("qtype", [INT8, E4M3])
@pytest.mark.parametrize("axis,rows,cols,blk", [(COLS, 300, 640, 128), (COLS, 64, 512, 256), (COLS, 7, 11008, 128),
                                                (ROWS, 1024, 208, 128), (ROWS, 8320, 32, 128)])
def test_random_sign_rotation_parity(qtype, axis, rows, cols, blk):
    x = inputs.activations(rows, cols, seed=rows + cols + 5, device="cpu")
    s = _signs_t(cols if axis == COLS else rows, seed=rows)
    q, sc = halo.halo_hadamard_quantize_ex(_cuda(x), axis, blk, qtype, signs=_cuda(s))
    torch.cuda.synchronize()
    v = oracle.rotate_signed(x, blk, 1 if axis == COLS else 0, s.numpy())
    codes, scales, t = oracle.quantize(v, axis=0 if axis == COLS else 1, qtype=qtype)
    check_codes(q, sc, codes, scales, t, qtype, blk=blk, axis=1 if axis == COLS else 0)


@pytest.mark.parametrize("qtype", [INT8, E4M3])
@pytest.mark.parametrize("axis,rows,cols,blk", [(COLS, 300, 640, 128), (COLS, 64, 512, 256), (ROWS, 1024, 208, 128),
                                                (ROWS, 8320, 32, 128)])
def test_stochastic_rounding_parity(qtype, axis, rows, cols, blk):
    x = inputs.activations(rows, cols, seed=rows * 3 + cols, device="cpu")
    rb = _rand_bits(rows, cols, seed=cols)
    q, sc = halo.halo_hadamard_quantize_ex(_cuda(x), axis, blk, qtype, rand_bits=_cuda(rb))
    torch.cuda.synchronize()
    v = oracle.rotate(x, blk, 1 if axis == COLS else 0)
    codes, scales, t = oracle.quantize_stochastic(v, 0 if axis == COLS else 1, qtype, rb.numpy())
    from tests._parity import check_codes_stochastic

    n_ex, n_diff = check_codes_stochastic(q, sc, codes, scales, t, rb.numpy(), qtype, blk=blk,
                                          axis=1 if axis == COLS else 0)
    assert n_ex < 0.01 * x.numel()


def test_signs_and_stochastic_rounding_together_and_strided_random_bits():
    rows, cols = 256, 1024
    x = inputs.activations(rows, cols, seed=77, device="cpu")
    s = _signs_t(cols, seed=78)
    rb_full = _rand_bits(rows, cols + 64, seed=79)  # row stride cols + 64
    rb = rb_full[:, :cols]
    q, sc = halo.halo_hadamard_quantize_ex(_cuda(x), COLS, 128, INT8, signs=_cuda(s), rand_bits=_cuda(rb_full)[:, :cols])
    torch.cuda.synchronize()
    v = oracle.rotate_signed(x, 128, 1, s.numpy())
    codes, scales, t = oracle.quantize_stochastic(v, 0, INT8, rb.contiguous().numpy())
    from tests._parity import check_codes_stochastic

    check_codes_stochastic(q, sc, codes, scales, t, rb.contiguous().numpy(), INT8, blk=128, axis=1)


def test_random_sign_gemm_keeps_the_product():
    """Both operands rotated with the same signs along K: the quantised GEMM
    matches the oracle's signed-rotation GEMM, and stays close to X W^T."""
    m, n, k = 384, 320, 640
    x = inputs.activations(m, k, seed=81, device="cpu")
    w = inputs.weights(n, k, seed=82, device="cpu")
    s = _signs_t(k, seed=83)
    qx, sx = halo.halo_hadamard_quantize_ex(_cuda(x), COLS, 128, INT8, signs=_cuda(s))
    qw, sw = halo.halo_hadamard_quantize_ex(_cuda(w), COLS, 128, INT8, signs=_cuda(s))
    y = halo.halo_qgemm(qx, sx, 0, qw, sw, 0, m, n, k, INT8, FP32)
    torch.cuda.synchronize()
    cx, osx, _ = oracle.quantize(oracle.rotate_signed(x, 128, 1, s.numpy()), 0, INT8)
    cw, osw, _ = oracle.quantize(oracle.rotate_signed(w, 128, 1, s.numpy()), 0, INT8)
    ref = oracle.dequant(oracle.gemm_i8(cx, cw).astype(np.float64), osx, osw)
    check_output(y, ref)
    exact = x.double().numpy() @ w.double().numpy().T
    assert np.max(np.abs(ref - exact)) < 0.05 * np.max(np.abs(exact))


# ------------------------------------------------------------- dual INT8 + E4M3 output
@pytest.mark.parametrize("rows,cols,blk", [(300, 640, 128), (130, 512, 256), (3, 28672, 128)])
def test_rotq_dual_parity(rows, cols, blk):
    x = inputs.activations(rows, cols, seed=rows + cols, device="cpu")
    x[min(2, rows - 1)] = 0
    xd = _cuda(x)
    q8, s8, qf, sf = halo.halo_hadamard_quantize_dual(xd, blk)
    torch.cuda.synchronize()
    for q, s, qt in ((q8, s8, INT8), (qf, sf, E4M3)):
        codes, scales, t = oracle_operand(x, 1, blk, qt)
        check_codes(q, s, codes, scales, t, qt, blk=blk, axis=1)
        # byte for byte what the single-output call writes
        q1, s1 = halo.halo_hadamard_quantize(xd, COLS, blk, qt)
        torch.cuda.synchronize()
        assert torch.equal(q1.view(torch.uint8), q.view(torch.uint8)) and torch.equal(s1, s)


def test_rotq_dual_full_size_16384x4096():
    """The standalone rotate+quantise workload, both encodings from one read,
    checked on sampled rows (each row depends on that row alone)."""
    x = inputs.activations(16384, 4096, seed=2, device="cuda")
    q8, s8, qf, sf = halo.halo_hadamard_quantize_dual(x, 128)
    torch.cuda.synchronize()
    rows = torch.from_numpy(_sample(16384, 256, 5)).cuda()
    xs = x[rows].cpu()
    for q, s, qt in ((q8, s8, INT8), (qf, sf, E4M3)):
        codes, scales, t = oracle_operand(xs, 1, 128, qt)
        check_codes(q[rows], s[rows], codes, scales, t, qt, blk=128, axis=1)


# ------------------------------------------------------------ zero padding (ragged lengths)
@pytest.mark.parametrize("qtype", [INT8, E4M3])
@pytest.mark.parametrize("rows,cols,blk", [(37, 1000, 128), (5, 296, 256), (9, 72, 128), (3, 200, 256),
                                           (4, 32760, 128), (6, 384, 256), (3, 24504, 128), (300, 20000, 128),
                                           (2000, 8000, 128)])
def test_rotq_rows_padded_parity(qtype, rows, cols, blk):
    """Row length not a multiple of blk: the partial chunk arrives by its own
    TMA box (zeros past the row), whole padding chunks are zeros; the codes
    cover the padded length."""
    x = inputs.activations(rows, cols, seed=rows * 3 + cols, device="cpu")
    q, s = halo.halo_hadamard_quantize(_cuda(x), COLS, blk, qtype)
    torch.cuda.synchronize()
    assert tuple(q.shape) == (rows, halo.padded_length(cols, blk))
    codes, scales, t = oracle_operand(x, 1, blk, qtype)
    check_codes(q, s, codes, scales, t, qtype, blk=blk, axis=1)


@pytest.mark.parametrize("qtype", [INT8, E4M3])
@pytest.mark.parametrize("rows,cols", [(1000, 48), (200, 64), (70, 32), (130, 80), (8300, 16), (28700, 16)])
def test_rotq_cols_padded_parity(qtype, rows, cols):
    """Column length not a multiple of 128 (one-pass and two-pass kernels): rows
    past the input read as zeros; the codes cover the padded rows."""
    x = inputs.activations(rows, cols, seed=rows + 5 * cols, device="cpu")
    q, s = halo.halo_hadamard_quantize(_cuda(x), ROWS, 128, qtype)
    torch.cuda.synchronize()
    assert tuple(q.shape) == (halo.padded_length(rows, 128), cols)
    codes, scales, t = oracle_operand(x, 0, 128, qtype)
    check_codes(q, s, codes, scales, t, qtype, blk=128, axis=0)


def test_rotq_dual_padded_parity():
    x = inputs.activations(7, 1000, seed=77, device="cpu")
    q8, s8, qf, sf = halo.halo_hadamard_quantize_dual(_cuda(x), 128)
    torch.cuda.synchronize()
    for q, s, qt in ((q8, s8, INT8), (qf, sf, E4M3)):
        codes, scales, t = oracle_operand(x, 1, 128, qt)
        check_codes(q, s, codes, scales, t, qt, blk=128, axis=1)


@pytest.mark.parametrize("axis,rows,cols", [(COLS, 37, 1000), (ROWS, 1000, 48)])
def test_padded_variants_parity(axis, rows, cols):
    """Signs and random bits cover the padded length (their padded entries meet
    zeros and change nothing)."""
    x = inputs.activations(rows, cols, seed=91, device="cpu")
    n = cols if axis == COLS else rows
    npad = halo.padded_length(n, 128)
    s = _signs_t(npad, seed=92)
    shape = (rows, npad) if axis == COLS else (npad, cols)
    rb = _rand_bits(*shape, seed=93)
    q, sc = halo.halo_hadamard_quantize_ex(_cuda(x), axis, 128, INT8, signs=_cuda(s), rand_bits=_cuda(rb))
    torch.cuda.synchronize()
    along = 1 if axis == COLS else 0
    v = oracle.rotate_signed(x, 128, along, s.numpy()[:n])
    codes, scales, t = oracle.quantize_stochastic(v, 0 if along == 1 else 1, INT8, rb.numpy().view(np.uint16))
    check_codes_stochastic(q, sc, codes, scales, t, rb.numpy().view(np.uint16), INT8, blk=128, axis=along)


@pytest.mark.parametrize("blk", [128, 256])
def test_linear_fwd_padded_k(blk):
    m, n, k = 200, 136, 1000
    x = inputs.activations(m, k, seed=61, device="cpu")
    w = inputs.weights(n, k, seed=62, device="cpu")
    y = halo.halo_linear_fwd(_cuda(x), _cuda(w), blk, INT8, FP32)
    torch.cuda.synchronize()
    check_output(y, oracle.linear_fwd(x, w, blk, INT8))


def test_linear_bwd_padded_n_and_m():
    m, n, k = 1000, 200, 256
    dy = inputs.grads(m, n, seed=63, device="cpu")
    x = inputs.activations(m, k, seed=64, device="cpu")
    w = inputs.weights(n, k, seed=65, device="cpu")
    dx, _ = halo.halo_linear_bwd(_cuda(dy), None, _cuda(w), 128, INT8, FP32, FP32, want_dw=False)
    torch.cuda.synchronize()
    check_output(dx, oracle.linear_bwd_dx(dy, w, 128, INT8))          # N = 200, padded to 256
    n2 = 208  # dW needs N % 16
    dy2 = inputs.grads(m, n2, seed=66, device="cpu")
    _, dw = halo.halo_linear_bwd(_cuda(dy2), _cuda(x), None, 128, E4M3, FP32, FP32, want_dx=False)
    torch.cuda.synchronize()
    check_output(dw, oracle.linear_bwd_dw(dy2, x, 128, E4M3))         # M = 1000, padded to 1024


# -------------------------------------------------------------- group-wise scales
@pytest.mark.parametrize("qtype", [INT8, E4M3])
@pytest.mark.parametrize("rows,cols,blk,group", [(300, 640, 128, 64), (300, 640, 128, 128), (130, 512, 256, 64),
                                                 (5, 1000, 128, 64), (3, 28672, 128, 128), (3, 24576, 128, 64),
                                                 (300, 28672, 128, 128), (2000, 8192, 128, 64)])
def test_rotq_rows_grouped_parity(qtype, rows, cols, blk, group):
    x = inputs.activations(rows, cols, seed=rows + 2 * cols + group, device="cpu")
    x[min(1, rows - 1), :64] = 0  # an all-zero group
    q, s = halo.halo_hadamard_quantize_grouped(_cuda(x), COLS, blk, group, qtype)
    torch.cuda.synchronize()
    codes, scales, t = oracle.quantize_grouped(oracle.rotate(x, blk, 1), 1, group, qtype)
    assert tuple(s.shape) == scales.shape
    check_codes(q, s, codes, scales, t, qtype, blk=blk, axis=1)


@pytest.mark.parametrize("qtype", [INT8, E4M3])
@pytest.mark.parametrize("rows,cols,group", [(1024, 208, 64), (1024, 208, 128), (1000, 48, 64), (8320, 32, 128),
                                             (128, 16, 64)])
def test_rotq_cols_grouped_parity(qtype, rows, cols, group):
    x = inputs.activations(rows, cols, seed=rows + 3 * cols + group, device="cpu")
    x[:64, min(3, cols - 1)] = 0  # an all-zero group
    q, s = halo.halo_hadamard_quantize_grouped(_cuda(x), ROWS, 128, group, qtype)
    torch.cuda.synchronize()
    codes, scales, t = oracle.quantize_grouped(oracle.rotate(x, 128, 0), 0, group, qtype)
    assert tuple(s.shape) == scales.shape
    check_codes(q, s, codes, scales, t, qtype, blk=128, axis=0)


def _group_scales(outer, ngroups, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.rand((outer, ngroups), generator=g) * 1.5 + 0.25).to(torch.float32)


@pytest.mark.parametrize("qtype", [INT8, E4M3])
@pytest.mark.parametrize("group", [64, 128])
@pytest.mark.parametrize("a_major,b_major", [(0, 0), (1, 1), (0, 1), (1, 0)])
@pytest.mark.parametrize("m,n,k", [(300, 520, 640), (16, 16, 256), (640, 272, 1024)])
def test_qgemm_grouped_parity(qtype, group, a_major, b_major, m, n, k):
    """Random codes and group scales; the GPU promotes each group's exact
    partial product into fp32 running sums, the oracle sums in fp64."""
    if a_major == 1 and m % 16 or b_major == 1 and n % 16:
        pytest.skip("MN-major storage needs a 16-byte row stride")
    a = _rand_codes(m, k, qtype, seed=m + k + group)
    b = _rand_codes(n, k, qtype, seed=n * 3 + k)
    sa = _group_scales(m, k // group, seed=m)
    sb = _group_scales(n, k // group, seed=n + 1)
    # scale layouts follow the code storage: [outer, K/g] K-major, [K/g, outer] MN-major
    sa_dev = _cuda(sa if a_major == 0 else sa.t().contiguous())
    sb_dev = _cuda(sb if b_major == 0 else sb.t().contiguous())
    c = halo.halo_qgemm_grouped(_cuda(_stored(a, a_major)), sa_dev, a_major, _cuda(_stored(b, b_major)), sb_dev,
                                b_major, m, n, k, group, qtype, FP32)
    torch.cuda.synchronize()
    ref = oracle.gemm_grouped(a.view(torch.uint8).numpy(), sa.numpy(), b.view(torch.uint8).numpy(), sb.numpy(),
                              group, qtype)
    err = np.abs(c.cpu().numpy().astype(np.float64) - ref).max() / np.abs(ref).max()
    assert err < 1e-5, err


@pytest.mark.parametrize("qtype", [INT8, E4M3])
@pytest.mark.parametrize("group", [64, 128])
@pytest.mark.parametrize("a_major,b_major", [(0, 0), (1, 1)])
def test_qgemm_grouped_many_tiles_sampled(qtype, group, a_major, b_major):
    """4096 x 4000 x 1920: 512 tiles of 128 x 256 over 148 CTAs (each CTA runs
    several tiles, the partial and scale-staging phases carry across them),
    15 or 30 groups (a ragged last scale chunk), N not a multiple of 256 (the
    last tile's second B box lies past the matrix).  Sampled rows and columns
    against the oracle's grouped product of those rows and columns."""
    m, n, k = 4096, 4000, 1920
    a = _rand_codes(m, k, qtype, seed=91 + group)
    b = _rand_codes(n, k, qtype, seed=92 + group)
    sa = _group_scales(m, k // group, seed=93)
    sb = _group_scales(n, k // group, seed=94)
    sa_dev = _cuda(sa if a_major == 0 else sa.t().contiguous())
    sb_dev = _cuda(sb if b_major == 0 else sb.t().contiguous())
    c = halo.halo_qgemm_grouped(_cuda(_stored(a, a_major)), sa_dev, a_major, _cuda(_stored(b, b_major)), sb_dev,
                                b_major, m, n, k, group, qtype, FP32)
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(95)
    rows = torch.cat([torch.tensor([0, 127, 128, m - 1]), torch.randint(0, m, (28,), generator=g)])
    cols = torch.cat([torch.tensor([0, 255, 256, 3839, 3840, n - 1]), torch.randint(0, n, (26,), generator=g)])
    ref = oracle.gemm_grouped(a[rows].view(torch.uint8).numpy(), sa[rows].numpy(), b[cols].view(torch.uint8).numpy(),
                              sb[cols].numpy(), group, qtype)
    got = c.cpu()[rows][:, cols].numpy().astype(np.float64)
    err = np.abs(got - ref).max() / np.abs(ref).max()
    assert err < 1e-5, err
    st, site = halo.halo_device_error()
    assert st == halo.HALO_OK, f"bounded wait ran out at site {site:#x}"


@pytest.mark.parametrize("qtype", [INT8, E4M3])
@pytest.mark.parametrize("group", [64, 128])
def test_linear_grouped_parity(qtype, group):
    m, n, k = 384, 320, 640
    x = inputs.activations(m, k, seed=71, device="cpu")
    w = inputs.weights(n, k, seed=72, device="cpu")
    dy = inputs.grads(m, n, seed=73, device="cpu")
    y = halo.halo_linear_fwd_grouped(_cuda(x), _cuda(w), 128, group, qtype, FP32)
    dx, dw = halo.halo_linear_bwd_grouped(_cuda(dy), _cuda(x), _cuda(w), 128, group, qtype, FP32, FP32)
    torch.cuda.synchronize()
    check_output(y, oracle.linear_fwd_grouped(x, w, 128, group, qtype))
    check_output(dx, oracle.linear_bwd_dx_grouped(dy, w, 128, group, qtype))
    check_output(dw, oracle.linear_bwd_dw_grouped(dy, x, 128, group, qtype))


def test_linear_grouped_padded_and_bf16():
    m, n, k = 200, 136, 1000
    x = inputs.activations(m, k, seed=74, device="cpu")
    w = inputs.weights(n, k, seed=75, device="cpu")
    y = halo.halo_linear_fwd_grouped(_cuda(x), _cuda(w), 128, 64, INT8, BF16)
    torch.cuda.synchronize()
    check_output(y, oracle.linear_fwd_grouped(x, w, 128, 64, INT8))


# ------------------------------------------------------------------- edge cases
def test_single_token_forward_and_tiny_backward():
    x = inputs.activations(1, 256, seed=91, device="cpu")
    w = inputs.weights(16, 256, seed=92, device="cpu")
    y = halo.halo_linear_fwd(_cuda(x), _cuda(w), 128, INT8, FP32)
    torch.cuda.synchronize()
    check_output(y, oracle.linear_fwd(x, w, 128, INT8))
    m, n, k = 128, 128, 16  # one 128-block along tokens and along N
    dy = inputs.grads(m, n, seed=93, device="cpu")
    xb = inputs.activations(m, k, seed=94, device="cpu")
    wb = inputs.weights(n, k, seed=95, device="cpu")
    dx, dw = halo.halo_linear_bwd(_cuda(dy), _cuda(xb), _cuda(wb), 128, INT8, FP32, FP32)
    torch.cuda.synchronize()
    check_output(dx, oracle.linear_bwd_dx(dy, wb, 128, INT8))
    check_output(dw, oracle.linear_bwd_dw(dy, xb, 128, INT8))


def test_all_zero_operands_give_zero_scales_codes_and_outputs():
    x = torch.zeros((256, 512), dtype=torch.bfloat16, device="cuda")
    w = inputs.weights(128, 512, seed=96, device="cuda")
    for axis in (COLS, ROWS):
        q, s = halo.halo_hadamard_quantize(x, axis, 128, INT8)
        torch.cuda.synchronize()
        assert torch.all(s == 0) and torch.all(q.view(torch.uint8) == 0)
    y = halo.halo_linear_fwd(x, w, 128, INT8, FP32)
    torch.cuda.synchronize()
    assert torch.all(y == 0)


@pytest.mark.parametrize("qtype", [INT8, E4M3])
def test_rotq_rows_longest_row(qtype):
    """32768 elements per row: 256 chunks, a row group of 8 warps (the largest)."""
    x = inputs.activations(6, 32768, seed=97, device="cpu")
    q, s = halo.halo_hadamard_quantize(_cuda(x), COLS, 128, qtype)
    torch.cuda.synchronize()
    codes, scales, t = oracle_operand(x, 1, 128, qtype)
    check_codes(q, s, codes, scales, t, qtype, blk=128, axis=1)


# ------------------------------------------------------- dY's two code sets from one read
@pytest.mark.parametrize("qtype", [INT8, E4M3])
@pytest.mark.parametrize("rows,cols", [(4096, 1024), (1000, 528), (256, 8192)])
def test_rotq_both_axes_parity(qtype, rows, cols):
    """halo_hadamard_quantize_both: the per-row codes (rotation along the
    contiguous dim) and the per-column codes (along dim 0) of one matrix, byte
    for byte those of the two separate calls, and both against the oracle."""
    x = inputs.grads(rows, cols, seed=rows + cols, device="cpu")
    x[:, 1] = 0  # an all-zero column
    xd = _cuda(x)
    qr, sr, qc, sc = halo.halo_hadamard_quantize_both(xd, 128, qtype)
    q1, s1 = halo.halo_hadamard_quantize(xd, COLS, 128, qtype)
    q0, s0 = halo.halo_hadamard_quantize(xd, ROWS, 128, qtype)
    torch.cuda.synchronize()
    assert torch.equal(qr.view(torch.uint8), q1.view(torch.uint8)) and torch.equal(sr, s1)
    assert torch.equal(qc.view(torch.uint8), q0.view(torch.uint8)) and torch.equal(sc, s0)
    codes, scales, t = oracle_operand(x, 1, 128, qtype)
    check_codes(qr, sr, codes, scales, t, qtype, blk=128, axis=1)
    codes, scales, t = oracle_operand(x, 0, 128, qtype)
    check_codes(qc, sc, codes, scales, t, qtype, blk=128, axis=0)


@pytest.mark.parametrize("axis,rows,cols", [(ROWS, 4096, 1024), (ROWS, 16384, 96), (ROWS, 28672, 64)])
def test_dim0_variants_on_every_kernel_shape(axis, rows, cols):
    """Random signs and stochastic rounding along dim 0 at the heights that
    select each dimension-0 kernel configuration."""
    x = inputs.activations(rows, cols, seed=rows + cols + 7, device="cpu")
    s = _signs_t(rows, seed=rows + 1)
    rb = _rand_bits(rows, cols, seed=cols + 3)
    q, sc = halo.halo_hadamard_quantize_ex(_cuda(x), axis, 128, INT8, signs=_cuda(s), rand_bits=_cuda(rb))
    torch.cuda.synchronize()
    v = oracle.rotate_signed(x, 128, 0, s.numpy())
    codes, scales, t = oracle.quantize_stochastic(v, 1, INT8, rb.numpy())
    check_codes_stochastic(q, sc, codes, scales, t, rb.numpy(), INT8, blk=128, axis=0)
