"""Pins for the CPU oracle: each check compares it with something other than itself.

Sources of truth used here: dense Sylvester matrices (hand-written golden files
and an independent np.block / scipy construction), orthogonality and
involution of the normalised transform, rotation invariance of the product,
closed-form quantiser bounds, hand-worked quantiser and E4M3 fixtures, torch's
own float8_e4m3fn conversion, and numpy integer / float matmul.
"""
import os

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_bits(x: torch.Tensor) -> np.ndarray:
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def _read_blocks(name):
    mats, cur, key = {}, [], None
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("H"):
            if key:
                mats[key] = np.array(cur, dtype=np.float64)
            key, cur = line, []
        else:
            cur.append([float(v) for v in line.split()])
    mats[key] = np.array(cur, dtype=np.float64)
    return mats


def _rows(name):
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            yield [part.strip() for part in line.split("|")]


def _sylvester_block(n):
    """Independent dense construction: H_{2n} = [[H, H], [H, -H]] via np.block."""
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


# --------------------------------------------------------------------------- FWHT
def test_golden_sylvester_matrices_match_oracle_transform():
    mats = _read_blocks("sylvester_h4_h8.txt")
    for key, h in mats.items():
        n = h.shape[0]
        got = oracle.fwht(np.eye(n))  # row i = transform of e_i = column i of H/sqrt(n)
        np.testing.assert_allclose(got.T * np.sqrt(n), h, atol=1e-12)


def test_golden_worked_transforms():
    for inp, exp in _rows("fwht_worked.txt"):
        x = np.array([float(v) for v in inp.split()])
        e = np.array([float(v) for v in exp.split()])
        np.testing.assert_allclose(oracle.fwht(x), e, atol=1e-12)


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64])
def test_fwht_equals_dense_sylvester(n):
    rng = np.random.default_rng(n)
    x = rng.standard_normal((5, n))
    dense = _sylvester_block(n) / np.sqrt(n)
    np.testing.assert_allclose(oracle.fwht(x), x @ dense.T, rtol=0, atol=1e-12)
    if n >= 2:
        np.testing.assert_array_equal(scipy.linalg.hadamard(n), _sylvester_block(n))


def test_fwht_special_cases():
    np.testing.assert_array_equal(oracle.fwht(np.array([3.25])), [3.25])  # n = 1: identity
    a, b = 1.5, -0.25
    np.testing.assert_allclose(oracle.fwht(np.array([a, b])), [(a + b) / np.sqrt(2), (a - b) / np.sqrt(2)], atol=1e-15)


@pytest.mark.parametrize("n", [16, 128, 256])
def test_fwht_orthogonal_and_involution(n):
    m = oracle.fwht(np.eye(n))
    np.testing.assert_allclose(m @ m.T, np.eye(n), atol=1e-12)
    rng = np.random.default_rng(7)
    x = rng.standard_normal((3, n))
    np.testing.assert_allclose(oracle.fwht(oracle.fwht(x)), x, atol=1e-12)


def test_fwht_is_natural_order_not_bit_reversed():
    """The HALO blog page's recursive even/odd FHT gives the bit-reversed row order of
    Sylvester's matrix; the oracle follows the QWHA page's iterative, natural order."""

    def recursive_even_odd(x):  # restated from the blog page, sec. 2.1 (unnormalised)
        if len(x) == 1:
            return x
        even = recursive_even_odd(x[::2])
        odd = recursive_even_odd(x[1::2])
        return np.concatenate([even + odd, even - odd])

    n = 8
    rec = np.array([recursive_even_odd(e) for e in np.eye(n)]).T  # columns = images of e_j
    bitrev = [int(f"{i:03b}"[::-1], 2) for i in range(n)]
    np.testing.assert_array_equal(rec, _sylvester_block(n)[bitrev])
    got = oracle.fwht(np.eye(n)).T * np.sqrt(n)
    np.testing.assert_allclose(got, _sylvester_block(n), atol=1e-12)


def test_block_local_rotation_is_block_diagonal():
    rng = np.random.default_rng(3)
    x = torch.from_numpy(rng.standard_normal((6, 512)).astype(np.float32)).to(torch.bfloat16)
    xf = x.float().double().numpy()
    for blk in (128, 256):
        hb = _sylvester_block(blk) / np.sqrt(blk)
        dense = scipy.linalg.block_diag(*([hb] * (512 // blk)))
        got = oracle.rotate(x, blk, axis=1)
        np.testing.assert_allclose(got, xf @ dense.T, atol=1e-11)
        # dimension-0 rotation of x^T is the transpose of the dimension-1 rotation of x
        got0 = oracle.rotate(x.t().contiguous(), blk, axis=0)
        np.testing.assert_allclose(got0, got.T, atol=1e-12)


def test_bf16_widening_matches_torch():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy().astype(np.float64)
    got = oracle.bf16_to_f64(bits)
    finite = np.isfinite(t)
    np.testing.assert_array_equal(got[finite], t[finite])


def test_rotation_invariance_of_the_product():
    """(X H)(W H)^T = X W^T: the rotation is orthogonal along the contraction dim."""
    rng = np.random.default_rng(11)
    x = torch.from_numpy(rng.standard_normal((32, 512)).astype(np.float32)).to(torch.bfloat16)
    w = torch.from_numpy((0.02 * rng.standard_normal((24, 512))).astype(np.float32)).to(torch.bfloat16)
    xr = oracle.rotate(x, 128, axis=1)
    wr = oracle.rotate(w, 128, axis=1)
    ref = x.double().numpy() @ w.double().numpy().T
    got = xr @ wr.T
    assert np.max(np.abs(got - ref)) <= 1e-5 * np.max(np.abs(ref))
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref)) * 512


# ----------------------------------------------------------------------- quantiser
def test_golden_int8_quantisation():
    for inp, scale, codes in _rows("quantize_int8_worked.txt"):
        v = np.array([[float(t) for t in inp.split()]])
        q, s, _ = oracle.quantize(v, axis=0, qtype=oracle.INT8)
        assert s[0] == np.float32(float(scale))
        np.testing.assert_array_equal(q.view(np.int8)[0], [int(c) for c in codes.split()])


def test_int8_quantiser_bounds():
    rng = np.random.default_rng(5)
    v = rng.standard_normal((40, 300)) * np.exp(rng.standard_normal((40, 1)))
    v[3, 17] = 123.0  # an outlier row
    q, s, t = oracle.quantize(v, axis=0, qtype=oracle.INT8)
    qi = q.view(np.int8).astype(np.int64)
    assert np.all(np.abs(qi) <= 127)
    for r in range(v.shape[0]):
        j = np.argmax(np.abs(v[r]))
        assert abs(qi[r, j]) == 127 and np.sign(qi[r, j]) == np.sign(v[r, j])
        assert np.float32(np.max(np.abs(v[r])) / 127.0) == s[r]
        err = np.abs(v[r] - qi[r] * np.float64(s[r]))
        assert np.all(err <= 0.5 * np.float64(s[r]) * (1 + 1e-12))
    # per-column grouping is the transpose of per-row grouping
    q2, s2, _ = oracle.quantize(v.T.copy(), axis=1, qtype=oracle.INT8)
    np.testing.assert_array_equal(q2.T, q)
    np.testing.assert_array_equal(s2, s)


def test_zero_group_gives_zero_scale_and_codes():
    v = np.zeros((2, 8))
    v[1, 3] = -2.0
    for qt in (oracle.INT8, oracle.E4M3):
        q, s, _ = oracle.quantize(v, axis=0, qtype=qt)
        assert s[0] == 0.0 and np.all(q[0] == 0)
        assert s[1] > 0


def test_golden_e4m3_encodings():
    for value, code in _rows("e4m3_worked.txt"):
        assert oracle.e4m3_encode(np.array([float(value)]))[0] == int(code, 16), value


def test_e4m3_decode_matches_torch_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().double().numpy()
    got = oracle.e4m3_decode(codes)
    nan = np.isnan(ref)
    np.testing.assert_array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], ref[~nan])


def test_e4m3_encode_matches_torch_on_every_bf16_value():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float()
    v64 = vals.double().numpy()
    finite = np.isfinite(v64)
    inrange = finite & (np.abs(v64) <= 448.0)
    ref = vals[torch.from_numpy(inrange)].to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(v64[inrange])
    np.testing.assert_array_equal(got, ref)
    # above the largest finite value the conversion saturates to +-448
    big = v64[finite & (np.abs(v64) > 448.0)]
    enc = oracle.e4m3_encode(big)
    np.testing.assert_array_equal(enc, np.where(big > 0, 0x7E, 0xFE))


def test_e4m3_quantiser_error_bound():
    rng = np.random.default_rng(9)
    v = rng.standard_normal((16, 256)) * 3
    q, s, t = oracle.quantize(v, axis=0, qtype=oracle.E4M3)
    dec = oracle.e4m3_decode(q)
    assert np.all(np.abs(dec) <= 448)
    a = np.abs(t)
    # half the grid spacing at |t|: 2^-10 below 2^-6, else 2^(floor(log2|t|) - 4)
    half_ulp = np.where(a < 2.0**-6, 2.0**-10, 2.0 ** (np.floor(np.log2(np.maximum(a, 1e-300))) - 4))
    assert np.all(np.abs(t - dec) <= half_ulp * (1 + 1e-12))
    for r in range(v.shape[0]):
        j = np.argmax(np.abs(v[r]))
        assert abs(dec[r, j]) == 448.0


def test_boundary_distance():
    d = oracle.boundary_distance(np.array([2.5, 2.0, -7.5, 0.0]), oracle.INT8)
    np.testing.assert_allclose(d, [0.0, 0.25, 0.0, np.inf])
    d = oracle.boundary_distance(np.array([17.0, 16.0, 1.0625]), oracle.E4M3)
    np.testing.assert_allclose(d, [0.0, 1.0 / 16, 0.0])


# --------------------------------------------------------------------------- GEMMs
def test_int_gemm_equals_numpy():
    rng = np.random.default_rng(1)
    a = rng.integers(-127, 128, size=(37, 96)).astype(np.int8)
    b = rng.integers(-127, 128, size=(53, 96)).astype(np.int8)
    np.testing.assert_array_equal(oracle.gemm_i8(a, b), a.astype(np.int64) @ b.astype(np.int64).T)


def test_e4m3_gemm_equals_numpy_on_torch_decoded_values():
    rng = np.random.default_rng(2)
    a = rng.integers(0, 256, size=(19, 64)).astype(np.uint8)
    b = rng.integers(0, 256, size=(23, 64)).astype(np.uint8)
    a[(a & 0x7F) == 0x7F] = 0  # drop NaN codes
    b[(b & 0x7F) == 0x7F] = 0
    da = torch.from_numpy(a).view(torch.float8_e4m3fn).double().numpy()
    db = torch.from_numpy(b).view(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_allclose(oracle.gemm_e4m3(a, b), da @ db.T, rtol=1e-14, atol=1e-14)


# ------------------------------------------------------------------ linear layer
def _bound(xr, sx, wr, sw, qmax_half):
    """Worst-case |Y - Xr Wr^T| from per-element quantisation errors |dx| <= e_x, |dw| <= e_w."""
    ex = qmax_half(xr, sx)
    ew = qmax_half(wr, sw)
    return ex @ np.abs(wr).T + np.abs(xr) @ ew.T + ex @ ew.T


def _int8_err(v, s_row):
    return np.broadcast_to(0.5 * s_row.astype(np.float64)[:, None], v.shape)


@pytest.mark.parametrize("blk", [128, 256])
def test_linear_fwd_within_quantisation_bound(blk):
    rng = np.random.default_rng(21)
    x = torch.from_numpy(rng.standard_normal((48, 512)).astype(np.float32))
    x[:, [5, 300]] *= 50
    x = x.to(torch.bfloat16)
    w = torch.from_numpy((0.02 * rng.standard_normal((40, 512))).astype(np.float32)).to(torch.bfloat16)
    y = oracle.linear_fwd(x, w, blk, oracle.INT8)
    exact = x.double().numpy() @ w.double().numpy().T
    xr = oracle.rotate(x, blk, 1)
    wr = oracle.rotate(w, blk, 1)
    _, sx, _ = oracle.quantize(xr, 0, oracle.INT8)
    _, sw, _ = oracle.quantize(wr, 0, oracle.INT8)
    bound = _bound(xr, sx, wr, sw, _int8_err)
    assert np.all(np.abs(y - exact) <= bound * (1 + 1e-9) + 1e-12)
    # a transposed or mis-indexed scale would break the bound by far
    assert np.max(np.abs(y - exact)) < 0.05 * np.max(np.abs(exact))


def test_linear_bwd_within_quantisation_bound():
    rng = np.random.default_rng(22)
    m, n, k, blk = 256, 128, 384, 128
    dy = torch.from_numpy((1e-3 * rng.standard_normal((m, n))).astype(np.float32)).to(torch.bfloat16)
    w = torch.from_numpy((0.02 * rng.standard_normal((n, k))).astype(np.float32)).to(torch.bfloat16)
    xf = torch.from_numpy(rng.standard_normal((m, k)).astype(np.float32))
    xf[:, 7] *= 50
    x = xf.to(torch.bfloat16)
    dyd, wd, xd = dy.double().numpy(), w.double().numpy(), x.double().numpy()
    # dX = dY W, contraction over n
    dx = oracle.linear_bwd_dx(dy, w, blk, oracle.INT8)
    a = oracle.rotate(dy, blk, 1)                      # [m, n]
    b = oracle.rotate(w, blk, 0).T                     # [k, n]
    _, sa, _ = oracle.quantize(a, 0, oracle.INT8)
    _, sb, _ = oracle.quantize(b.copy(), 0, oracle.INT8)
    exact = dyd @ wd
    assert np.all(np.abs(dx - exact) <= _bound(a, sa, b, sb, _int8_err) * (1 + 1e-9) + 1e-15)
    assert np.max(np.abs(dx - exact)) < 0.05 * np.max(np.abs(exact))
    # dW = dY^T X, contraction over m
    dw = oracle.linear_bwd_dw(dy, x, blk, oracle.INT8)
    a = oracle.rotate(dy, blk, 0).T                    # [n, m]
    b = oracle.rotate(x, blk, 0).T                     # [k, m]
    _, sa, _ = oracle.quantize(a.copy(), 0, oracle.INT8)
    _, sb, _ = oracle.quantize(b.copy(), 0, oracle.INT8)
    exact = dyd.T @ xd
    assert np.all(np.abs(dw - exact) <= _bound(a, sa, b, sb, _int8_err) * (1 + 1e-9) + 1e-15)
    assert np.max(np.abs(dw - exact)) < 0.05 * np.max(np.abs(exact))


def test_linear_fwd_e4m3_close_to_exact():
    rng = np.random.default_rng(23)
    x = torch.from_numpy(rng.standard_normal((32, 256)).astype(np.float32)).to(torch.bfloat16)
    w = torch.from_numpy((0.02 * rng.standard_normal((16, 256))).astype(np.float32)).to(torch.bfloat16)
    y = oracle.linear_fwd(x, w, 128, oracle.E4M3)
    exact = x.double().numpy() @ w.double().numpy().T
    # E4M3 keeps 3 mantissa bits: per-element relative error <= 2^-4; products and
    # sums of K terms give a normwise error well under 10%.
    assert np.max(np.abs(y - exact)) < 0.1 * np.max(np.abs(exact))


def test_rotation_reduces_error_on_outlier_channels():
    """Informational property behind the method: rotating spreads outlier channels, so the
    quantised product lands closer to the exact one than without rotation."""
    rng = np.random.default_rng(24)
    xf = torch.from_numpy(rng.standard_normal((64, 512)).astype(np.float32))
    xf[:, [3, 99, 250, 400]] *= 50
    x = xf.to(torch.bfloat16)
    w = torch.from_numpy((0.02 * rng.standard_normal((64, 512))).astype(np.float32)).to(torch.bfloat16)
    exact = x.double().numpy() @ w.double().numpy().T
    y_rot = oracle.linear_fwd(x, w, 128, oracle.INT8)
    # no rotation: quantise the raw operands with the same quantiser
    qx, sx, _ = oracle.quantize(x.double().numpy(), 0, oracle.INT8)
    qw, sw, _ = oracle.quantize(w.double().numpy(), 0, oracle.INT8)
    y_plain = oracle.dequant(oracle.gemm_i8(qx, qw).astype(np.float64), sx, sw)
    assert np.linalg.norm(y_rot - exact) < 0.8 * np.linalg.norm(y_plain - exact)


def test_composition_of_rotated_qgemm_parts():
    rng = np.random.default_rng(25)
    x = torch.from_numpy(rng.standard_normal((16, 256)).astype(np.float32)).to(torch.bfloat16)
    w = torch.from_numpy(rng.standard_normal((8, 256)).astype(np.float32)).to(torch.bfloat16)
    aq, sa, bq, sb = oracle.rotated_qgemm_parts(x, True, w, True, 128, oracle.INT8)
    y = oracle.dequant(oracle.gemm_i8(aq, bq).astype(np.float64), sa, sb)
    np.testing.assert_array_equal(y, oracle.linear_fwd(x, w, 128, oracle.INT8))


# ------------------------------------------------------------- random-sign rotation
def _signs(n, seed):
    rng = np.random.default_rng(seed)
    return np.where(rng.random(n) < 0.5, -1, 1).astype(np.int8)


def test_signed_rotation_all_plus_is_plain_rotation():
    rng = np.random.default_rng(31)
    x = torch.from_numpy(rng.standard_normal((8, 512)).astype(np.float32)).to(torch.bfloat16)
    ones = np.ones(512, dtype=np.int8)
    np.testing.assert_array_equal(oracle.rotate_signed(x, 128, 1, ones), oracle.rotate(x, 128, 1))
    np.testing.assert_array_equal(oracle.rotate_signed(x.t().contiguous(), 128, 0, ones),
                                  oracle.rotate(x.t().contiguous(), 128, 0))


def test_signed_rotation_equals_dense_h_times_diag():
    rng = np.random.default_rng(32)
    x = torch.from_numpy(rng.standard_normal((5, 256)).astype(np.float32)).to(torch.bfloat16)
    s = _signs(256, 1)
    hb = _sylvester_block(128) / np.sqrt(128)
    dense = scipy.linalg.block_diag(hb, hb) @ np.diag(s.astype(np.float64))
    np.testing.assert_allclose(oracle.rotate_signed(x, 128, 1, s), x.double().numpy() @ dense.T, atol=1e-11)
    got0 = oracle.rotate_signed(x.t().contiguous(), 128, 0, s)
    np.testing.assert_allclose(got0, oracle.rotate_signed(x, 128, 1, s).T, atol=1e-12)


def test_signed_rotation_keeps_the_product_only_with_matching_signs():
    rng = np.random.default_rng(33)
    x = torch.from_numpy(rng.standard_normal((16, 384)).astype(np.float32)).to(torch.bfloat16)
    w = torch.from_numpy(rng.standard_normal((12, 384)).astype(np.float32)).to(torch.bfloat16)
    s = _signs(384, 2)
    ref = x.double().numpy() @ w.double().numpy().T
    same = oracle.rotate_signed(x, 128, 1, s) @ oracle.rotate_signed(w, 128, 1, s).T
    np.testing.assert_allclose(same, ref, atol=1e-10 * np.max(np.abs(ref)))
    other = oracle.rotate_signed(x, 128, 1, s) @ oracle.rotate_signed(w, 128, 1, _signs(384, 3)).T
    assert np.max(np.abs(other - ref)) > 0.1 * np.max(np.abs(ref))


# ----------------------------------------------------------- stochastic rounding
def test_golden_stochastic_quantisation():
    for qt, row, bits, codes in _rows("quantize_stochastic_worked.txt"):
        v = np.array([[float(t) for t in row.split()]])
        rb = np.array([[int(b) for b in bits.split()]], dtype=np.uint16)
        qtype = oracle.INT8 if qt == "int8" else oracle.E4M3
        q, s, _ = oracle.quantize_stochastic(v, 0, qtype, rb)
        assert s[0] == 1.0
        if qtype == oracle.INT8:
            np.testing.assert_array_equal(q.view(np.int8)[0], [int(c) for c in codes.split()])
        else:
            np.testing.assert_array_equal(q[0], [int(c, 16) for c in codes.split()])


def test_stochastic_codes_are_grid_neighbours_with_rne_scales():
    rng = np.random.default_rng(34)
    v = rng.standard_normal((20, 256)) * 3
    rb = rng.integers(0, 65536, size=v.shape).astype(np.uint16)
    for qt in (oracle.INT8, oracle.E4M3):
        q, s, t = oracle.quantize_stochastic(v, 0, qt, rb)
        _, s_rne, t_rne = oracle.quantize(v, 0, qt)
        np.testing.assert_array_equal(s, s_rne)
        np.testing.assert_array_equal(t, t_rne)
        if qt == oracle.INT8:
            qi = q.view(np.int8).astype(np.float64)
            assert np.all((qi == np.floor(t)) | (qi == np.floor(t) + 1) | (np.abs(qi) == 127))
        else:
            d = oracle.e4m3_decode(q)
            a = np.abs(t)
            quantum = np.where(a < 2.0**-6, 2.0**-9, 2.0 ** (np.floor(np.log2(np.maximum(a, 1e-300))) - 3))
            lo = np.floor(a / quantum) * quantum
            assert np.all((np.abs(d) == lo) | (np.abs(d) == lo + quantum) | (np.abs(d) == 448))
            assert np.all((d == 0) | (np.sign(d) == np.sign(t)))


def test_stochastic_rounding_is_unbiased():
    """E[q] = t up to the 2^-16 resolution of the random bits."""
    rng = np.random.default_rng(35)
    row = np.concatenate([[127.0], rng.uniform(-120, 120, 63)])
    trials = 4000
    v = np.tile(row, (trials, 1))
    rb = rng.integers(0, 65536, size=v.shape).astype(np.uint16)
    q, s, t = oracle.quantize_stochastic(v, 0, oracle.INT8, rb)
    mean = q.view(np.int8).astype(np.float64).mean(axis=0)
    # each code is a Bernoulli step of 1: sd <= 0.5 / sqrt(trials)
    assert np.all(np.abs(mean - t[0]) <= 5 * 0.5 / np.sqrt(trials) + 2.0**-16)
    # round to nearest is biased on the same values; stochastic is not
    q_rne, _, _ = oracle.quantize(v[:1], 0, oracle.INT8)
    assert np.mean(np.abs(q_rne.view(np.int8)[0] - t[0])) > 4 * np.mean(np.abs(mean - t[0]))


# ------------------------------------------------------------------ zero padding
@pytest.mark.parametrize("blk", [128, 256])
@pytest.mark.parametrize("axis,shape", [(1, (3, 300)), (1, (2, 5)), (0, (200, 3)), (0, (70, 2))])
def test_padded_rotation_equals_dense_h_on_zero_extended_input(blk, axis, shape):
    """A rotated length that is not a multiple of blk: the oracle's rotation
    equals the dense normalised Sylvester matrix applied block by block to the
    input extended with zeros (built here independently)."""
    if axis == 0 and blk == 256:
        pytest.skip("dimension-0 rotations use block 128")
    rng = np.random.default_rng(sum(shape) + blk)
    x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).to(torch.bfloat16)
    xd = x.double().numpy()
    rows, cols = shape
    n = cols if axis == 1 else rows
    n_pad = -(-n // blk) * blk
    h = _sylvester_block(blk) / np.sqrt(blk)
    if axis == 1:
        ext = np.zeros((rows, n_pad))
        ext[:, :cols] = xd
        expect = np.concatenate([ext[:, b:b + blk] @ h.T for b in range(0, n_pad, blk)], axis=1)
    else:
        ext = np.zeros((n_pad, cols))
        ext[:rows, :] = xd
        expect = np.concatenate([h @ ext[b:b + blk, :] for b in range(0, n_pad, blk)], axis=0)
    got = oracle.rotate(x, blk, axis)
    assert got.shape == expect.shape
    np.testing.assert_allclose(got, expect, rtol=1e-12, atol=1e-12 * np.abs(expect).max())


def test_padded_linear_layers_within_quantisation_bound():
    """fwd with K, dX with N, dW with M not multiples of 128: the results stay
    within the worst-case quantisation bound around the exact unpadded
    products (zero padding leaves every product unchanged; anything else in the
    padded positions would not)."""
    rng = np.random.default_rng(31)
    m, n, k, blk = 200, 136, 328, 128
    x = torch.from_numpy(rng.standard_normal((m, k)).astype(np.float32))
    x[:, 3] *= 50
    x = x.to(torch.bfloat16)
    w = torch.from_numpy((0.02 * rng.standard_normal((n, k))).astype(np.float32)).to(torch.bfloat16)
    dy = torch.from_numpy((1e-3 * rng.standard_normal((m, n))).astype(np.float32)).to(torch.bfloat16)
    xd, wd, dyd = x.double().numpy(), w.double().numpy(), dy.double().numpy()

    def check(got, exact, a, b):
        _, sa, _ = oracle.quantize(a, 0, oracle.INT8)
        _, sb, _ = oracle.quantize(b, 0, oracle.INT8)
        assert got.shape == exact.shape
        assert np.all(np.abs(got - exact) <= _bound(a, sa, b, sb, _int8_err) * (1 + 1e-9) + 1e-15)
        assert np.max(np.abs(got - exact)) < 0.05 * np.max(np.abs(exact))

    # Y = X W^T over K = 328 (padded to 384)
    check(oracle.linear_fwd(x, w, blk, oracle.INT8), xd @ wd.T, oracle.rotate(x, blk, 1), oracle.rotate(w, blk, 1))
    # dX = dY W over N = 136 (padded to 256)
    check(oracle.linear_bwd_dx(dy, w, blk, oracle.INT8), dyd @ wd, oracle.rotate(dy, blk, 1),
          np.ascontiguousarray(oracle.rotate(w, blk, 0).T))
    # dW = dY^T X over M = 200 (padded to 256)
    check(oracle.linear_bwd_dw(dy, x, blk, oracle.INT8), dyd.T @ xd,
          np.ascontiguousarray(oracle.rotate(dy, blk, 0).T), np.ascontiguousarray(oracle.rotate(x, blk, 0).T))


def test_padding_is_zero_not_garbage():
    """A plausible mistake, planted on the CPU: padding with anything but zeros
    breaks the product (the check above would fail on it)."""
    rng = np.random.default_rng(32)
    x = torch.from_numpy(rng.standard_normal((8, 200)).astype(np.float32)).to(torch.bfloat16)
    w = torch.from_numpy(rng.standard_normal((6, 200)).astype(np.float32)).to(torch.bfloat16)
    xp = oracle.pad_to_blocks(x, 128, 1)
    assert xp.shape == (8, 256) and np.all(xp[:, 200:] == 0)
    exact = x.double().numpy() @ w.double().numpy().T
    xr, wr = oracle.rotate(x, 128, 1), oracle.rotate(w, 128, 1)
    np.testing.assert_allclose(xr @ wr.T, exact, rtol=1e-10, atol=1e-10)
    # ones in both operands' padding add 56 to every product
    bad_x, bad_w = xp.copy(), oracle.pad_to_blocks(w, 128, 1)
    bad_x[:, 200:] = _bf16_bits(torch.ones(8, 56, dtype=torch.bfloat16))
    bad_w[:, 200:] = _bf16_bits(torch.ones(6, 56, dtype=torch.bfloat16))
    bad = oracle.rotate(bad_x, 128, 1) @ oracle.rotate(bad_w, 128, 1).T
    np.testing.assert_allclose(bad - exact, 56.0, rtol=1e-9)


# ------------------------------------------------------------ group-wise scales
def test_golden_grouped_quantisation():
    for qt, group, inp, scales, codes in _rows("quantize_grouped_worked.txt"):
        qtype = oracle.INT8 if qt == "int8" else oracle.E4M3
        v = np.array([[float(t) for t in inp.split()]])
        g = int(group)
        q, s, _ = oracle.quantize_grouped(v, 1, g, qtype)
        np.testing.assert_array_equal(s[0], np.array([float(x) for x in scales.split()], dtype=np.float32))
        if qtype == oracle.INT8:
            np.testing.assert_array_equal(q.view(np.int8)[0], [int(c) for c in codes.split()])
        else:
            np.testing.assert_array_equal(q[0], [int(c, 16) for c in codes.split()])
        # the same values down a column (groups of consecutive rows)
        qc, sc, _ = oracle.quantize_grouped(v.T.copy(), 0, g, qtype)
        np.testing.assert_array_equal(qc[:, 0], q[0])
        np.testing.assert_array_equal(sc[:, 0], s[0])


@pytest.mark.parametrize("qtype", [oracle.INT8, oracle.E4M3])
def test_grouped_with_one_group_is_the_per_row_quantiser(qtype):
    rng = np.random.default_rng(41)
    v = rng.standard_normal((7, 256)) * np.exp(rng.standard_normal((7, 1)))
    q1, s1, t1 = oracle.quantize(v, 0, qtype)
    qg, sg, tg = oracle.quantize_grouped(v, 1, 256, qtype)
    np.testing.assert_array_equal(qg, q1)
    np.testing.assert_array_equal(sg[:, 0], s1)
    np.testing.assert_array_equal(tg, t1)
    qc, sc, _ = oracle.quantize_grouped(v.T.copy(), 0, 256, qtype)     # one group down each column
    q0, s0, _ = oracle.quantize(v.T.copy(), 1, qtype)
    np.testing.assert_array_equal(qc, q0)
    np.testing.assert_array_equal(sc[0], s0)


def test_grouped_int8_bounds():
    rng = np.random.default_rng(42)
    v = rng.standard_normal((9, 512))
    v[2, 100] = 77.0
    q, s, _ = oracle.quantize_grouped(v, 1, 64, oracle.INT8)
    qi = q.view(np.int8).astype(np.int64).reshape(9, 8, 64)
    vg = v.reshape(9, 8, 64)
    assert np.all(np.abs(qi) <= 127)
    assert np.all(np.abs(qi).max(axis=2) == 127)             # every group's max maps to +-qmax
    sd = s.astype(np.float64)[:, :, None]
    assert np.all(np.abs(vg - qi * sd) <= sd / 2 * (1 + 1e-6))
    # an outlier only coarsens its own group
    assert s[2, 1] > 20 * np.median(s)
    assert np.sum(s > 20 * np.median(s)) == 1


def test_grouped_gemm_against_numpy_group_sums():
    """numpy computes each group's integer product on its own (einsum over the
    group axis) and weights it by the two scales: a swapped or transposed
    group index anywhere in the oracle fails this."""
    rng = np.random.default_rng(43)
    m, n, k, g = 12, 10, 256, 64
    a = rng.integers(-127, 128, (m, k)).astype(np.int8)
    b = rng.integers(-127, 128, (n, k)).astype(np.int8)
    sa = rng.uniform(0.5, 2.0, (m, k // g)).astype(np.float32)
    sb = rng.uniform(0.5, 2.0, (n, k // g)).astype(np.float32)
    y = oracle.gemm_grouped(a.view(np.uint8), sa, b.view(np.uint8), sb, g, oracle.INT8)
    parts = np.einsum("igk,jgk->ijg", a.reshape(m, k // g, g).astype(np.int64), b.reshape(n, k // g, g).astype(np.int64))
    expect = np.einsum("ijg,ig,jg->ij", parts.astype(np.float64), sa.astype(np.float64), sb.astype(np.float64))
    np.testing.assert_allclose(y, expect, rtol=1e-12)
    # unit scales: the plain integer product
    ones_a, ones_b = np.ones((m, k // g), np.float32), np.ones((n, k // g), np.float32)
    np.testing.assert_array_equal(oracle.gemm_grouped(a.view(np.uint8), ones_a, b.view(np.uint8), ones_b, g,
                                                      oracle.INT8), (a.astype(np.int64) @ b.astype(np.int64).T))
    # E4M3 on torch-decoded values
    ca = rng.integers(0, 256, (m, k)).astype(np.uint8)
    cb = rng.integers(0, 256, (n, k)).astype(np.uint8)
    ca[(ca & 0x7F) == 0x7F] = 0   # no NaN codes
    cb[(cb & 0x7F) == 0x7F] = 0
    da = torch.from_numpy(ca).view(torch.float8_e4m3fn).double().numpy().reshape(m, k // g, g)
    db = torch.from_numpy(cb).view(torch.float8_e4m3fn).double().numpy().reshape(n, k // g, g)
    expect = np.einsum("igk,jgk,ig,jg->ij", da, db, sa.astype(np.float64), sb.astype(np.float64))
    np.testing.assert_allclose(oracle.gemm_grouped(ca, sa, cb, sb, g, oracle.E4M3), expect, rtol=1e-12, atol=1e-12)


def test_grouped_linear_layers_within_quantisation_bound():
    """The three products with group-wise scales (g = 64) stay within the
    worst-case bound of their per-group quantisation errors around the exact
    products, and are tighter than the per-row scales on outlier inputs."""
    rng = np.random.default_rng(44)
    m, n, k, blk, g = 256, 128, 384, 128, 64
    xf = torch.from_numpy(rng.standard_normal((m, k)).astype(np.float32))
    xf[:, 9] *= 50
    x = xf.to(torch.bfloat16)
    w = torch.from_numpy((0.02 * rng.standard_normal((n, k))).astype(np.float32)).to(torch.bfloat16)
    dy = torch.from_numpy((1e-3 * rng.standard_normal((m, n))).astype(np.float32)).to(torch.bfloat16)
    xd, wd, dyd = x.double().numpy(), w.double().numpy(), dy.double().numpy()

    def bound(a_rot, b_rot, along_a, along_b):
        # per-element INT8 errors <= s/2 of the element's own group
        def err(v, along):
            _, s, _ = oracle.quantize_grouped(v, along, g, oracle.INT8)
            e = np.repeat(0.5 * s.astype(np.float64), g, axis=1 if along == 1 else 0)
            return (e if along == 1 else e.T), (v if along == 1 else v.T)
        ea, va = err(a_rot, along_a)
        eb, vb = err(b_rot, along_b)
        return ea @ np.abs(vb).T + np.abs(va) @ eb.T + ea @ eb.T

    y = oracle.linear_fwd_grouped(x, w, blk, g, oracle.INT8)
    exact = xd @ wd.T
    assert np.all(np.abs(y - exact) <= bound(oracle.rotate(x, blk, 1), oracle.rotate(w, blk, 1), 1, 1) * (1 + 1e-9) + 1e-15)
    yr = oracle.linear_fwd(x, w, blk, oracle.INT8)
    assert np.abs(y - exact).max() < np.abs(yr - exact).max()
    dx = oracle.linear_bwd_dx_grouped(dy, w, blk, g, oracle.INT8)
    assert np.all(np.abs(dx - dyd @ wd) <= bound(oracle.rotate(dy, blk, 1), oracle.rotate(w, blk, 0), 1, 0) * (1 + 1e-9) + 1e-15)
    dw = oracle.linear_bwd_dw_grouped(dy, x, blk, g, oracle.INT8)
    assert np.all(np.abs(dw - dyd.T @ xd) <= bound(oracle.rotate(dy, blk, 0), oracle.rotate(x, blk, 0), 0, 0) * (1 + 1e-9) + 1e-15)
