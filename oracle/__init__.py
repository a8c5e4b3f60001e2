"""CPU oracle for the Hadamard-rotated quantized linear layer (HALO, arXiv 2501.02625).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA product path never imports, links or calls it, and the two
share no code: the arithmetic lives in ``halo_oracle.c`` (plain C, fp64), this
module only marshals numpy arrays into it.

What each function computes, and the passage it follows, is stated in
``halo_oracle.c``.  Every function is pinned by ``tests/test_oracle_pins.py``
against something other than itself.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "halo_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libhalo_oracle.so")

INT8 = 0
E4M3 = 1
QMAX = {INT8: 127.0, E4M3: 448.0}

_lib = None


def build(force: bool = False) -> str:
    """Compile ``halo_oracle.c`` into ``libhalo_oracle.so`` with the host gcc."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", _SRC, "-o", _LIB_PATH, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB_PATH)
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    I = ctypes.c_int
    D = ctypes.c_double
    sigs = {
        "halo_oracle_bf16_to_f64": (D, [ctypes.c_uint16]),
        "halo_oracle_bf16_array_to_f64": (None, [P, I64, P]),
        "halo_oracle_fwht": (None, [P, I64]),
        "halo_oracle_rotate_along_cols": (None, [P, I64, I64, I64, I64, P]),
        "halo_oracle_rotate_along_rows": (None, [P, I64, I64, I64, I64, P]),
        "halo_oracle_e4m3_decode": (D, [ctypes.c_uint8]),
        "halo_oracle_e4m3_encode": (ctypes.c_uint8, [D]),
        "halo_oracle_boundary_distance": (D, [D, I]),
        "halo_oracle_e4m3_encode_array": (None, [P, I64, P]),
        "halo_oracle_quantize_grouped": (None, [P, I64, I64, I, I64, I, P, P, P]),
        "halo_oracle_gemm_grouped": (None, [P, P, P, P, I64, I64, I64, I64, I, P]),
        "halo_oracle_e4m3_decode_array": (None, [P, I64, P]),
        "halo_oracle_boundary_distance_array": (None, [P, I64, I, P]),
        "halo_oracle_quantize": (None, [P, I64, I64, I, I, P, P, P]),
        "halo_oracle_rotate_signed_along_cols": (None, [P, I64, I64, I64, I64, P, P]),
        "halo_oracle_rotate_signed_along_rows": (None, [P, I64, I64, I64, I64, P, P]),
        "halo_oracle_quantize_stochastic": (None, [P, I64, I64, I, I, P, P, P, P]),
        "halo_oracle_gemm_i8": (None, [P, P, I64, I64, I64, P]),
        "halo_oracle_gemm_e4m3": (None, [P, P, I64, I64, I64, P]),
        "halo_oracle_dequant": (None, [P, P, P, I64, I64, P]),
        "halo_oracle_rotated_qgemm": (None, [P, I64, I, P, I64, I, I64, I64, I64, I64, I, P, P, P]),
        "halo_oracle_linear_fwd": (None, [P, P, I64, I64, I64, I64, I, P]),
        "halo_oracle_linear_bwd_dx": (None, [P, P, I64, I64, I64, I64, I, P]),
        "halo_oracle_linear_bwd_dw": (None, [P, P, I64, I64, I64, I64, I, P]),
        "halo_oracle_num_threads": (I, []),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _bf16_bits(x) -> np.ndarray:
    """Accept a numpy uint16 array of bf16 bit patterns or a torch bf16 tensor."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch  # only for marshalling a tensor's bytes

    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def num_threads() -> int:
    return int(_load().halo_oracle_num_threads())


def bf16_to_f64(x) -> np.ndarray:
    xb = _bf16_bits(x)
    out = np.empty(xb.shape, dtype=np.float64)
    _load().halo_oracle_bf16_array_to_f64(_ptr(xb), xb.size, _ptr(out))
    return out


def fwht(x: np.ndarray) -> np.ndarray:
    """Normalised Walsh-Hadamard transform of each row of a 2-D fp64 array."""
    lib = _load()
    out = np.array(x, dtype=np.float64, copy=True, order="C")
    if out.ndim == 1:
        lib.halo_oracle_fwht(_ptr(out), out.shape[0])
        return out
    for r in range(out.shape[0]):
        row = np.ascontiguousarray(out[r])
        lib.halo_oracle_fwht(_ptr(row), row.shape[0])
        out[r] = row
    return out


def padded_length(n: int, blk: int) -> int:
    """Length of a dimension of n elements after zero-padding to whole blocks."""
    return -(-n // blk) * blk


def pad_to_blocks(x, blk: int, axis: int) -> np.ndarray:
    """Zero-pad a bf16 matrix along its rotated dimension to a multiple of blk
    (QWHA page sec. 3.1 and 5: inputs whose length is not the transform's are
    filled up with zeros before the transform; with block-local rotations only
    the last block is filled).  axis=1: pad the columns; axis=0: pad the rows.
    bf16 bit patterns in, bf16 bit patterns out (0x0000 is +0)."""
    xb = _bf16_bits(x)
    rows, cols = xb.shape
    if axis == 1:
        out = np.zeros((rows, padded_length(cols, blk)), dtype=np.uint16)
    else:
        out = np.zeros((padded_length(rows, blk), cols), dtype=np.uint16)
    out[:rows, :cols] = xb
    return out


def rotate(x, blk: int, axis: int) -> np.ndarray:
    """Block-local rotation of a bf16 matrix.

    axis=1: along the contiguous dimension (blocks of ``blk`` consecutive
    elements of each row).  axis=0: along dimension 0 (blocks of ``blk``
    consecutive rows of each column).  Returns fp64 of the same shape.  A
    rotated dimension that is not a multiple of blk is zero-padded first
    (``pad_to_blocks``), and the result has the padded shape.
    """
    xb = _bf16_bits(x)
    if (xb.shape[1] if axis == 1 else xb.shape[0]) % blk:
        xb = pad_to_blocks(xb, blk, axis)
    rows, cols = xb.shape
    out = np.empty((rows, cols), dtype=np.float64)
    lib = _load()
    if axis == 1:
        assert cols % blk == 0
        lib.halo_oracle_rotate_along_cols(_ptr(xb), rows, cols, cols, blk, _ptr(out))
    else:
        assert rows % blk == 0
        lib.halo_oracle_rotate_along_rows(_ptr(xb), rows, cols, cols, blk, _ptr(out))
    return out


def rotate_signed(x, blk: int, axis: int, signs) -> np.ndarray:
    """Random-sign rotation H (D x): each element times the +-1 sign of its
    position along the rotated dimension, then the block transform."""
    xb = _bf16_bits(x)
    sg = np.ascontiguousarray(signs, dtype=np.int8)
    n = xb.shape[1] if axis == 1 else xb.shape[0]
    if n % blk:
        # padded positions hold zeros, whose sign does not matter
        xb = pad_to_blocks(xb, blk, axis)
        sg = np.concatenate([sg[:n], np.ones(padded_length(n, blk) - n, dtype=np.int8)])
    rows, cols = xb.shape
    assert sg.shape == ((cols,) if axis == 1 else (rows,))
    out = np.empty((rows, cols), dtype=np.float64)
    lib = _load()
    if axis == 1:
        lib.halo_oracle_rotate_signed_along_cols(_ptr(xb), rows, cols, cols, blk, _ptr(sg), _ptr(out))
    else:
        lib.halo_oracle_rotate_signed_along_rows(_ptr(xb), rows, cols, cols, blk, _ptr(sg), _ptr(out))
    return out


def quantize_stochastic(v: np.ndarray, axis: int, qtype: int, rand_bits):
    """Stochastic-rounding quantiser: u = rand_bits / 65536 per element (uint16, layout of v)."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    rows, cols = v.shape
    rb = np.ascontiguousarray(rand_bits, dtype=np.uint16)
    assert rb.shape == v.shape
    codes = np.empty((rows, cols), dtype=np.uint8)
    scales = np.empty(rows if axis == 0 else cols, dtype=np.float32)
    t = np.empty((rows, cols), dtype=np.float64)
    _load().halo_oracle_quantize_stochastic(_ptr(v), rows, cols, axis, qtype, _ptr(rb), _ptr(codes), _ptr(scales),
                                            _ptr(t))
    return codes, scales, t


def quantize(v: np.ndarray, axis: int, qtype: int):
    """Symmetric absmax quantisation with one scale per row (axis=0) or per column (axis=1).

    Returns (codes uint8 [same shape], scales float32 [groups], t float64 [same shape]).
    INT8 codes are two's-complement bytes; E4M3 codes are OCP E4M3 bytes.
    """
    v = np.ascontiguousarray(v, dtype=np.float64)
    rows, cols = v.shape
    codes = np.empty((rows, cols), dtype=np.uint8)
    scales = np.empty(rows if axis == 0 else cols, dtype=np.float32)
    t = np.empty((rows, cols), dtype=np.float64)
    _load().halo_oracle_quantize(_ptr(v), rows, cols, axis, qtype, _ptr(codes), _ptr(scales), _ptr(t))
    return codes, scales, t


def quantize_grouped(v: np.ndarray, along: int, group: int, qtype: int):
    """Group-wise scales along the contraction dimension: along=1 groups of
    ``group`` consecutive elements of a row (scales [rows, cols/group]);
    along=0 groups of ``group`` consecutive rows of a column (scales
    [rows/group, cols]).  Returns (codes, scales, t)."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    rows, cols = v.shape
    assert (cols if along == 1 else rows) % group == 0
    codes = np.empty((rows, cols), dtype=np.uint8)
    shape = (rows, cols // group) if along == 1 else (rows // group, cols)
    scales = np.empty(shape, dtype=np.float32)
    t = np.empty((rows, cols), dtype=np.float64)
    _load().halo_oracle_quantize_grouped(_ptr(v), rows, cols, along, group, qtype, _ptr(codes), _ptr(scales),
                                         _ptr(t))
    return codes, scales, t


def gemm_grouped(a, sa, b, sb, group: int, qtype: int) -> np.ndarray:
    """y[i, j] = sum_G sa[i, G] sb[j, G] sum_{k in G} a[i, k] b[j, k]; codes
    [M, K] / [N, K] with the contraction dimension contiguous, scales [M, K/g] / [N, K/g]."""
    a = np.ascontiguousarray(a).view(np.uint8)
    b = np.ascontiguousarray(b).view(np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sb = np.ascontiguousarray(sb, dtype=np.float32)
    m, k = a.shape
    n, k2 = b.shape
    assert k == k2 and k % group == 0 and sa.shape == (m, k // group) and sb.shape == (n, k // group)
    y = np.empty((m, n), dtype=np.float64)
    _load().halo_oracle_gemm_grouped(_ptr(a), _ptr(sa), _ptr(b), _ptr(sb), m, n, k, group, qtype, _ptr(y))
    return y


def grouped_operand(x, blk: int, along: int, group: int, qtype: int):
    """Rotate (zero-padding as ``rotate``) and group-quantise one operand;
    returns its codes and scales with the contraction dimension last:
    ([outer, K], [outer, K/g]) whichever way the operand is stored."""
    v = rotate(x, blk, along)
    codes, scales, _ = quantize_grouped(v, along, group, qtype)
    if along == 0:
        codes, scales = codes.T, scales.T
    return np.ascontiguousarray(codes), np.ascontiguousarray(scales)


def linear_fwd_grouped(x, w, blk: int, group: int, qtype: int) -> np.ndarray:
    """Y = X W^T with both operands rotated along K and quantised with one
    scale per group of ``group`` consecutive K positions."""
    xa, sx = grouped_operand(x, blk, 1, group, qtype)
    wa, sw = grouped_operand(w, blk, 1, group, qtype)
    return gemm_grouped(xa, sx, wa, sw, group, qtype)


def linear_bwd_dx_grouped(dy, w, blk: int, group: int, qtype: int) -> np.ndarray:
    """dX = dY W: dY rotated along N (its rows), W along N (dimension 0), group-wise along N."""
    a, sa = grouped_operand(dy, blk, 1, group, qtype)
    b, sb = grouped_operand(w, blk, 0, group, qtype)
    return gemm_grouped(a, sa, b, sb, group, qtype)


def linear_bwd_dw_grouped(dy, x, blk: int, group: int, qtype: int) -> np.ndarray:
    """dW = dY^T X: both rotated along M (dimension 0), group-wise along M."""
    a, sa = grouped_operand(dy, blk, 0, group, qtype)
    b, sb = grouped_operand(x, blk, 0, group, qtype)
    return gemm_grouped(a, sa, b, sb, group, qtype)


def e4m3_encode(t) -> np.ndarray:
    flat = np.ascontiguousarray(np.asarray(t, dtype=np.float64).ravel())
    out = np.empty(flat.shape, dtype=np.uint8)
    _load().halo_oracle_e4m3_encode_array(_ptr(flat), flat.size, _ptr(out))
    return out.reshape(np.shape(t))


def e4m3_decode(codes) -> np.ndarray:
    flat = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8).ravel())
    out = np.empty(flat.shape, dtype=np.float64)
    _load().halo_oracle_e4m3_decode_array(_ptr(flat), flat.size, _ptr(out))
    return out.reshape(np.shape(codes))


def e4m3_decode_table() -> np.ndarray:
    return e4m3_decode(np.arange(256, dtype=np.uint8))


def boundary_distance(t: np.ndarray, qtype: int) -> np.ndarray:
    """Distance of each pre-rounding value to its nearest rounding midpoint, relative to |t|."""
    flat = np.ascontiguousarray(np.asarray(t, dtype=np.float64).ravel())
    out = np.empty(flat.shape, dtype=np.float64)
    _load().halo_oracle_boundary_distance_array(_ptr(flat), flat.size, qtype, _ptr(out))
    return out.reshape(np.shape(t))


def gemm_i8(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """C[i, j] = sum_k a[i, k] b[j, k] on int8 codes, exact int64 accumulation."""
    a = np.ascontiguousarray(a).view(np.int8)
    b = np.ascontiguousarray(b).view(np.int8)
    m, k = a.shape
    n, k2 = b.shape
    assert k == k2
    c = np.empty((m, n), dtype=np.int64)
    _load().halo_oracle_gemm_i8(_ptr(a), _ptr(b), m, n, k, _ptr(c))
    return c


def gemm_e4m3(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """C[i, j] = sum_k dec(a[i, k]) dec(b[j, k]) in fp64 on E4M3 codes."""
    a = np.ascontiguousarray(a).view(np.uint8)
    b = np.ascontiguousarray(b).view(np.uint8)
    m, k = a.shape
    n, k2 = b.shape
    assert k == k2
    c = np.empty((m, n), dtype=np.float64)
    _load().halo_oracle_gemm_e4m3(_ptr(a), _ptr(b), m, n, k, _ptr(c))
    return c


def dequant(acc: np.ndarray, sa: np.ndarray, sb: np.ndarray) -> np.ndarray:
    acc = np.ascontiguousarray(acc, dtype=np.float64)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sb = np.ascontiguousarray(sb, dtype=np.float32)
    m, n = acc.shape
    y = np.empty((m, n), dtype=np.float64)
    _load().halo_oracle_dequant(_ptr(acc), _ptr(sa), _ptr(sb), m, n, _ptr(y))
    return y


def linear_fwd(x, w, blk: int, qtype: int) -> np.ndarray:
    """Y[M, N] = X W^T with both operands rotated along K and quantised per row
    (K not a multiple of blk: both zero-padded along K first)."""
    xb, wb = _bf16_bits(x), _bf16_bits(w)
    if xb.shape[1] % blk:
        xb, wb = pad_to_blocks(xb, blk, 1), pad_to_blocks(wb, blk, 1)
    m, k = xb.shape
    n, _ = wb.shape
    y = np.empty((m, n), dtype=np.float64)
    _load().halo_oracle_linear_fwd(_ptr(xb), _ptr(wb), m, n, k, blk, qtype, _ptr(y))
    return y


def linear_bwd_dx(dy, w, blk: int, qtype: int) -> np.ndarray:
    """dX[M, K] = dY W with both operands rotated along N (N not a multiple of
    blk: dY's columns and W's rows zero-padded first)."""
    dyb, wb = _bf16_bits(dy), _bf16_bits(w)
    if dyb.shape[1] % blk:
        dyb, wb = pad_to_blocks(dyb, blk, 1), pad_to_blocks(wb, blk, 0)
    m, n = dyb.shape
    _, k = wb.shape
    dx = np.empty((m, k), dtype=np.float64)
    _load().halo_oracle_linear_bwd_dx(_ptr(dyb), _ptr(wb), m, n, k, blk, qtype, _ptr(dx))
    return dx


def linear_bwd_dw(dy, x, blk: int, qtype: int) -> np.ndarray:
    """dW[N, K] = dY^T X with both operands rotated along M (tokens; M not a
    multiple of blk: the rows of both zero-padded first)."""
    dyb, xb = _bf16_bits(dy), _bf16_bits(x)
    if dyb.shape[0] % blk:
        dyb, xb = pad_to_blocks(dyb, blk, 0), pad_to_blocks(xb, blk, 0)
    m, n = dyb.shape
    _, k = xb.shape
    dw = np.empty((n, k), dtype=np.float64)
    _load().halo_oracle_linear_bwd_dw(_ptr(dyb), _ptr(xb), m, n, k, blk, qtype, _ptr(dw))
    return dw


def rotated_qgemm_parts(a, a_kdim_contig: bool, b, b_kdim_contig: bool, blk: int, qtype: int):
    """Rotate+quantise both operands of one GEMM and return (A codes [M,K], sa, B codes [N,K], sb).

    ``a`` is A[M, K] when ``a_kdim_contig`` else A^T stored [K, M]; same for ``b``.
    """
    out = []
    for x, contig in ((a, a_kdim_contig), (b, b_kdim_contig)):
        if contig:
            v = rotate(x, blk, axis=1)
            codes, s, _ = quantize(v, axis=0, qtype=qtype)
            out += [codes, s]
        else:
            v = rotate(x, blk, axis=0)
            codes, s, _ = quantize(v, axis=1, qtype=qtype)
            out += [np.ascontiguousarray(codes.T), s]
    return tuple(out)
