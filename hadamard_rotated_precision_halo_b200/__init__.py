"""B200 (sm_100a) Hadamard-rotated quantized linear layer (HALO, arXiv 2501.02625).

Thin Python binding over the C ABI in ``include/halo.h`` (``libhalo.so``, built
in-tree by ``build.py``).  The functions carry the C names; they only marshal
torch tensors into device pointers, allocate outputs with torch and pass the
current CUDA stream.  Every step of the computation runs in the library's
CUDA kernels; there is no other path, and calling without the built library
raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhalo.so")

HALO_OK = 0
HALO_ERR_NULL = 1
HALO_ERR_SHAPE = 2
HALO_ERR_BLOCK = 3
HALO_ERR_ALIGN = 4
HALO_ERR_DTYPE = 5
HALO_ERR_WORKSPACE = 6
HALO_ERR_CUDA = 7
HALO_ERR_TIMEOUT = 8
HALO_ERR_UNSUPPORTED = 9

HALO_Q_INT8 = 0
HALO_Q_E4M3 = 1
HALO_OUT_FP32 = 0
HALO_OUT_BF16 = 1
HALO_AXIS_COLS = 0
HALO_AXIS_ROWS = 1
HALO_MAJOR_K = 0
HALO_MAJOR_MN = 1

EXPORTS = (
    "halo_hadamard_quantize",
    "halo_hadamard_quantize_ex",
    "halo_hadamard_quantize_dual",
    "halo_hadamard_quantize_grouped",
    "halo_qgemm_grouped",
    "halo_workspace_size_grouped",
    "halo_linear_fwd_grouped",
    "halo_linear_bwd_grouped",
    "halo_qgemm",
    "halo_workspace_size",
    "halo_linear_fwd",
    "halo_linear_bwd",
    "halo_linear_fwd_noalloc",
    "halo_hadamard_colmax",
    "halo_hadamard_quantize_both",
    "halo_hadamard_quantize_colmax",
    "halo_status_string",
    "halo_device_error",
    "halo_selftest_wait_timeout",
    "halo_last_cuda_error",
    "halo_last_error_detail",
)

_lib = None


class HaloError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = status_text(status)
        if status == HALO_ERR_CUDA and _lib is not None:
            msg += f" (cuda error {_lib.halo_last_cuda_error()}: {_lib.halo_last_error_detail().decode()})"
        super().__init__(f"{what}: {msg}" if what else msg)


def lib():
    """Load ``libhalo.so`` (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m hadamard_rotated_precision_halo_b200.build` "
            "or `__graft_entry__.build()`; there is no fallback path"
        )
    L = ctypes.CDLL(LIB_PATH)
    P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    L.halo_hadamard_quantize.argtypes = [P, I64, I64, I64, I, I, I, P, I64, P, P]
    L.halo_hadamard_quantize.restype = I
    L.halo_hadamard_quantize_ex.argtypes = [P, I64, I64, I64, I, I, I, P, P, I64, P, I64, P, P]
    L.halo_hadamard_quantize_ex.restype = I
    L.halo_hadamard_quantize_dual.argtypes = [P, I64, I64, I64, I, P, I64, P, P, I64, P, P]
    L.halo_hadamard_quantize_dual.restype = I
    L.halo_hadamard_quantize_grouped.argtypes = [P, I64, I64, I64, I, I, I, I, P, I64, P, P]
    L.halo_hadamard_quantize_grouped.restype = I
    L.halo_qgemm_grouped.argtypes = [P, P, I, I64, P, P, I, I64, I64, I64, I64, I, I, P, I, I64, P]
    L.halo_qgemm_grouped.restype = I
    L.halo_workspace_size_grouped.argtypes = [I64, I64, I64, I, I]
    L.halo_workspace_size_grouped.restype = SZ
    L.halo_linear_fwd_grouped.argtypes = [P, P, I64, I64, I64, I, I, I, P, I, P, SZ, P]
    L.halo_linear_fwd_grouped.restype = I
    L.halo_linear_bwd_grouped.argtypes = [P, P, P, I64, I64, I64, I, I, I, P, I, P, I, P, SZ, P]
    L.halo_linear_bwd_grouped.restype = I
    L.halo_selftest_wait_timeout.argtypes = [I64, P]
    L.halo_selftest_wait_timeout.restype = I
    L.halo_qgemm.argtypes = [P, P, I, I64, P, P, I, I64, I64, I64, I64, I, P, I, I64, P]
    L.halo_qgemm.restype = I
    L.halo_workspace_size.argtypes = [I64, I64, I64, I]
    L.halo_workspace_size.restype = SZ
    L.halo_linear_fwd.argtypes = [P, P, I64, I64, I64, I, I, P, I, P, SZ, P]
    L.halo_linear_fwd.restype = I
    L.halo_linear_bwd.argtypes = [P, P, P, I64, I64, I64, I, I, P, I, P, I, P, SZ, P]
    L.halo_linear_bwd.restype = I
    L.halo_linear_fwd_noalloc.argtypes = [P, P, I64, I64, I64, I, I, P, I, P]
    L.halo_linear_fwd_noalloc.restype = I
    L.halo_hadamard_quantize_both.argtypes = [P, I64, I64, I64, I, I, P, I64, P, P, I64, P, P]
    L.halo_hadamard_quantize_both.restype = I
    L.halo_hadamard_colmax.argtypes = [P, I64, I64, I64, I, P, P]
    L.halo_hadamard_colmax.restype = I
    L.halo_hadamard_quantize_colmax.argtypes = [P, I64, I64, I64, I, I, P, P, I64, P, P]
    L.halo_hadamard_quantize_colmax.restype = I
    L.halo_status_string.argtypes = [I]
    L.halo_status_string.restype = ctypes.c_char_p
    L.halo_device_error.argtypes = [ctypes.POINTER(ctypes.c_int)]
    L.halo_device_error.restype = I
    L.halo_last_cuda_error.argtypes = []
    L.halo_last_cuda_error.restype = I
    L.halo_last_error_detail.argtypes = []
    L.halo_last_error_detail.restype = ctypes.c_char_p
    _lib = L
    return L


def status_text(status: int) -> str:
    return lib().halo_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != HALO_OK:
        raise HaloError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _code_dtype(qtype: int):
    return torch.int8 if qtype == HALO_Q_INT8 else torch.float8_e4m3fn


def _out_dtype(otype: int):
    return torch.float32 if otype == HALO_OUT_FP32 else torch.bfloat16


def padded_length(n: int, blk: int) -> int:
    """A rotated dimension of n elements, zero-padded to whole blocks."""
    return -(-n // blk) * blk


def codes_shape(rows: int, cols: int, axis: int, blk: int):
    """Shape of the codes: the rotated dimension zero-padded to whole blocks
    (blocks of 128 rows along dimension 0)."""
    if axis == HALO_AXIS_COLS:
        return rows, padded_length(cols, blk)
    return padded_length(rows, 128), cols


def halo_hadamard_quantize(x: torch.Tensor, axis: int, blk: int, qtype: int, q_out=None, scales_out=None,
                           stream=None):
    """Rotate + quantise a bf16 [rows, cols] matrix; returns (codes, scales).

    axis HALO_AXIS_COLS: blocks along each row, one scale per row.
    axis HALO_AXIS_ROWS: blocks along dimension 0, one scale per column.
    The codes cover the rotated dimension zero-padded to whole blocks.
    """
    rows, cols = x.shape
    if q_out is None:
        q_out = torch.empty(codes_shape(rows, cols, axis, blk), dtype=_code_dtype(qtype), device=x.device)
    if scales_out is None:
        scales_out = torch.empty(rows if axis == HALO_AXIS_COLS else cols, dtype=torch.float32, device=x.device)
    st = lib().halo_hadamard_quantize(_ptr(x), rows, cols, x.stride(0), axis, blk, qtype, _ptr(q_out),
                                      q_out.stride(0), _ptr(scales_out), _stream(stream))
    _check(st, "halo_hadamard_quantize")
    return q_out, scales_out


def halo_hadamard_quantize_ex(x: torch.Tensor, axis: int, blk: int, qtype: int, signs=None, rand_bits=None,
                              q_out=None, scales_out=None, stream=None):
    """halo_hadamard_quantize with optional +-1 signs along the rotated dimension
    (int8 tensor) and optional per-element random bits for stochastic rounding
    (uint16 stored as int16/uint16 tensor of x's shape)."""
    rows, cols = x.shape
    if q_out is None:
        q_out = torch.empty(codes_shape(rows, cols, axis, blk), dtype=_code_dtype(qtype), device=x.device)
    if scales_out is None:
        scales_out = torch.empty(rows if axis == HALO_AXIS_COLS else cols, dtype=torch.float32, device=x.device)
    ld_rand = rand_bits.stride(0) if rand_bits is not None else 0
    st = lib().halo_hadamard_quantize_ex(_ptr(x), rows, cols, x.stride(0), axis, blk, qtype, _ptr(signs),
                                         _ptr(rand_bits), ld_rand, _ptr(q_out), q_out.stride(0), _ptr(scales_out),
                                         _stream(stream))
    _check(st, "halo_hadamard_quantize_ex")
    return q_out, scales_out


def halo_hadamard_quantize_both(x: torch.Tensor, blk: int, qtype: int, outs=None, stream=None):
    """Both code sets of x, rotated along the contiguous dimension (per-row
    scales) and along dimension 0 (per-column scales), the second rotation
    reading x from L2; returns (q_rows, scales_rows, q_cols, scales_cols)."""
    rows, cols = x.shape
    if outs is None:
        outs = (torch.empty(codes_shape(rows, cols, HALO_AXIS_COLS, blk), dtype=_code_dtype(qtype), device=x.device),
                torch.empty(rows, dtype=torch.float32, device=x.device),
                torch.empty(codes_shape(rows, cols, HALO_AXIS_ROWS, 128), dtype=_code_dtype(qtype), device=x.device),
                torch.empty(cols, dtype=torch.float32, device=x.device))
    qr, sr, qc, sc = outs
    _check(lib().halo_hadamard_quantize_both(_ptr(x), rows, cols, x.stride(0), blk, qtype, _ptr(qr), qr.stride(0),
                                             _ptr(sr), _ptr(qc), qc.stride(0), _ptr(sc), _stream(stream)),
           "halo_hadamard_quantize_both")
    return outs


def halo_hadamard_colmax(x: torch.Tensor, blk: int = 128, amax_out=None, stream=None) -> torch.Tensor:
    """Per-column maxima of |H_128 x| (unnormalised block transform along
    dimension 0) over the rows of x: fp32 [cols]."""
    rows, cols = x.shape
    if amax_out is None:
        amax_out = torch.empty(cols, dtype=torch.float32, device=x.device)
    _check(lib().halo_hadamard_colmax(_ptr(x), rows, cols, x.stride(0), blk, _ptr(amax_out), _stream(stream)),
           "halo_hadamard_colmax")
    return amax_out


def halo_hadamard_quantize_colmax(x: torch.Tensor, blk: int, qtype: int, amax: torch.Tensor, q_out=None,
                                  scales_out=None, stream=None):
    """Codes and scales of x rotated along dimension 0 with given per-column
    maxima (halo_hadamard_colmax merged over every holder of x's rows)."""
    rows, cols = x.shape
    shape = codes_shape(rows, cols, HALO_AXIS_ROWS, blk)
    if q_out is None:
        q_out = torch.empty(shape, dtype=_code_dtype(qtype), device=x.device)
    if scales_out is None:
        scales_out = torch.empty(cols, dtype=torch.float32, device=x.device)
    _check(lib().halo_hadamard_quantize_colmax(_ptr(x), rows, cols, x.stride(0), blk, qtype, _ptr(amax), _ptr(q_out),
                                               q_out.stride(0), _ptr(scales_out), _stream(stream)),
           "halo_hadamard_quantize_colmax")
    return q_out, scales_out


def halo_hadamard_quantize_dual(x: torch.Tensor, blk: int, q_int8=None, scales_int8=None, q_e4m3=None,
                                scales_e4m3=None, stream=None):
    """Rotate along the contiguous dim once, quantise to INT8 and to E4M3;
    returns (int8 codes, int8 scales, e4m3 codes, e4m3 scales)."""
    rows, cols = x.shape
    shape = codes_shape(rows, cols, HALO_AXIS_COLS, blk)
    if q_int8 is None:
        q_int8 = torch.empty(shape, dtype=_code_dtype(HALO_Q_INT8), device=x.device)
    if q_e4m3 is None:
        q_e4m3 = torch.empty(shape, dtype=_code_dtype(HALO_Q_E4M3), device=x.device)
    if scales_int8 is None:
        scales_int8 = torch.empty(rows, dtype=torch.float32, device=x.device)
    if scales_e4m3 is None:
        scales_e4m3 = torch.empty(rows, dtype=torch.float32, device=x.device)
    st = lib().halo_hadamard_quantize_dual(_ptr(x), rows, cols, x.stride(0), blk, _ptr(q_int8), q_int8.stride(0),
                                           _ptr(scales_int8), _ptr(q_e4m3), q_e4m3.stride(0), _ptr(scales_e4m3),
                                           _stream(stream))
    _check(st, "halo_hadamard_quantize_dual")
    return q_int8, scales_int8, q_e4m3, scales_e4m3


def halo_hadamard_quantize_grouped(x: torch.Tensor, axis: int, blk: int, group: int, qtype: int, q_out=None,
                                   scales_out=None, stream=None):
    """Rotate + quantise with one scale per `group` positions along the rotated
    dimension; returns (codes, scales) with scales [rows, cols_p/group]
    (HALO_AXIS_COLS) or [rows_p/group, cols] (HALO_AXIS_ROWS)."""
    rows, cols = x.shape
    shape = codes_shape(rows, cols, axis, blk)
    if q_out is None:
        q_out = torch.empty(shape, dtype=_code_dtype(qtype), device=x.device)
    if scales_out is None:
        sshape = (rows, shape[1] // group) if axis == HALO_AXIS_COLS else (shape[0] // group, cols)
        scales_out = torch.empty(sshape, dtype=torch.float32, device=x.device)
    st = lib().halo_hadamard_quantize_grouped(_ptr(x), rows, cols, x.stride(0), axis, blk, group, qtype, _ptr(q_out),
                                              q_out.stride(0), _ptr(scales_out), _stream(stream))
    _check(st, "halo_hadamard_quantize_grouped")
    return q_out, scales_out


def halo_qgemm_grouped(a_q, s_a, a_major, b_q, s_b, b_major, m, n, k, group, qtype, otype, c=None, stream=None):
    """C[m, n] = sum_G s_a[., G] s_b[., G] (A_G B_G^T) on 8-bit codes with group-wise scales."""
    if c is None:
        c = torch.empty((m, n), dtype=_out_dtype(otype), device=a_q.device)
    st = lib().halo_qgemm_grouped(_ptr(a_q), _ptr(s_a), a_major, a_q.stride(0), _ptr(b_q), _ptr(s_b), b_major,
                                  b_q.stride(0), m, n, k, group, qtype, _ptr(c), otype, c.stride(0), _stream(stream))
    _check(st, "halo_qgemm_grouped")
    return c


def halo_linear_fwd_grouped(x, w, blk, group, qtype, otype, y=None, ws=None, stream=None):
    m, k = x.shape
    n = w.shape[0]
    if y is None:
        y = torch.empty((m, n), dtype=_out_dtype(otype), device=x.device)
    if ws is None:
        ws = torch.empty(int(lib().halo_workspace_size_grouped(m, n, k, group, 0)), dtype=torch.uint8, device=x.device)
    st = lib().halo_linear_fwd_grouped(_ptr(x), _ptr(w), m, n, k, blk, group, qtype, _ptr(y), otype, _ptr(ws),
                                       ws.numel(), _stream(stream))
    _check(st, "halo_linear_fwd_grouped")
    return y


def halo_linear_bwd_grouped(dy, x, w, blk, group, qtype, otype_dx, otype_dw, dx=None, dw=None, want_dx=True,
                            want_dw=True, ws=None, stream=None):
    m, n = dy.shape
    k = (x if x is not None else w).shape[1]
    dev = dy.device
    if want_dx and dx is None:
        dx = torch.empty((m, k), dtype=_out_dtype(otype_dx), device=dev)
    if want_dw and dw is None:
        dw = torch.empty((n, k), dtype=_out_dtype(otype_dw), device=dev)
    if ws is None:
        ws = torch.empty(int(lib().halo_workspace_size_grouped(m, n, k, group, 1)), dtype=torch.uint8, device=dev)
    st = lib().halo_linear_bwd_grouped(_ptr(dy), _ptr(x), _ptr(w), m, n, k, blk, group, qtype,
                                       _ptr(dx if want_dx else None), otype_dx, _ptr(dw if want_dw else None),
                                       otype_dw, _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "halo_linear_bwd_grouped")
    return dx, dw


def halo_qgemm(a_q, s_a, a_major, b_q, s_b, b_major, m, n, k, qtype, otype, c=None, stream=None):
    """C[m, n] = (A B^T) * s_a[:, None] * s_b[None, :] on 8-bit codes."""
    if c is None:
        c = torch.empty((m, n), dtype=_out_dtype(otype), device=a_q.device)
    st = lib().halo_qgemm(_ptr(a_q), _ptr(s_a), a_major, a_q.stride(0), _ptr(b_q), _ptr(s_b), b_major,
                          b_q.stride(0), m, n, k, qtype, _ptr(c), otype, c.stride(0), _stream(stream))
    _check(st, "halo_qgemm")
    return c


def halo_workspace_size(m: int, n: int, k: int, which: int) -> int:
    return int(lib().halo_workspace_size(m, n, k, which))


def workspace(m: int, n: int, k: int, which: int, device) -> torch.Tensor:
    return torch.empty(halo_workspace_size(m, n, k, which), dtype=torch.uint8, device=device)


def halo_linear_fwd(x, w, blk, qtype, otype, y=None, ws=None, stream=None):
    """Y = X W^T with both operands Hadamard-rotated along K and quantised."""
    m, k = x.shape
    n = w.shape[0]
    if y is None:
        y = torch.empty((m, n), dtype=_out_dtype(otype), device=x.device)
    if ws is None:
        ws = workspace(m, n, k, 0, x.device)
    st = lib().halo_linear_fwd(_ptr(x), _ptr(w), m, n, k, blk, qtype, _ptr(y), otype, _ptr(ws), ws.numel(),
                               _stream(stream))
    _check(st, "halo_linear_fwd")
    return y


def halo_linear_bwd(dy, x, w, blk, qtype, otype_dx, otype_dw, dx=None, dw=None, want_dx=True, want_dw=True,
                    ws=None, stream=None):
    """(dX, dW) for Y = X W^T; either may be skipped."""
    m, n = dy.shape
    k = (x if x is not None else w).shape[1]
    dev = dy.device
    if want_dx and dx is None:
        dx = torch.empty((m, k), dtype=_out_dtype(otype_dx), device=dev)
    if want_dw and dw is None:
        dw = torch.empty((n, k), dtype=_out_dtype(otype_dw), device=dev)
    if ws is None:
        ws = workspace(m, n, k, 1, dev)
    st = lib().halo_linear_bwd(_ptr(dy), _ptr(x), _ptr(w), m, n, k, blk, qtype, _ptr(dx if want_dx else None),
                               otype_dx, _ptr(dw if want_dw else None), otype_dw, _ptr(ws), ws.numel(),
                               _stream(stream))
    _check(st, "halo_linear_bwd")
    return dx, dw


def halo_device_error():
    """(status, site): synchronises and reports/clears a kernel's bounded-wait error."""
    where = ctypes.c_int(0)
    st = lib().halo_device_error(ctypes.byref(where))
    return st, where.value
