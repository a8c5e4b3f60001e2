"""halo_linear_fwd_noalloc: the forward linear layer for callers that cannot
allocate device memory (for instance a plugin whose host interface hands it
only input and output pointers, or a loop that must not call cudaMalloc
because it can synchronise the device).  Its scratch is a fixed array inside
the library, so the call takes X, W and Y only.

This file is collected last on purpose.  Its test must give the same result as
the workspace entry point, on two calls in a row (the shared array keeps the
previous call's contents), both in a fresh process and after every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import hadamard_rotated_precision_halo_b200 as halo
from hadamard_rotated_precision_halo_b200 import inputs
import oracle
from tests._parity import check_codes, check_output, oracle_operand

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 64 << 20  # HALO_NOALLOC_SCRATCH_BYTES in include/halo.h


def _call(lib, x, w, y, blk, qtype, otype):
    m, k = x.shape
    n = w.shape[0]
    return lib.halo_linear_fwd_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(w.data_ptr()), m, n, k, blk,
                                       qtype, ctypes.c_void_p(y.data_ptr()), otype,
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("qtype,otype", [(halo.HALO_Q_INT8, halo.HALO_OUT_FP32),
                                         (halo.HALO_Q_E4M3, halo.HALO_OUT_BF16)])
def test_noalloc_forward_matches_workspace_forward(qtype, otype):
    lib = halo.lib()
    m, n, k, blk = 1024, 768, 2048, 128
    assert lib.halo_workspace_size(m, n, k, 0) <= SCRATCH_BYTES
    x = inputs.activations(m, k, seed=61, device="cuda")
    w = inputs.weights(n, k, seed=62, device="cuda")
    ref = halo.halo_linear_fwd(x, w, blk, qtype, otype)  # the existing entry point, caller workspace
    torch.cuda.synchronize()
    out_dtype = torch.float32 if otype == halo.HALO_OUT_FP32 else torch.bfloat16
    for _ in range(2):  # the second call finds the first call's codes still in the array
        y = torch.full((m, n), float("nan"), dtype=out_dtype, device="cuda")
        st = _call(lib, x, w, y, blk, qtype, otype)
        assert st == halo.HALO_OK, halo.status_text(st)
        torch.cuda.synchronize()
        # the same kernels on the same inputs: bit for bit the workspace call's output
        assert torch.equal(y, ref)
    # and the oracle's arithmetic: the operands' codes (the same kernels write
    # them) checked against the oracle's, then the oracle's GEMM and
    # dequantisation on those codes.  (Against the oracle's own codes the bound
    # would have to allow for the codes the band exempts: on these outlier
    # inputs one E4M3 step of a large code moves Y by up to a few 1e-3.)
    codes = []
    for t in (x, w):
        q, s = halo.halo_hadamard_quantize(t, halo.HALO_AXIS_COLS, blk, qtype)
        torch.cuda.synchronize()
        c, sc, tt = oracle_operand(t.cpu(), 1, blk, qtype)
        check_codes(q, s, c, sc, tt, qtype, blk=blk, axis=1)
        codes.append((q.view(torch.uint8).cpu().numpy(), s.cpu().numpy()))
    (cx, sx), (cw, sw) = codes
    acc = oracle.gemm_i8(cx, cw).astype(np.float64) if qtype == halo.HALO_Q_INT8 else oracle.gemm_e4m3(cx, cw)
    check_output(y, oracle.dequant(acc, sx, sw), rel=1e-5)
    st, site = halo.halo_device_error()
    assert st == halo.HALO_OK, f"bounded wait ran out at site {site:#x}"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = halo.lib()
    m, n, k = 8192, 8192, 4096  # 64 MiB of codes alone, plus scales
    assert lib.halo_workspace_size(m, n, k, 0) > SCRATCH_BYTES
    x = torch.empty((16, 16), dtype=torch.bfloat16, device="cuda")  # never read: rejected before any launch
    st = lib.halo_linear_fwd_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(x.data_ptr()), m, n, k, 128,
                                     halo.HALO_Q_INT8, ctypes.c_void_p(x.data_ptr()), halo.HALO_OUT_FP32, None)
    assert st == halo.HALO_ERR_WORKSPACE
    assert b"scratch" in lib.halo_last_error_detail()


def test_noalloc_rejects_misaligned_pointers_before_touching_the_device():
    lib = halo.lib()
    buf = torch.zeros(4096, dtype=torch.bfloat16, device="cuda")
    p = buf.data_ptr()
    st = lib.halo_linear_fwd_noalloc(ctypes.c_void_p(p + 2), ctypes.c_void_p(p), 16, 16, 128, 128,
                                     halo.HALO_Q_INT8, ctypes.c_void_p(p), halo.HALO_OUT_FP32, None)
    assert st == halo.HALO_ERR_ALIGN
    st = lib.halo_linear_fwd_noalloc(ctypes.c_void_p(p), ctypes.c_void_p(p), 16, 6, 128, 128, halo.HALO_Q_INT8,
                                     ctypes.c_void_p(p), halo.HALO_OUT_BF16, None)  # a 12-byte output row
    assert st == halo.HALO_ERR_ALIGN
    assert torch.all(buf == 0)
