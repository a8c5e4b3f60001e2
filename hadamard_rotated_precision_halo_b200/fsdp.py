"""Fully sharded data parallelism for the rotated quantised linear layer, with
8-bit communication (HALO paper page, "technical framework": FSDP integration
with low-precision communication).

Every rank of the process group holds its own tokens -- X_r [M_r, K] and, in
the backward pass, dY_r [M_r, N] -- and one shard of the weight: rows
[r N/P, (r + 1) N/P) of W [N, K], with N/P a multiple of 128 so that no
128-row rotation block straddles two shards.

forward, Y_r = X_r W^T
    Each rank rotates its weight rows along K and quantises them per row (a
    row's scale needs nothing from other ranks); the 1-byte codes and the fp32
    row scales are all-gathered, giving every rank the codes of the whole W.
    X_r is rotated and quantised locally and multiplied with them.  The result
    is the single-device result, bit for bit.
dX_r = dY_r W (contraction over N, which the shards split)
    W is rotated along N (dimension 0) with one scale per column over all N
    rows: each rank computes its rows' column maxima, one all-reduce(max) of a
    K-vector merges them, each rank quantises its rows with the merged maxima
    and the codes are all-gathered.  Also the single-device result, bit for bit.
dW = sum_r dY_r^T X_r (contraction over the tokens, which the ranks split)
    Each rank rotates its own dY_r and X_r along its tokens (one scale per
    column over its own tokens) and multiplies; the fp32 partial products are
    reduce-scattered (summed) so that rank r receives the rows of its shard.

Communication per rank and step: the weight codes twice (1 B per element,
half the bf16 weight), N + K fp32 scales and a K-vector of maxima, and the
fp32 dW reduce-scatter.  Gathered codes land in local buffers before any
kernel reads them: no kernel reads another device's memory.

The compute steps go through `ops` (default: this library's CUDA kernels,
CudaOps); the collectives through torch.distributed (NCCL on GPUs).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

BLK = 128


class CudaOps:
    """The compute steps on this library's kernels (device tensors)."""

    def __init__(self):
        import hadamard_rotated_precision_halo_b200 as halo

        self.h = halo

    def quantize_rows(self, x, qtype):
        """Rotate along the contiguous dimension, one scale per row."""
        return self.h.halo_hadamard_quantize(x, self.h.HALO_AXIS_COLS, BLK, qtype)

    def quantize_cols(self, x, qtype):
        """Rotate along dimension 0, one scale per column over x's rows."""
        return self.h.halo_hadamard_quantize(x, self.h.HALO_AXIS_ROWS, BLK, qtype)

    def colmax(self, x):
        return self.h.halo_hadamard_colmax(x, BLK)

    def quantize_cols_given(self, x, qtype, amax):
        return self.h.halo_hadamard_quantize_colmax(x, BLK, qtype, amax)

    def gemm(self, a, sa, a_kmajor, b, sb, b_kmajor, m, n, k, qtype, out_fp32):
        h = self.h
        return h.halo_qgemm(a, sa, h.HALO_MAJOR_K if a_kmajor else h.HALO_MAJOR_MN, b, sb,
                            h.HALO_MAJOR_K if b_kmajor else h.HALO_MAJOR_MN, m, n, k, qtype,
                            h.HALO_OUT_FP32 if out_fp32 else h.HALO_OUT_BF16)


def _world(group):
    if not dist.is_available() or not dist.is_initialized():
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def _all_gather_rows(t: torch.Tensor, world: int, group) -> torch.Tensor:
    """Concatenate every rank's t along dimension 0 (1-byte codes travel as
    uint8, whatever their type)."""
    if world == 1:
        return t
    raw = t.contiguous().view(torch.uint8) if t.element_size() == 1 else t.contiguous()
    out = torch.empty((world * raw.shape[0],) + tuple(raw.shape[1:]), dtype=raw.dtype, device=raw.device)
    dist.all_gather_into_tensor(out, raw, group=group)
    return out.view(t.dtype) if t.element_size() == 1 else out


class ShardedLinear:
    """One linear layer Y = X W^T with W sharded by rows over the process group.

    w_shard: this rank's rows of W [N/P, K] (bf16; N/P % 128 == 0, K % 128 == 0).
    qtype: 0 INT8, 1 E4M3.  ops: the compute steps (CudaOps by default)."""

    def __init__(self, w_shard: torch.Tensor, qtype: int = 0, group=None, ops=None):
        self.world, self.rank = _world(group)
        self.group = group
        self.w = w_shard
        self.qtype = qtype
        self.ops = ops if ops is not None else CudaOps()
        rows, self.k = w_shard.shape
        if rows % BLK or self.k % BLK:
            raise ValueError(f"weight shard rows ({rows}) and K ({self.k}) must be multiples of {BLK}")
        self.n = rows * self.world

    # ------------------------------------------------------------------ forward
    def gather_weight_codes_rows(self):
        """Codes and scales of the whole W rotated along K, from every rank's shard."""
        q, s = self.ops.quantize_rows(self.w, self.qtype)
        return _all_gather_rows(q, self.world, self.group), _all_gather_rows(s, self.world, self.group)

    def forward(self, x: torch.Tensor, out_fp32: bool = False) -> torch.Tensor:
        m = x.shape[0]
        wq, ws = self.gather_weight_codes_rows()
        xq, xs = self.ops.quantize_rows(x, self.qtype)
        return self.ops.gemm(xq, xs, True, wq, ws, True, m, self.n, self.k, self.qtype, out_fp32)

    # ----------------------------------------------------------------- backward
    def gather_weight_codes_cols(self):
        """Codes [N, K] and column scales [K] of the whole W rotated along N:
        the column maxima merged over the ranks, then each shard quantised."""
        amax = self.ops.colmax(self.w)
        if self.world > 1:
            dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=self.group)
        q, s = self.ops.quantize_cols_given(self.w, self.qtype, amax)
        return _all_gather_rows(q, self.world, self.group), s

    def backward(self, dy: torch.Tensor, x: torch.Tensor, dx_fp32: bool = False):
        """(dX_r [M_r, K], dW shard [N/P, K] fp32) for this rank's tokens."""
        m = dy.shape[0]
        # dX_r = dY_r W: dY_r rotated along N (per row), W along N (per column).
        wq, ws = self.gather_weight_codes_cols()
        dyq, dys = self.ops.quantize_rows(dy, self.qtype)
        dx = self.ops.gemm(dyq, dys, True, wq, ws, False, m, self.k, self.n, self.qtype, dx_fp32)
        # dW partial = dY_r^T X_r, both rotated along this rank's tokens.
        dyc, dycs = self.ops.quantize_cols(dy, self.qtype)
        xc, xcs = self.ops.quantize_cols(x, self.qtype)
        mp = dyc.shape[0]  # tokens zero-padded to whole blocks
        dw_full = self.ops.gemm(dyc, dycs, False, xc, xcs, False, self.n, self.k, mp, self.qtype, True)
        if self.world == 1:
            return dx, dw_full
        dw = torch.empty((self.n // self.world, self.k), dtype=dw_full.dtype, device=dw_full.device)
        dist.reduce_scatter_tensor(dw, dw_full.contiguous(), op=dist.ReduceOp.SUM, group=self.group)
        return dx, dw
