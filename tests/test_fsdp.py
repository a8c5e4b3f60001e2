"""Fully sharded data parallelism with 8-bit communication (fsdp.ShardedLinear).

CPU: two gloo ranks run the sharded layer's collectives -- weight codes and
scales all-gathered, column maxima all-reduced, dW reduce-scattered -- with the
oracle doing the compute steps (OracleOps below, test infrastructure), and the
results are compared with the oracle's single-device products:
  Y_r  = oracle linear_fwd(X_r, W)           (bit for bit)
  dX_r = oracle linear_bwd_dx(dY_r, W)       (bit for bit)
  dW   = sum_r oracle linear_bwd_dw(dY_r, X_r), rows of this rank's shard.
GPU: one process, the same layer on the CUDA ops equals the single-device
entry points bit for bit, and the split dimension-0 calls reproduce the
unsplit codes when the rows are cut into two shards.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

N, K, M_R = 512, 384, 192  # two shards of 256 weight rows; 192 tokens per rank (padded to 256 for dW)


class OracleOps:
    """The compute steps of ShardedLinear on the CPU oracle (tests only).
    Codes travel as uint8 tensors, scales and products as float64."""

    def __init__(self):
        import oracle

        self.o = oracle

    def _pair(self, codes, scales):
        return torch.from_numpy(np.ascontiguousarray(codes)), torch.from_numpy(np.asarray(scales, dtype=np.float64))

    def quantize_rows(self, x, qtype):
        codes, scales, _ = self.o.quantize(self.o.rotate(x, 128, 1), 0, qtype)
        return self._pair(codes, scales)

    def quantize_cols(self, x, qtype):
        codes, scales, _ = self.o.quantize(self.o.rotate(x, 128, 0), 1, qtype)
        return self._pair(codes, scales)

    def colmax(self, x):
        v = self.o.rotate(x, 128, 0)
        return torch.from_numpy(np.abs(v).max(axis=0))

    def quantize_cols_given(self, x, qtype, amax):
        # The oracle's own quantiser on the shard's rotated rows plus one row
        # holding the merged maxima: every column's maximum is then the merged
        # one, and the shard's codes are those of the whole matrix.
        v = self.o.rotate(x, 128, 0)
        codes, scales, _ = self.o.quantize(np.vstack([v, amax.numpy()[None, :]]), 1, qtype)
        return self._pair(codes[:-1], scales)

    def gemm(self, a, sa, a_kmajor, b, sb, b_kmajor, m, n, k, qtype, out_fp32):
        a_np = a.numpy() if a_kmajor else a.numpy().T
        b_np = b.numpy() if b_kmajor else b.numpy().T
        a_np, b_np = np.ascontiguousarray(a_np[:m, :k]), np.ascontiguousarray(b_np[:n, :k])
        if qtype == self.o.INT8:
            acc = self.o.gemm_i8(a_np, b_np).astype(np.float64)
        else:
            acc = self.o.gemm_e4m3(a_np, b_np)
        return torch.from_numpy(self.o.dequant(acc, sa.numpy(), sb.numpy()))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, qtype, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from hadamard_rotated_precision_halo_b200 import inputs
    from hadamard_rotated_precision_halo_b200.fsdp import ShardedLinear

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w_full = inputs.weights(N, K, seed=11, device="cpu")
        rows = N // world
        layer = ShardedLinear(w_full[rank * rows:(rank + 1) * rows].clone(), qtype=qtype, ops=OracleOps())
        x = inputs.activations(M_R, K, seed=20 + rank, device="cpu")
        dy = inputs.grads(M_R, N, seed=30 + rank, device="cpu")
        y = layer.forward(x, out_fp32=True)
        dx, dw = layer.backward(dy, x, dx_fp32=True)
        out[rank] = (y.numpy(), dx.numpy(), dw.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("qtype", [0, 1])
def test_two_rank_sharded_layer_matches_the_oracle(qtype):
    sys.path.insert(0, ROOT)
    import oracle
    from hadamard_rotated_precision_halo_b200 import inputs

    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), qtype, out), nprocs=world, join=True)
    w_full = inputs.weights(N, K, seed=11, device="cpu")
    xs = [inputs.activations(M_R, K, seed=20 + r, device="cpu") for r in range(world)]
    dys = [inputs.grads(M_R, N, seed=30 + r, device="cpu") for r in range(world)]
    dw_sum = sum(oracle.linear_bwd_dw(dys[r], xs[r], 128, qtype) for r in range(world))
    rows = N // world
    for r in range(world):
        y, dx, dw = out[r]
        np.testing.assert_array_equal(y, oracle.linear_fwd(xs[r], w_full, 128, qtype))
        np.testing.assert_array_equal(dx, oracle.linear_bwd_dx(dys[r], w_full, 128, qtype))
        np.testing.assert_allclose(dw, dw_sum[r * rows:(r + 1) * rows], rtol=1e-12, atol=0)


def test_shard_rows_must_be_whole_blocks():
    sys.path.insert(0, ROOT)
    from hadamard_rotated_precision_halo_b200.fsdp import ShardedLinear

    with pytest.raises(ValueError):
        ShardedLinear(torch.zeros((200, 256), dtype=torch.bfloat16), ops=OracleOps())


# ------------------------------------------------------------------------------ GPU
@pytest.mark.gpu
@pytest.mark.parametrize("qtype", [0, 1])
def test_one_process_sharded_layer_equals_the_single_device_calls(qtype):
    import hadamard_rotated_precision_halo_b200 as halo
    from hadamard_rotated_precision_halo_b200 import inputs
    from hadamard_rotated_precision_halo_b200.fsdp import ShardedLinear

    m, n, k = 640, 1024, 768
    x = inputs.activations(m, k, seed=41, device="cuda")
    w = inputs.weights(n, k, seed=42, device="cuda")
    dy = inputs.grads(m, n, seed=43, device="cuda")
    layer = ShardedLinear(w, qtype=qtype)
    y = layer.forward(x, out_fp32=True)
    dx, dw = layer.backward(dy, x, dx_fp32=True)
    y_ref = halo.halo_linear_fwd(x, w, 128, qtype, halo.HALO_OUT_FP32)
    dx_ref, dw_ref = halo.halo_linear_bwd(dy, x, w, 128, qtype, halo.HALO_OUT_FP32, halo.HALO_OUT_FP32)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref) and torch.equal(dx, dx_ref) and torch.equal(dw, dw_ref)
    st, site = halo.halo_device_error()
    assert st == halo.HALO_OK, f"bounded wait ran out at site {site:#x}"


@pytest.mark.gpu
@pytest.mark.parametrize("qtype", [0, 1])
@pytest.mark.parametrize("rows,cols,cut", [(1024, 768, 512), (1000, 208, 384), (8192, 96, 4096)])
def test_split_dim0_codes_equal_the_whole_matrix_codes(qtype, rows, cols, cut):
    """Rows cut into two shards at a block boundary: the shards' column maxima
    merged by maximum, then each shard quantised with them, give the codes and
    scales of the whole matrix; the maxima match the oracle's."""
    import hadamard_rotated_precision_halo_b200 as halo
    import oracle
    from hadamard_rotated_precision_halo_b200 import inputs

    x = inputs.activations(rows, cols, seed=rows + cols, device="cuda")
    x[:, 3] = 0  # an all-zero column
    parts = [x[:cut], x[cut:]]
    amax = torch.maximum(halo.halo_hadamard_colmax(parts[0]), halo.halo_hadamard_colmax(parts[1]))
    codes = [halo.halo_hadamard_quantize_colmax(p, 128, qtype, amax) for p in parts]
    q, s = halo.halo_hadamard_quantize(x, halo.HALO_AXIS_ROWS, 128, qtype)
    torch.cuda.synchronize()
    got = torch.cat([codes[0][0].view(torch.uint8), codes[1][0].view(torch.uint8)])
    assert torch.equal(got, q.view(torch.uint8))
    assert torch.equal(codes[0][1], s) and torch.equal(codes[1][1], s)
    v = oracle.rotate(x.cpu(), 128, 0)
    ref = np.abs(v).max(axis=0) * np.sqrt(128.0)  # maxima of the unnormalised transform
    got_amax = amax.cpu().numpy().astype(np.float64)
    assert np.all(got_amax[ref == 0] == 0)
    nz = ref > 0
    assert np.max(np.abs(got_amax[nz] - ref[nz]) / ref[nz]) < 1e-6
    st, site = halo.halo_device_error()
    assert st == halo.HALO_OK, f"bounded wait ran out at site {site:#x}"
