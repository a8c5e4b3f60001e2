"""The parity tests' exemption band for quantised codes, checked on the CPU.

The GPU evaluates the block transform in fp32; the oracle in fp64.  Where the
block's outputs cancel to far below its inputs (next to outlier channels) the
fp32 rounding of the transform can move the pre-rounding value t by much more
than 1e-6 |t|, so a code may round the other way.  rotation_rounding_band()
bounds that move from the arithmetic; these tests simulate an fp32 transform
(any order of the log2(b) butterfly levels) and check that the bound holds for
every element, and that it covers the element a GPU run showed crossing a
midpoint.
"""
import numpy as np
import pytest

import oracle
from hadamard_rotated_precision_halo_b200 import inputs
from tests._parity import rotation_rounding_band


def _fwht_f32_rows(x32: np.ndarray, blk: int, order) -> np.ndarray:
    """Unnormalised block transform of each row in fp32, butterfly levels in `order`."""
    rows, cols = x32.shape
    v = x32.reshape(rows, cols // blk, blk).copy()
    for h in order:
        v = v.reshape(rows, cols // blk, blk // (2 * h), 2, h)
        a = v[:, :, :, 0, :].copy()
        b = v[:, :, :, 1, :].copy()
        v[:, :, :, 0, :] = a + b
        v[:, :, :, 1, :] = a - b
    return v.reshape(rows, cols)


def _t_f32(x, blk, qmax, order):
    """t as the GPU forms it: fp32 transform u, then u * fl(qmax / max|u|) per row."""
    x32 = oracle.bf16_to_f64(x).astype(np.float32)
    u = _fwht_f32_rows(x32, blk, order)
    amax = np.abs(u).max(axis=1, keepdims=True)
    r = np.where(amax > 0, np.float32(qmax) / np.where(amax > 0, amax, np.float32(1)), np.float32(0))
    return (u * r.astype(np.float32)).astype(np.float64)


@pytest.mark.parametrize("qtype", [oracle.INT8, oracle.E4M3])
@pytest.mark.parametrize("order", ["up", "down"])
def test_band_bounds_fp32_transform(qtype, order):
    blk = 128
    x = inputs.activations(64, 4096, seed=21, device="cpu")  # outlier channels x50
    levels = [1 << i for i in range(7)]
    t32 = _t_f32(x, blk, oracle.QMAX[qtype], levels if order == "up" else levels[::-1])
    _, scales, t64 = oracle.quantize(oracle.rotate(x, blk, 1), axis=0, qtype=qtype)
    band = rotation_rounding_band(t64, scales, blk, 1) + 1e-6 * np.abs(t64)
    err = np.abs(t32 - t64)
    assert np.all(err <= band), f"max err/band {np.max(err / np.maximum(band, 1e-300)):.3f}"
    # the bound is not vacuous: it stays far below one quantisation step
    assert np.max(band) < 0.05


def test_band_covers_the_crossing_seen_on_the_gpu():
    """Row 288, column 6064 of the 300 x 28672 group-128 E4M3 parity case: the
    oracle's t is -0.2421813 (rounds to -0.234375), an fp32 transform gives
    -0.2421878, past the midpoint -0.2421875 (rounds to -0.25)."""
    x = inputs.activations(300, 28672, seed=300 + 2 * 28672 + 128, device="cpu")
    x[1, :64] = 0
    r, c0 = 288, (6064 // 128) * 128
    xb = x[r:r + 1, c0:c0 + 128]
    _, scales, t64 = oracle.quantize_grouped(oracle.rotate(xb, 128, 1), 1, 128, oracle.E4M3)
    t32 = _t_f32(xb, 128, 448.0, [1 << i for i in range(7)])
    j = 6064 - c0
    mid = -0.2421875
    assert t64[0, j] > mid > t32[0, j]  # the two sides of the midpoint
    band = rotation_rounding_band(t64, scales, 128, 1)
    assert abs(t64[0, j] - mid) <= band[0, j]
    assert abs(t64[0, j] - mid) > 1e-6 * abs(t64[0, j])  # outside the relative band alone


def test_exemption_counts_are_recorded_and_bounded(monkeypatch):
    """check_codes records how many codes each term of the band exempts, and
    fails when the exempt share passes its ceiling.  Here the oracle's own
    codes stand in for the GPU's (nothing differs); widening the fixed relative
    term to 0.05 exempts ~10% of the codes and must trip the ceiling."""
    import torch

    from tests import _parity

    x = inputs.activations(64, 1024, seed=5, device="cpu")
    for qt in (oracle.INT8, oracle.E4M3):
        codes, scales, t = _parity.oracle_operand(x, 1, 128, qt)
        gpu_codes = torch.from_numpy(np.ascontiguousarray(codes))
        gpu_scales = torch.from_numpy(np.asarray(scales, dtype=np.float32))
        before = len(_parity.EXEMPT_LOG)
        n_ex, n_diff = _parity.check_codes(gpu_codes, gpu_scales, codes, scales, t, qt, blk=128, axis=1)
        rec = _parity.EXEMPT_LOG[before]
        assert len(_parity.EXEMPT_LOG) == before + 1
        assert rec["codes"] == x.numel() and n_diff == 0 and rec["differ"] == 0
        assert rec["exempt_rel"] + rec["exempt_band_only"] == n_ex
        assert n_ex <= _parity.rne_exempt_ceiling(128) * x.numel()
        monkeypatch.setattr(_parity, "BOUNDARY_REL", 0.05)
        with pytest.raises(AssertionError, match="ceiling"):
            _parity.check_codes(gpu_codes, gpu_scales, codes, scales, t, qt, blk=128, axis=1)
        del _parity.EXEMPT_LOG[before + 1:]  # the planted widening is not a parity record
        monkeypatch.setattr(_parity, "BOUNDARY_REL", 1e-6)
