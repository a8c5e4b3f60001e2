"""Comparison helpers shared by the GPU parity tests (no method arithmetic here:
the expected values always come from the oracle)."""
import numpy as np
import torch

import oracle

# Quantised codes must match the oracle bit for bit, except where the oracle's
# pre-rounding value lies within this relative distance of a rounding midpoint
# (the GPU computes v * (qmax / amax) in fp32; the oracle v / s in fp64).
BOUNDARY_REL = 1e-6
# Scales: fp32 on both sides from differently ordered arithmetic.
SCALE_REL = 1e-6
# Final fp32 / bf16 outputs: max |Y - Y_ref| / max |Y_ref|.
OUT_REL = 1e-3


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.uint8).cpu().numpy()


def check_codes(gpu_codes, gpu_scales, ora_codes, ora_scales, ora_t, qtype):
    """Returns (#exempt elements, #exempt elements that differ)."""
    g = u8(gpu_codes)
    gs = gpu_scales.detach().cpu().numpy().astype(np.float64)
    os_ = np.asarray(ora_scales, dtype=np.float64)
    zero = os_ == 0
    assert np.all(gs[zero] == 0), "zero groups must give zero scales"
    rel = np.abs(gs[~zero] - os_[~zero]) / os_[~zero]
    assert rel.size == 0 or rel.max() <= SCALE_REL, f"scale rel err {rel.max():.3e}"
    exempt = oracle.boundary_distance(ora_t, qtype) < BOUNDARY_REL
    diff = g != ora_codes
    bad = diff & ~exempt
    if bad.any():
        idx = np.argwhere(bad)[:5]
        details = [(tuple(i), int(g[tuple(i)]), int(ora_codes[tuple(i)]), float(ora_t[tuple(i)])) for i in idx]
        raise AssertionError(f"{int(bad.sum())} code mismatches outside the boundary band, e.g. {details}")
    return int(exempt.sum()), int((diff & exempt).sum())


def check_output(gpu_out: torch.Tensor, ref: np.ndarray, rel: float = OUT_REL):
    y = gpu_out.detach().float().cpu().numpy().astype(np.float64)
    assert y.shape == ref.shape
    assert np.all(np.isfinite(y))
    scale = np.max(np.abs(ref))
    err = np.max(np.abs(y - ref)) / (scale if scale > 0 else 1.0)
    assert err <= rel, f"normwise error {err:.3e} > {rel:.1e}"
    if gpu_out.dtype == torch.bfloat16:
        # beyond the normwise bound, most elements sit within one bf16 ulp
        big = np.abs(ref) > 1e-2 * scale
        r = np.abs(y[big] - ref[big]) / np.abs(ref[big])
        assert np.median(r) <= 2.0**-8
    return err


def oracle_operand(x_bf16_cpu: torch.Tensor, axis_along: int, blk: int, qtype: int):
    """Oracle codes/scales/t of one operand.  axis_along=1: rotate along the
    contiguous dim, one scale per row; axis_along=0: along dim 0, one per column."""
    v = oracle.rotate(x_bf16_cpu, blk, axis=axis_along)
    return oracle.quantize(v, axis=0 if axis_along == 1 else 1, qtype=qtype)
