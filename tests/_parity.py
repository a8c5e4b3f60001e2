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


def check_codes_stochastic(gpu_codes, gpu_scales, ora_codes, ora_scales, ora_t, rand_bits, qtype, band=1e-4):
    """Stochastic rounding: codes must match the oracle's except where the
    decision is within `band` of flipping -- the random threshold u close to the
    oracle's fraction p = (t - lo) / (hi - lo), or t close to a grid point (p
    near 0 or 1) -- since the GPU forms t in fp32 (about 1e-7 relative).
    Returns (#exempt, #exempt that differ)."""
    g = u8(gpu_codes)
    gs = gpu_scales.detach().cpu().numpy().astype(np.float64)
    os_ = np.asarray(ora_scales, dtype=np.float64)
    zero = os_ == 0
    assert np.all(gs[zero] == 0)
    rel = np.abs(gs[~zero] - os_[~zero]) / os_[~zero]
    assert rel.size == 0 or rel.max() <= SCALE_REL
    t = np.asarray(ora_t)
    u = np.asarray(rand_bits, dtype=np.float64) / 65536.0
    if qtype == oracle.INT8:
        p = t - np.floor(t)
    else:
        a = np.abs(t)
        quantum = np.where(a < 2.0**-6, 2.0**-9, 2.0 ** (np.floor(np.log2(np.maximum(a, 1e-300))) - 3))
        p = (a - np.floor(a / quantum) * quantum) / quantum
    exempt = (np.abs(u - p) < band) | (p < band) | (p > 1 - band)
    diff = g != ora_codes
    bad = diff & ~exempt
    if bad.any():
        idx = np.argwhere(bad)[:5]
        details = [(tuple(i), int(g[tuple(i)]), int(ora_codes[tuple(i)]), float(t[tuple(i)]), float(u[tuple(i)]))
                   for i in idx]
        raise AssertionError(f"{int(bad.sum())} stochastic code mismatches outside the band, e.g. {details}")
    return int(exempt.sum()), int((diff & exempt).sum())


def bf16_half_ulp(y: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers (8 significant bits) at |y|."""
    a = np.abs(y)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 8), 0.0)


def check_output(gpu_out: torch.Tensor, ref: np.ndarray, rel: float = OUT_REL):
    """max |Y - Y_ref| / max |Y_ref| <= rel.  For bf16 outputs the bound applies to
    the value before the final rounding, so each element may differ by a further
    half bf16 ulp of itself (the rounding to bf16 alone is up to 2^-9 relative)."""
    y = gpu_out.detach().float().cpu().numpy().astype(np.float64)
    assert y.shape == ref.shape
    assert np.all(np.isfinite(y))
    scale = np.max(np.abs(ref))
    diff = np.abs(y - ref)
    if gpu_out.dtype == torch.bfloat16:
        diff = np.maximum(diff - bf16_half_ulp(y), 0.0)
    err = np.max(diff) / (scale if scale > 0 else 1.0)
    assert err <= rel, f"normwise error {err:.3e} > {rel:.1e}"
    return err


def oracle_operand(x_bf16_cpu: torch.Tensor, axis_along: int, blk: int, qtype: int):
    """Oracle codes/scales/t of one operand.  axis_along=1: rotate along the
    contiguous dim, one scale per row; axis_along=0: along dim 0, one per column."""
    v = oracle.rotate(x_bf16_cpu, blk, axis=axis_along)
    return oracle.quantize(v, axis=0 if axis_along == 1 else 1, qtype=qtype)
