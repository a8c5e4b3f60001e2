"""Comparison helpers shared by the GPU parity tests (no method arithmetic here:
the expected values always come from the oracle)."""
import os

import numpy as np
import torch

import oracle

# Quantised codes must match the oracle bit for bit, except where the oracle's
# pre-rounding value lies within this relative distance of a rounding midpoint
# (the GPU computes v * (qmax / amax) in fp32; the oracle v / s in fp64), or
# within the fp32 transform's own rounding bound of it (rotation_rounding_band).
BOUNDARY_REL = 1e-6
# Scales: fp32 on both sides from differently ordered arithmetic.
SCALE_REL = 1e-6
# Final fp32 / bf16 outputs: max |Y - Y_ref| / max |Y_ref|.
OUT_REL = 1e-3
# Ceilings on the share of an operand's codes that the band may exempt from
# bit-exactness, so that a widened band cannot hide a systematic mismatch.
# The exempt set depends on the oracle's values alone (fixed seeds), so these
# checks cannot flake.  Round to nearest: 0.2% for 128-blocks, 0.4% for
# 256-blocks (the fp32 transform's bound grows with the block); the test inputs
# measure at most 0.16% and 0.36%, and 0.003%-0.08% on the large outlier
# operands.  Stochastic rounding also exempts a decision within 1e-4 of
# flipping (about 0.04% of codes) and every group's maximum (t = +-qmax lies on
# the grid): 1%, against at most 0.45% measured.
EXEMPT_MAX_FRAC_RNE_128 = 2e-3
EXEMPT_MAX_FRAC_STOCHASTIC = 1e-2


def rne_exempt_ceiling(blk) -> float:
    return EXEMPT_MAX_FRAC_RNE_128 * (blk if blk else 128) / 128

# One record per code comparison, printed at the end of the test session
# (tests/conftest.py): which test, the shape and type, how many codes, how many
# the 1e-6 relative term exempts, how many only the fp32 transform's bound
# exempts, and how many exempt codes actually differ.
EXEMPT_LOG = []


def _record(kind, shape, qtype, n, by_rel, by_band, differ, ceiling):
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    EXEMPT_LOG.append({"test": test, "kind": kind, "shape": tuple(int(d) for d in shape),
                       "qtype": "int8" if qtype == oracle.INT8 else "e4m3", "codes": int(n),
                       "exempt_rel": int(by_rel), "exempt_band_only": int(by_band), "differ": int(differ),
                       "ceiling": ceiling})
    frac = (by_rel + by_band) / max(n, 1)
    assert frac <= ceiling, (
        f"the band exempts {by_rel + by_band} of {n} codes ({100 * frac:.3f}%, "
        f"{by_rel} by the fixed relative term, {by_band} by the fp32 transform bound only), "
        f"above the {100 * ceiling:.1f}% ceiling")


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.uint8).cpu().numpy()


def _scale_per_element(scales, shape, axis: int) -> np.ndarray:
    """Each element's scale: one per row when the blocks run along the
    contiguous dim (axis 1), one per column when they run along dim 0; 2-D
    group-wise scales repeat over their group."""
    s = np.asarray(scales, dtype=np.float64)
    if s.ndim == 1:
        return np.broadcast_to(s[:, None] if axis == 1 else s[None, :], shape)
    if axis == 1:
        return np.repeat(s, shape[1] // s.shape[1], axis=1)
    return np.repeat(s, shape[0] // s.shape[0], axis=0)


def rotation_rounding_band(t, scales, blk: int, axis: int) -> np.ndarray:
    """Upper bound, in the units of the pre-rounding value t = v / s, on how far
    the GPU's fp32 evaluation of t can lie from the oracle's fp64 one.

    The b-point transform is log2(b) levels of additions, each partial sum
    rounded once, so each output is off by at most log2(b) u sum_j |x_j| / sqrt(b)
    (u = 2^-24, x the block's inputs; pairwise summation), and
    sum_j |x_j| / sqrt(b) <= ||x||_2 = ||v_block||_2 (the normalised transform is
    orthogonal).  The scale comes from the largest |v| of its group, computed the
    same way, whose relative error is at most log2(b) u sqrt(b).  Bit-exact codes
    cannot be asked for where t lies closer to a rounding midpoint than this:
    the transform is evaluated in fp32 and its rounding may carry t across.  The
    bound is small except where the block's outputs cancel to far below its
    inputs (|v| much less than ||v_block||), e.g. next to outlier channels."""
    t = np.asarray(t, dtype=np.float64)
    se = _scale_per_element(scales, t.shape, axis)
    v = t * se
    rows, cols = t.shape
    if axis == 1:
        nrm = np.sqrt((v.reshape(rows, cols // blk, blk) ** 2).sum(axis=2))
        nrm = np.repeat(nrm, blk, axis=1)
    else:
        nrm = np.sqrt((v.reshape(rows // blk, blk, cols) ** 2).sum(axis=1))
        nrm = np.repeat(nrm, blk, axis=0)
    lg = np.log2(blk)
    u = 2.0 ** -24
    with np.errstate(divide="ignore", invalid="ignore"):
        band = lg * u * (np.where(se > 0, nrm / se, 0.0) + np.sqrt(blk) * np.abs(t))
    return band


def check_codes(gpu_codes, gpu_scales, ora_codes, ora_scales, ora_t, qtype, blk=None, axis=None):
    """Returns (#exempt elements, #exempt elements that differ).  With `blk` and
    `axis` (1: blocks along the contiguous dim, 0: along dim 0) the exemption
    also covers the fp32 transform's rounding bound (rotation_rounding_band).
    The counts, split by the term that exempts each code, are recorded in
    EXEMPT_LOG, and the exempt share must stay within EXEMPT_MAX_FRAC."""
    g = u8(gpu_codes)
    gs = gpu_scales.detach().cpu().numpy().astype(np.float64)
    os_ = np.asarray(ora_scales, dtype=np.float64)
    zero = os_ == 0
    assert np.all(gs[zero] == 0), "zero groups must give zero scales"
    rel = np.abs(gs[~zero] - os_[~zero]) / os_[~zero]
    assert rel.size == 0 or rel.max() <= SCALE_REL, f"scale rel err {rel.max():.3e}"
    rel_d = oracle.boundary_distance(ora_t, qtype)
    by_rel = rel_d < BOUNDARY_REL
    exempt = by_rel.copy()
    if blk is not None:
        with np.errstate(invalid="ignore"):  # t = 0 has no midpoint (relative distance inf)
            exempt |= rel_d * np.abs(ora_t) <= rotation_rounding_band(ora_t, ora_scales, blk, axis)
    diff = g != ora_codes
    _record("rne", g.shape, qtype, g.size, by_rel.sum(), (exempt & ~by_rel).sum(), (diff & exempt).sum(),
            rne_exempt_ceiling(blk))
    bad = diff & ~exempt
    if bad.any():
        idx = np.argwhere(bad)[:5]
        details = [(tuple(i), int(g[tuple(i)]), int(ora_codes[tuple(i)]), float(ora_t[tuple(i)])) for i in idx]
        raise AssertionError(f"{int(bad.sum())} code mismatches outside the boundary band, e.g. {details}")
    far = diff & exempt & ~_one_step_apart(g, np.asarray(ora_codes), qtype)
    assert not far.any(), f"{int(far.sum())} exempt codes differ by more than one quantisation step"
    return int(exempt.sum()), int((diff & exempt).sum())


def _one_step_apart(a, b, qtype) -> np.ndarray:
    """Codes that are equal or neighbours on the quantisation grid."""
    if qtype == oracle.INT8:
        return np.abs(a.view(np.int8).astype(np.int16) - b.view(np.int8).astype(np.int16)) <= 1
    da = oracle.e4m3_decode(a)
    db = oracle.e4m3_decode(b)
    m = np.maximum(np.abs(da), np.abs(db))
    step = np.where(m <= 2.0 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(m, 2.0 ** -6))) - 3))
    return np.abs(da - db) <= step


def check_codes_stochastic(gpu_codes, gpu_scales, ora_codes, ora_scales, ora_t, rand_bits, qtype, band=1e-4,
                           blk=None, axis=None):
    """Stochastic rounding: codes must match the oracle's except where the
    decision is within `band` of flipping -- the random threshold u close to the
    oracle's fraction p = (t - lo) / (hi - lo), or t close to a grid point (p
    near 0 or 1) -- since the GPU forms t in fp32 (about 1e-7 relative).  With
    `blk` and `axis` the band also covers the fp32 transform's rounding bound
    (rotation_rounding_band) in units of p.  Returns (#exempt, #exempt that differ)."""
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
    bp = np.full(t.shape, band)
    bp_rel = bp
    if blk is not None:
        q_unit = 1.0 if qtype == oracle.INT8 else quantum
        bp = np.maximum(bp, rotation_rounding_band(t, ora_scales, blk, axis) / q_unit)
    # t = 0 exactly (an all-zero group, or zero padding meeting zeros) is code 0
    # on both sides: nothing to exempt there.
    nz = t != 0
    by_rel = nz & ((np.abs(u - p) < bp_rel) | (p < bp_rel) | (p > 1 - bp_rel))
    exempt = nz & ((np.abs(u - p) < bp) | (p < bp) | (p > 1 - bp))
    diff = g != ora_codes
    _record("stochastic", g.shape, qtype, g.size, by_rel.sum(), (exempt & ~by_rel).sum(), (diff & exempt).sum(),
            EXEMPT_MAX_FRAC_STOCHASTIC)
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
