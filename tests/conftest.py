import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch

        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device in this process")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Per code comparison: how many codes the parity band exempted from
    bit-exactness, split by the term that exempts them, and how many of those
    actually differ (tests/_parity.py EXEMPT_LOG)."""
    mod = sys.modules.get("tests._parity")
    log = getattr(mod, "EXEMPT_LOG", None) if mod is not None else None
    if not log:
        return
    tr = terminalreporter
    tr.write_sep("=", "code parity: exempt codes per comparison")
    tr.write_line(f"{'test':<72} {'kind':<10} {'qtype':<5} {'shape':<14} {'codes':>10} {'rel':>6} "
                  f"{'band':>6} {'differ':>6} {'exempt%':>8} {'ceil%':>6}")
    tot = {}
    worst = 0.0
    for r in log:
        n_ex = r["exempt_rel"] + r["exempt_band_only"]
        frac = n_ex / max(r["codes"], 1)
        worst = max(worst, frac / r["ceiling"])
        shape = "x".join(str(d) for d in r["shape"])
        name = r["test"][6:] if r["test"].startswith("tests/") else r["test"]
        tr.write_line(f"{name[-72:]:<72} {r['kind']:<10} {r['qtype']:<5} {shape:<14} {r['codes']:>10} "
                      f"{r['exempt_rel']:>6} {r['exempt_band_only']:>6} {r['differ']:>6} {100 * frac:>8.4f} "
                      f"{100 * r['ceiling']:>6.2f}")
        t = tot.setdefault((r["kind"], r["qtype"]), [0, 0, 0, 0, 0])
        t[0] += 1
        t[1] += r["codes"]
        t[2] += r["exempt_rel"]
        t[3] += r["exempt_band_only"]
        t[4] += r["differ"]
    for (kind, qt), (k, n, a, b, d) in sorted(tot.items()):
        tr.write_line(f"total {kind} {qt}: {k} comparisons, {n} codes, exempt {a} (relative term) + {b} "
                      f"(fp32 transform bound only) = {100 * (a + b) / max(n, 1):.4f}%, of which {d} differ")
    tr.write_line(f"largest exempt share relative to its ceiling: {worst:.2f}")
