"""Benchmark: Hadamard-rotated quantized linear layer on B200.

A step is one pass of the whole hot path over one Llama-70B layer at 4096
tokens (hidden 8192, FFN 28672, 8 KV heads of 128): forward, dX and dW of the
seven linear layers q, k, v, o, gate, up, down -- 21 GEMMs, each rotating both
operands with a block-128 Walsh-Hadamard transform along its contraction
dimension, quantising per row / column to INT8 and multiplying on the tensor
cores with a dequantising epilogue.  Inputs are seeded synthetic bf16
(activations N(0,1) with outlier channels, weights N(0, 0.02^2), output
gradients N(0, 1e-3^2)); they exceed the 126 MB L2 several times over.

The metric is whole-job throughput in TOPS (2 * M * N * K per GEMM, summed,
including the rotation and quantisation launches) over the device-timed
steps, which replay the step's launches as one captured CUDA graph
(`--no-graph`: launched from the host); rotate+quantise GB/s and the GEMM
kernels' own TOPS are reported beside it, and `e2e` times the same step through
the linear-layer calls with host buffers.  The same line carries the other
workloads measured on their own (`configs`): the tiny forward, rotate+quantise
of [16384, 4096] activations, the Llama-7B attention-projection forward and
FFN down-projection backward (INT8 and E4M3), and the 70B layer in E4M3.
`--qtype e4m3` runs FP8 as the headline, `--group 64|128` group-wise scales.  `--impl reference` times the CPU oracle on a
bounded sample of the same workload instead.  `--measure-peaks` and
`--rotq-shapes` print the GEMM peak comparison and the per-shape
rotate+quantise table.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from hadamard_rotated_precision_halo_b200 import inputs  # noqa: E402

METRIC = "rotated-qGEMM TOPS & rotate+quant GB/s at Llama shapes vs B200 peak (1 GPU)"
# DRAM bytes (read + write) per qgemm_pair_kernel launch, averaged over the 21
# GEMMs of the INT8 layer step, from one ncu capture, and the SHA-256 prefix of
# the GEMM kernel source (csrc/qgemm.cuh) that capture ran.  The bench reports
# the figure only while the source still hashes the same, null otherwise.
GEMM_TRAFFIC_BYTES_PER_LAUNCH_INT8_LAYER = 462.3e6
GEMM_TRAFFIC_SOURCE_SHA = "2eae0e678d021206"
UNIT = "TOPS"
BLK = 128
# The sustained 8-bit denominator applies when the timed region lasts long
# enough for the board to settle at its power cap; shorter regions run at the
# burst clock.
SUSTAINED_REGION_S = 2.0


def gemm_source_sha() -> str:
    import hashlib

    path = os.path.join(ROOT, "hadamard_rotated_precision_halo_b200", "csrc", "qgemm.cuh")
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def peaks(path: str = None):
    """HBM copy GB/s and dense bf16 TFLOP/s (burst, sustained) measured on this
    pool's B200s (MEASURED_PEAKS.json at the repository root), else the
    fallback figures, saying which."""
    path = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16": p["bf16_tflops"], "bf16_sustained": p["bf16_tflops_sustained"],
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


def gemm_peak(pk: dict, region_s: float):
    """The dense 8-bit denominator for the GEMM roofline: the measured bf16
    figure times the nominal 8-bit : bf16 ratio (4.5 : 2.25), burst for a timed
    region shorter than SUSTAINED_REGION_S, sustained (power-capped) otherwise.
    Returns (peak, kind, burst, sustained)."""
    burst, sustained = 2.0 * pk["bf16"], 2.0 * pk["bf16_sustained"]
    if region_s >= SUSTAINED_REGION_S:
        return sustained, "sustained", burst, sustained
    return burst, "burst", burst, sustained


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------- workload
class LayerStep:
    """All tensors and launches of one layer step (forward + dX + dW of 7 GEMMs)."""

    def __init__(self, shapes: inputs.LayerShapes, seed: int, device, qtype: int, kinds=("fwd", "dx", "dw"),
                 group: int = 0):
        import hadamard_rotated_precision_halo_b200 as halo

        self.halo = halo
        self.group = group  # 0: one scale per row / column; 64 or 128: group-wise scales along K
        self.kinds = kinds
        self.shapes = shapes
        self.qtype = qtype
        self.dev = device
        self.t = inputs.layer_inputs(shapes, seed, device)
        t = shapes.tokens
        self.y, self.dx, self.dw = {}, {}, {}
        code_dt = torch.int8 if qtype == halo.HALO_Q_INT8 else torch.float8_e4m3fn
        max_mk = max(t * g.k for g in shapes.gemms)
        max_nk = max(g.n * g.k for g in shapes.gemms)
        max_mn = max(t * g.n for g in shapes.gemms)
        max_vec = max(max(t, g.n, g.k) for g in shapes.gemms)
        # Code / scale buffers for the two operands of the GEMM in flight.
        self.qa = torch.empty(max(max_mk, max_mn), dtype=torch.uint8, device=device)
        self.qb = torch.empty(max(max_nk, max_mk), dtype=torch.uint8, device=device)
        n_scales = max(max_vec, max(max_mk, max_nk, max_mn) // group) if group else max_vec
        self.sa = torch.empty(n_scales, dtype=torch.float32, device=device)
        self.sb = torch.empty(n_scales, dtype=torch.float32, device=device)
        self.code_dt = code_dt
        for g in shapes.gemms:
            self.y[g.name] = torch.empty((t, g.n), dtype=torch.bfloat16, device=device)
            self.dx[g.name] = torch.empty((t, g.k), dtype=torch.bfloat16, device=device)
            self.dw[g.name] = torch.empty((g.n, g.k), dtype=torch.float32, device=device)
        if group:
            wsz = lambda m, n, k, which: int(halo.lib().halo_workspace_size_grouped(m, n, k, group, which))
        else:
            wsz = halo.halo_workspace_size
        self.ws_fwd = max(wsz(t, g.n, g.k, 0) for g in shapes.gemms)
        self.ws_bwd = max(wsz(t, g.n, g.k, 1) for g in shapes.gemms)
        self.ws = torch.empty(max(self.ws_fwd, self.ws_bwd), dtype=torch.uint8, device=device)

    def ops_per_step(self) -> int:
        return self.shapes.total_ops(self.kinds)

    def _codes(self, buf, rows, cols):
        return buf[: rows * cols].view(self.code_dt).view(rows, cols)

    def n_scales(self, x, ax) -> int:
        """Scales of one rotate+quantise of x along axis ax: one per row / column,
        or one per group of the rotated dimension."""
        rows, cols = x.shape
        if ax == self.halo.HALO_AXIS_COLS:
            return rows * (cols // self.group if self.group else 1)
        return cols * (rows // self.group if self.group else 1)

    def gemms(self):
        """The step as (a, a_axis, b, b_axis, m, n, k, out) launch groups, in order."""
        h = self.halo
        t = self.shapes.tokens
        out = []
        for g in self.shapes.gemms:
            x, w = self.t["x"][g.x_key], self.t["w"][g.name]
            if "fwd" in self.kinds:
                out.append(("fwd", g.name, x, h.HALO_AXIS_COLS, w, h.HALO_AXIS_COLS, t, g.n, g.k, self.y[g.name]))
        for g in self.shapes.gemms:
            x, w, dy = self.t["x"][g.x_key], self.t["w"][g.name], self.t["dy"][g.name]
            if "dx" in self.kinds:
                out.append(("dx", g.name, dy, h.HALO_AXIS_COLS, w, h.HALO_AXIS_ROWS, t, g.k, g.n, self.dx[g.name]))
            if "dw" in self.kinds:
                out.append(("dw", g.name, dy, h.HALO_AXIS_ROWS, x, h.HALO_AXIS_ROWS, g.n, g.k, t, self.dw[g.name]))
        return out

    def plan(self):
        """The step's launches in order.  An operand rotated along the same axis
        for several GEMMs (the attention input for q, k, v and the MLP input for
        gate, up, in the forward and in dW) is rotated once per step into a code
        buffer of its own and reused; every other operand goes through the two
        scratch code buffers.  Entries: ("rotq", x, axis, codes, scales) and
        ("gemm", (codes_a, scales_a, axis_a), (codes_b, scales_b, axis_b), m, n, k, out)."""
        if getattr(self, "_plan", None) is not None:
            return self._plan
        h = self.halo
        gem = self.gemms()
        count = {}
        for g in gem:
            for x, ax in ((g[2], g[3]), (g[4], g[5])):
                key = (x.data_ptr(), ax)
                count[key] = count.get(key, 0) + 1
        self.shared = {}
        for g in gem:
            for x, ax in ((g[2], g[3]), (g[4], g[5])):
                key = (x.data_ptr(), ax)
                if count[key] > 1 and key not in self.shared:
                    q = torch.empty(x.shape, dtype=self.code_dt, device=self.dev)
                    sc = torch.empty(self.n_scales(x, ax), dtype=torch.float32, device=self.dev)
                    self.shared[key] = (q, sc)
        # dY feeds dX (rotated along its columns) and dW (along its rows): when
        # the step has both, its two code sets come from one call
        # (halo_hadamard_quantize_both: the second rotation reads dY from L2),
        # the dim-0 set into a buffer of its own, kept until the dW GEMM.
        both = {}
        if self.group == 0 and "dx" in self.kinds and "dw" in self.kinds:
            for g in self.shapes.gemms:
                dy = self.t["dy"][g.name]
                key = (dy.data_ptr(), h.HALO_AXIS_ROWS)
                if key not in self.shared:
                    q = torch.empty(self.halo.codes_shape(dy.shape[0], dy.shape[1], h.HALO_AXIS_ROWS, BLK),
                                    dtype=self.code_dt, device=self.dev)
                    self.shared[key] = (q, torch.empty(dy.shape[1], dtype=torch.float32, device=self.dev))
                both[dy.data_ptr()] = key
        plan, done = [], set()
        for kind, name, a, a_axis, b, b_axis, m, n, k, c in gem:
            operands = []
            for slot, x, ax in ((0, a, a_axis), (1, b, b_axis)):
                key = (x.data_ptr(), ax)
                if key in self.shared:
                    q, sc = self.shared[key]
                    if key not in done:
                        plan.append(("rotq", x, ax, q, sc))
                        done.add(key)
                else:
                    q = self._codes(self.qa if slot == 0 else self.qb, x.shape[0], x.shape[1])
                    sc = self.sa if slot == 0 else self.sb
                    if ax == h.HALO_AXIS_COLS and x.data_ptr() in both and both[x.data_ptr()] not in done:
                        qc, scc = self.shared[both[x.data_ptr()]]
                        plan.append(("both", x, q, sc, qc, scc))
                        done.add(both[x.data_ptr()])
                    else:
                        plan.append(("rotq", x, ax, q, sc))
                operands.append((q, sc, ax))
            plan.append(("gemm", operands[0], operands[1], m, n, k, c))
        self._plan = plan
        return plan

    def run(self, events=None):
        """One step through the C ABI (halo_hadamard_quantize, halo_qgemm).  With
        `events` (a list), record a CUDA event before every launch and one after
        the last, on the launching stream; returns the number of launches."""
        h = self.halo
        L = h.lib()
        stream = torch.cuda.current_stream()
        sp = h._stream(stream)
        plan = self.plan()
        for op in plan:
            if events is not None:
                ev = torch.cuda.Event(enable_timing=True)
                ev.record(stream)
                events.append(ev)
            if op[0] == "both":
                _, x, q, sc, qc, scc = op
                st = L.halo_hadamard_quantize_both(h._ptr(x), x.shape[0], x.shape[1], x.stride(0), BLK, self.qtype,
                                                   h._ptr(q), q.stride(0), h._ptr(sc), h._ptr(qc), qc.stride(0),
                                                   h._ptr(scc), sp)
                h._check(st, "halo_hadamard_quantize_both")
            elif op[0] == "rotq":
                _, x, ax, q, sc = op
                if self.group:
                    st = L.halo_hadamard_quantize_grouped(h._ptr(x), x.shape[0], x.shape[1], x.stride(0), ax, BLK,
                                                          self.group, self.qtype, h._ptr(q), q.stride(0), h._ptr(sc),
                                                          sp)
                else:
                    st = L.halo_hadamard_quantize(h._ptr(x), x.shape[0], x.shape[1], x.stride(0), ax, BLK,
                                                  self.qtype, h._ptr(q), q.stride(0), h._ptr(sc), sp)
                h._check(st, "halo_hadamard_quantize")
            else:
                _, (qa, sa, ax_a), (qb, sb, ax_b), m, n, k, c = op
                a_major = h.HALO_MAJOR_K if ax_a == h.HALO_AXIS_COLS else h.HALO_MAJOR_MN
                b_major = h.HALO_MAJOR_K if ax_b == h.HALO_AXIS_COLS else h.HALO_MAJOR_MN
                otype = h.HALO_OUT_FP32 if c.dtype == torch.float32 else h.HALO_OUT_BF16
                if self.group:
                    st = L.halo_qgemm_grouped(h._ptr(qa), h._ptr(sa), a_major, qa.stride(0), h._ptr(qb), h._ptr(sb),
                                              b_major, qb.stride(0), m, n, k, self.group, self.qtype, h._ptr(c),
                                              otype, c.stride(0), sp)
                else:
                    st = L.halo_qgemm(h._ptr(qa), h._ptr(sa), a_major, qa.stride(0), h._ptr(qb), h._ptr(sb),
                                      b_major, qb.stride(0), m, n, k, self.qtype, h._ptr(c), otype, c.stride(0), sp)
                h._check(st, "halo_qgemm")
        if events is not None:
            ev = torch.cuda.Event(enable_timing=True)
            ev.record(stream)
            events.append(ev)
        return self.launches_per_step()

    def attribute(self, events, steps):
        """Per-call durations from an instrumented run of `steps` steps:
        (gemm ms, [rotate+quantise ms, elements] per axis; key 2: both axes
        from one halo_hadamard_quantize_both call)."""
        plan = self.plan()
        gemm_ms, by_axis = 0.0, {0: [0.0, 0], 1: [0.0, 0], 2: [0.0, 0]}
        per = len(plan) + 1
        for s_i in range(steps):
            evs = events[s_i * per:(s_i + 1) * per]
            for j, op in enumerate(plan):
                dt = evs[j].elapsed_time(evs[j + 1])
                if op[0] == "gemm":
                    gemm_ms += dt
                else:
                    ax = 2 if op[0] == "both" else op[2]
                    by_axis[ax][0] += dt
                    by_axis[ax][1] += op[1].numel()
        return gemm_ms, by_axis

    def launches_per_step(self) -> int:
        """Kernel launches of one step (a "both" call launches two)."""
        return sum(2 if op[0] == "both" else 1 for op in self.plan())

    def rotq_bytes(self) -> int:
        """Algorithmic bytes of the step's rotate+quantise launches: bf16 in
        (2 B) + code out (1 B) per element + one fp32 scale per group."""
        h = self.halo
        total = 0
        for op in self.plan():
            if op[0] == "rotq":
                x, ax = op[1], op[2]
                total += 3 * x.numel() + 4 * self.n_scales(x, ax)
            elif op[0] == "both":  # one read, two code sets, a scale per row and per column
                x = op[1]
                total += 4 * x.numel() + 4 * (x.shape[0] + x.shape[1])
        return total

    def gemm_bytes(self) -> int:
        """Algorithmic DRAM bytes of the step's GEMMs: both code operands, the
        output and the two scale vectors."""
        total = 0
        for op in self.plan():
            if op[0] == "gemm":
                m, n, k, c = op[3], op[4], op[5], op[6]
                ng = k // self.group if self.group else 1
                total += m * k + n * k + m * n * c.element_size() + 4 * (m + n) * ng
        return total

    def gemm_ops(self) -> int:
        return sum(2 * op[3] * op[4] * op[5] for op in self.plan() if op[0] == "gemm")


def e2e_run(step: LayerStep, steps: int):
    """Same metric end to end through the public linear-layer calls with host
    buffers: every step copies all of its inputs from pinned host memory, runs
    halo_linear_fwd / halo_linear_bwd, and copies all outputs (Y, dX, dW) back.

    The copies run on their own streams, one per direction, so that they
    overlap the kernels and each other (PCIe is full duplex): a GEMM starts as
    soon as its operands have arrived, and each output is read back as soon as
    it is written.  Device inputs and outputs are double-buffered across steps,
    so step s + 1's uploads overlap step s's downloads; events order every
    reuse of a buffer after the previous use of it has finished."""
    h = step.halo
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(step.dev), torch.cuda.Stream(step.dev)
    host_in = {key: {n: v.cpu().pin_memory() for n, v in d.items()} for key, d in step.t.items()}
    outs = {"y": step.y, "dx": step.dx, "dw": step.dw}
    host_out = {key: {n: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for n, v in d.items()}
                for key, d in outs.items()}
    h2d = sum(v.numel() * v.element_size() for d in host_in.values() for v in d.values())
    d2h = sum(v.numel() * v.element_size() for d in host_out.values() for v in d.values())
    dev_in = [{key: {n: torch.empty_like(v, device=step.dev) for n, v in d.items()} for key, d in host_in.items()}
              for _ in range(2)]
    dev_out = [outs, {key: {n: torch.empty_like(v) for n, v in d.items()} for key, d in outs.items()}]
    inputs_free = [None, None]   # compute is done reading buffer b's inputs
    outputs_free = [None, None]  # the downloads of buffer b's outputs are done
    gemms = step.shapes.gemms

    def event(stream):
        e = torch.cuda.Event()
        e.record(stream)
        return e

    def one(s):
        b = s % 2
        din, dout = dev_in[b], dev_out[b]
        # uploads, in the order the kernels need them
        with torch.cuda.stream(up):
            if inputs_free[b] is not None:
                up.wait_event(inputs_free[b])
            ready = {}
            for g in gemms:
                for key, n in (("x", g.x_key), ("w", g.name)):
                    if (key, n) not in ready:
                        din[key][n].copy_(host_in[key][n], non_blocking=True)
                        ready[(key, n)] = event(up)
            for g in gemms:
                din["dy"][g.name].copy_(host_in["dy"][g.name], non_blocking=True)
                ready[("dy", g.name)] = event(up)
        # kernels
        if outputs_free[b] is not None:
            comp.wait_event(outputs_free[b])
        done = []
        for g in gemms:
            comp.wait_event(ready[("x", g.x_key)])
            comp.wait_event(ready[("w", g.name)])
            if step.group:
                h.halo_linear_fwd_grouped(din["x"][g.x_key], din["w"][g.name], BLK, step.group, step.qtype,
                                          h.HALO_OUT_BF16, y=dout["y"][g.name], ws=step.ws, stream=comp)
            else:
                h.halo_linear_fwd(din["x"][g.x_key], din["w"][g.name], BLK, step.qtype, h.HALO_OUT_BF16,
                                  y=dout["y"][g.name], ws=step.ws, stream=comp)
            done.append((("y", g.name), event(comp)))
        for g in gemms:
            comp.wait_event(ready[("dy", g.name)])
            if step.group:
                h.halo_linear_bwd_grouped(din["dy"][g.name], din["x"][g.x_key], din["w"][g.name], BLK, step.group,
                                          step.qtype, h.HALO_OUT_BF16, h.HALO_OUT_FP32, dx=dout["dx"][g.name],
                                          dw=dout["dw"][g.name], ws=step.ws, stream=comp)
            else:
                h.halo_linear_bwd(din["dy"][g.name], din["x"][g.x_key], din["w"][g.name], BLK, step.qtype,
                                  h.HALO_OUT_BF16, h.HALO_OUT_FP32, dx=dout["dx"][g.name], dw=dout["dw"][g.name],
                                  ws=step.ws, stream=comp)
            e = event(comp)
            done += [(("dx", g.name), e), (("dw", g.name), e)]
        inputs_free[b] = event(comp)
        # downloads, each as soon as its output is written
        with torch.cuda.stream(down):
            for (key, n), e in done:
                down.wait_event(e)
                host_out[key][n].copy_(dout[key][n], non_blocking=True)
            outputs_free[b] = event(down)

    def run(n, first):
        for s in range(first, first + n):
            one(s)
        comp.wait_stream(up)
        comp.wait_stream(down)

    run(2, 0)  # warm-up: both buffers
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(comp)
    up.wait_stream(comp)
    down.wait_stream(comp)
    run(steps, 2)
    end.record(comp)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / steps
    del dev_in, dev_out, host_in, host_out
    return ms, h2d, d2h


# ------------------------------------------------------------------ CPU baseline
class OracleSample:
    """The oracle as it stands on a bounded sample of the layer step: the q
    projection forward (rotate + quantise the first `rows` token rows of X and
    all of W_q, integer GEMM, dequantise)."""

    def __init__(self):
        import oracle

        self.oracle = oracle
        oracle.build()
        self.g = inputs.LLAMA70B_LAYER.gemms[0]
        self.w = inputs.weights(self.g.n, self.g.k, seed=100, device="cpu")
        self.x_all = inputs.activations(inputs.LLAMA70B_LAYER.tokens, self.g.k, seed=101, device="cpu")
        self.rows = 16

    def run(self, rows=None):
        rows = rows or self.rows
        x = self.x_all[:rows]
        t0 = time.perf_counter()
        self.oracle.linear_fwd(x, self.w, BLK, self.oracle.INT8)
        dt = time.perf_counter() - t0
        return 2 * rows * self.g.n * self.g.k, dt

    def size_for(self, seconds: float):
        """Grow the row sample until one run takes about `seconds`."""
        rows = 16
        ops, dt = self.run(rows)
        cap = self.x_all.shape[0]
        while dt < 0.6 * seconds and rows < cap:
            rows = min(cap, rows * 2)
            ops, dt = self.run(rows)
        self.rows = rows
        return ops, dt

    def describe(self, dt):
        return (f"q-projection forward, {self.rows} of {inputs.LLAMA70B_LAYER.tokens} token rows x "
                f"W[{self.g.n},{self.g.k}] (rotate+quantise both, INT8 GEMM, dequantise), block 128, "
                f"{dt:.1f} s per sample")


def cpu_baseline(seconds_target: float = 15.0):
    s = OracleSample()
    ops, dt = s.size_for(seconds_target)
    return {"value": ops / dt / 1e12, "unit": UNIT, "cores": s.oracle.num_threads(), "kind": "oracle",
            "sample": s.describe(dt)}


# ---------------------------------------------------------- auxiliary measurements
def _clock_proc():
    return subprocess.Popen(["nvidia-smi", "-i", str(torch.cuda.current_device()),
                             "--query-gpu=clocks.sm,power.draw", "--format=csv,noheader,nounits", "-lms", "50"],
                            stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)


def _clock_stop(p):
    p.terminate()
    out, _ = p.communicate()
    vals = [l.split(",") for l in out.splitlines() if l.strip()]
    sm = sorted(float(v[0]) for v in vals)
    pw = sorted(float(v[1]) for v in vals)
    return (sm[len(sm) // 2] if sm else None), (pw[len(pw) // 2] if pw else None)


def measure_peaks(n: int = 8192, seconds: float = 3.0):
    """8-bit GEMM throughput at n^3 on this GPU: this library's halo_qgemm next to
    cuBLAS (torch._int_mm for INT8, torch._scaled_mm for FP8), best of 10 single
    launches (burst) and a `seconds`-long back-to-back loop (sustained, with the
    SM clock and power seen meanwhile).  Library GEMMs are the comparison here,
    not part of the product path."""
    import hadamard_rotated_precision_halo_b200 as halo

    g = torch.Generator(device="cuda").manual_seed(0)
    a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device="cuda", generator=g)
    b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device="cuda", generator=g)
    a8 = torch.randn(n, n, device="cuda", generator=g).to(torch.float8_e4m3fn)
    b8 = torch.randn(n, n, device="cuda", generator=g).to(torch.float8_e4m3fn)
    ones = torch.ones(n, dtype=torch.float32, device="cuda")
    one = torch.ones((), device="cuda")
    c = torch.empty((n, n), dtype=torch.bfloat16, device="cuda")
    cases = {
        "halo_int8": lambda: halo.halo_qgemm(a, ones, 0, b, ones, 0, n, n, n, 0, 1, c=c),
        "cublas_int8": lambda: torch._int_mm(a, b.t()),
        "halo_e4m3": lambda: halo.halo_qgemm(a8, ones, 0, b8, ones, 0, n, n, n, 1, 1, c=c),
        "cublas_e4m3": lambda: torch._scaled_mm(a8, b8.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16),
    }
    out = {}
    for name, fn in cases.items():
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        best = 1e30
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        proc = _clock_proc()
        time.sleep(0.3)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        t0, cnt = time.time(), 0
        while time.time() - t0 < seconds:
            for _ in range(20):
                fn()
            cnt += 20
            torch.cuda.synchronize()
        e1.record()
        torch.cuda.synchronize()
        sm, pw = _clock_stop(proc)
        out[name] = {"burst_tops": 2 * n ** 3 / (best * 1e-3) / 1e12,
                     "sustained_tops": 2 * n ** 3 * cnt / (e0.elapsed_time(e1) * 1e-3) / 1e12,
                     "sm_mhz_median": sm, "power_w_median": pw}
    return {"measure": "8-bit GEMM peaks", "n": n, "results": out}


ROTQ_SHAPES = {  # (rows, cols) of every rotate+quantise operand of the 70B layer, and the standalone case
    "along_contiguous_dim": [(4096, 8192), (8192, 8192), (1024, 8192), (28672, 8192), (4096, 28672),
                             (8192, 28672), (4096, 1024), (16384, 4096)],
    "along_dim0": [(8192, 8192), (1024, 8192), (28672, 8192), (8192, 28672), (4096, 8192), (4096, 28672),
                   (4096, 1024), (16384, 4096)],
}


def measure_rotq_shapes(repeats: int = 10, only=None):
    """halo_hadamard_quantize on each shape alone (INT8 and E4M3, block 128), a
    512 MB write between repeats to flush L2; median time and algorithmic GB/s
    (3 B per element + 4 B per scale).  `only` = (direction, (rows, cols)):
    that one case (both types) and nothing else, e.g. for a profiler."""
    import hadamard_rotated_precision_halo_b200 as halo

    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    out = []
    cases = ROTQ_SHAPES if only is None else {only[0]: [only[1]]}
    for name, shapes in cases.items():
        axis = halo.HALO_AXIS_COLS if name == "along_contiguous_dim" else halo.HALO_AXIS_ROWS
        for r, c in shapes:
            x = inputs.activations(r, c, seed=1, device="cuda")
            for qt in (halo.HALO_Q_INT8, halo.HALO_Q_E4M3):
                q, sc = halo.halo_hadamard_quantize(x, axis, BLK, qt)
                torch.cuda.synchronize()
                ts = []
                for _ in range(repeats):
                    flush.zero_()
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    halo.halo_hadamard_quantize(x, axis, BLK, qt, q_out=q, scales_out=sc)
                    e1.record()
                    torch.cuda.synchronize()
                    ts.append(e0.elapsed_time(e1))
                ms = sorted(ts)[len(ts) // 2]
                nbytes = 3 * x.numel() + 4 * sc.numel()
                out.append({"direction": name, "shape": [r, c], "qtype": "int8" if qt == 0 else "e4m3",
                            "us": ms * 1e3, "gbs": nbytes / (ms * 1e-3) / 1e9})
            del x, q, sc
    if only is not None:
        return {"measure": "rotate+quantise per shape", "block": BLK, "results": out}
    # Both encodings from one read (halo_hadamard_quantize_dual): 2 B in + 1 B
    # per code set per element, 4 B per scale of each set.
    for r, c in ROTQ_SHAPES["along_contiguous_dim"]:
        x = inputs.activations(r, c, seed=1, device="cuda")
        outs = halo.halo_hadamard_quantize_dual(x, BLK)
        torch.cuda.synchronize()
        ts = []
        for _ in range(repeats):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            halo.halo_hadamard_quantize_dual(x, BLK, *outs)
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        ms = sorted(ts)[len(ts) // 2]
        nbytes = 4 * x.numel() + 8 * r
        out.append({"direction": "along_contiguous_dim", "shape": [r, c], "qtype": "int8+e4m3 (one read)",
                    "us": ms * 1e3, "gbs": nbytes / (ms * 1e-3) / 1e9})
        del x, outs
    # Group-wise scales (halo_hadamard_quantize_grouped, INT8): 4 B per scale
    # of every group of 64 / 128 positions along the rotated dimension.
    for name, shapes in ROTQ_SHAPES.items():
        axis = halo.HALO_AXIS_COLS if name == "along_contiguous_dim" else halo.HALO_AXIS_ROWS
        for r, c in (shapes[1], shapes[-1]):
            x = inputs.activations(r, c, seed=1, device="cuda")
            for group in (64, 128):
                q, sc = halo.halo_hadamard_quantize_grouped(x, axis, BLK, group, halo.HALO_Q_INT8)
                torch.cuda.synchronize()
                ts = []
                for _ in range(repeats):
                    flush.zero_()
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    halo.halo_hadamard_quantize_grouped(x, axis, BLK, group, halo.HALO_Q_INT8, q_out=q, scales_out=sc)
                    e1.record()
                    torch.cuda.synchronize()
                    ts.append(e0.elapsed_time(e1))
                ms = sorted(ts)[len(ts) // 2]
                nbytes = 3 * x.numel() + 4 * sc.numel()
                out.append({"direction": name, "shape": [r, c], "qtype": "int8", "variant": f"group {group}",
                            "us": ms * 1e3, "gbs": nbytes / (ms * 1e-3) / 1e9})
                del q, sc
            del x
    # The variants (halo_hadamard_quantize_ex): random signs along the rotated
    # dimension and stochastic rounding from 16 random bits per element (which
    # add 2 B per element of input traffic).
    g = torch.Generator(device="cuda").manual_seed(7)
    for name, shapes in ROTQ_SHAPES.items():
        axis = halo.HALO_AXIS_COLS if name == "along_contiguous_dim" else halo.HALO_AXIS_ROWS
        for r, c in shapes[:2] + shapes[-1:]:
            x = inputs.activations(r, c, seed=1, device="cuda")
            signs = (torch.randint(0, 2, (c if axis == halo.HALO_AXIS_COLS else r,), device="cuda", generator=g,
                                   dtype=torch.int8) * 2 - 1).to(torch.int8)
            rand = torch.randint(0, 65536, (r, c), device="cuda", generator=g, dtype=torch.int32).to(torch.uint16)
            for variant, sg, rb in (("signs", signs, None), ("stochastic", None, rand), ("signs+stochastic", signs, rand)):
                q, sc = halo.halo_hadamard_quantize_ex(x, axis, BLK, halo.HALO_Q_INT8, signs=sg, rand_bits=rb)
                torch.cuda.synchronize()
                ts = []
                for _ in range(repeats):
                    flush.zero_()
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    halo.halo_hadamard_quantize_ex(x, axis, BLK, halo.HALO_Q_INT8, signs=sg, rand_bits=rb, q_out=q,
                                                   scales_out=sc)
                    e1.record()
                    torch.cuda.synchronize()
                    ts.append(e0.elapsed_time(e1))
                ms = sorted(ts)[len(ts) // 2]
                nbytes = (3 + (2 if rb is not None else 0)) * x.numel() + 4 * sc.numel() + (sg.numel() if sg is not None else 0)
                out.append({"direction": name, "shape": [r, c], "qtype": "int8", "variant": variant,
                            "us": ms * 1e3, "gbs": nbytes / (ms * 1e-3) / 1e9})
            del x, q, sc, rand, signs
    return {"measure": "rotate+quantise per shape", "block": BLK, "results": out}


# ------------------------------------------------------------ the other workloads
def capture_step(step: "LayerStep"):
    """The step's launches captured once as a CUDA graph (warmed up first)."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step.run()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step.run()
    torch.cuda.synchronize()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    return graph


def _timed(fn, reps: int, flush=None) -> list:
    """Device time (ms) of each of `reps` calls of fn, CUDA events on the
    current stream; `flush` (a buffer larger than L2) is overwritten before
    every call, outside the timed interval."""
    ts = []
    for _ in range(reps):
        if flush is not None:
            flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    return ts


def measure_other_configs(pk: dict, reps: int = 20) -> dict:
    """The remaining workloads, each on its own, after the headline step:
    the tiny forward X[64,256] W[128,256] (block 256, INT8, fp32 Y; latency);
    rotate+quantise of [16384, 4096] activations (INT8, E4M3, both from one
    read; GB/s against the HBM copy peak); the Llama-7B attention-projection
    forward 8192x4096x4096 and FFN down-projection backward (dX + dW,
    8192x11008x4096), INT8 and E4M3, TOPS including every rotate+quantise
    launch against the burst 8-bit peak; and the Llama-70B layer step in E4M3.
    Every call writes a 512 MB buffer first (outside the timing), so no input
    is served from L2.  Median over `reps` calls (10 steps for the 70B layer,
    whose inputs exceed L2 several times)."""
    import hadamard_rotated_precision_halo_b200 as halo

    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    hbm = pk["hbm_gbs"]
    peak8 = 2.0 * pk["bf16"]
    med = lambda ts: sorted(ts)[len(ts) // 2]
    out = {"peak_8bit_tops": peak8, "peak_hbm_gbs": hbm, "timing": f"median of {reps}, L2 flushed before each"}

    # tiny forward (latency-bound: report the call's device time)
    x = inputs.plain(64, 256, seed=0, device="cuda")
    w = inputs.plain(128, 256, seed=1, device="cuda")
    y = torch.empty((64, 128), dtype=torch.float32, device="cuda")
    ws = torch.empty(halo.halo_workspace_size(64, 128, 256, 0), dtype=torch.uint8, device="cuda")
    fn = lambda: halo.halo_linear_fwd(x, w, 256, halo.HALO_Q_INT8, halo.HALO_OUT_FP32, y=y, ws=ws)
    for _ in range(3):
        fn()
    ms = med(_timed(fn, reps, flush))
    out["tiny_fwd_64x128x256"] = {"us": ms * 1e3, "tops": 2 * 64 * 128 * 256 / (ms * 1e-3) / 1e12,
                                  "launches": 3, "bound": "launch latency"}
    del x, w, y, ws

    # standalone rotate+quantise [16384, 4096]
    x = inputs.activations(16384, 4096, seed=2, device="cuda")
    rq = {}
    for name, qt in (("int8", halo.HALO_Q_INT8), ("e4m3", halo.HALO_Q_E4M3)):
        q, sc = halo.halo_hadamard_quantize(x, halo.HALO_AXIS_COLS, BLK, qt)
        ms = med(_timed(lambda: halo.halo_hadamard_quantize(x, halo.HALO_AXIS_COLS, BLK, qt, q_out=q,
                                                            scales_out=sc), reps, flush))
        gb = (3 * x.numel() + 4 * sc.numel()) / (ms * 1e-3) / 1e9
        rq[name] = {"us": ms * 1e3, "gbs": gb, "frac": gb / hbm}
        del q, sc
    outs = halo.halo_hadamard_quantize_dual(x, BLK)
    ms = med(_timed(lambda: halo.halo_hadamard_quantize_dual(x, BLK, *outs), reps, flush))
    gb = (4 * x.numel() + 8 * x.shape[0]) / (ms * 1e-3) / 1e9
    rq["int8+e4m3_one_read"] = {"us": ms * 1e3, "gbs": gb, "frac": gb / hbm}
    out["rotate_quantize_16384x4096"] = rq
    del x, outs

    # single-GEMM Llama-7B cases and the 70B layer in E4M3
    cases = [("llama7b_attn_proj_fwd", "int8"), ("llama7b_attn_proj_fwd", "e4m3"),
             ("llama7b_ffn_down_bwd", "int8"), ("llama7b_ffn_down_bwd", "e4m3"),
             ("llama70b_layer_fwd_bwd", "e4m3")]
    for wl, qname in cases:
        shapes, kinds = WORKLOADS[wl]
        qt = halo.HALO_Q_INT8 if qname == "int8" else halo.HALO_Q_E4M3
        st = LayerStep(shapes, seed=4, device=torch.device("cuda"), qtype=qt, kinds=kinds)
        g = capture_step(st)
        clk = None
        if wl == "llama70b_layer_fwd_bwd":
            with ClockSampler(torch.cuda.current_device()) as sampler:
                ts = _timed(g.replay, 20)
            clk = sampler.summary()
        else:
            ts = _timed(g.replay, reps, flush)
        ms = med(ts)
        tops = st.ops_per_step() / (ms * 1e-3) / 1e12
        out.setdefault(wl, {})[qname] = {"ms_per_step": ms, "tops": tops, "frac_burst": tops / peak8,
                                         "target_frac": 0.60, "launches": st.launches_per_step()}
        if clk is not None:
            out[wl][qname]["clocks"] = clk
            out[wl][qname]["ms_min_max"] = [min(ts), max(ts)]
        del g, st
        torch.cuda.synchronize()
    return out


# ------------------------------------------------------------------ multi-rank
def max_over_ranks(ms: float, world: int, device) -> float:
    """Device-timed region of this rank -> the maximum over all ranks (the
    job's time).  One all-reduce; every rank calls it in the same place."""
    if world <= 1:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(ops_per_step: int, steps: int, world: int, ms_total: float) -> float:
    """Whole-job throughput in TOPS: every rank runs `steps` steps of the same
    work (replicas, weak scaling), over the max-over-ranks time."""
    return ops_per_step * steps * world / (ms_total * 1e-3) / 1e12


# ------------------------------------------------------------------------- main
WORKLOADS = {
    "llama70b_layer_fwd_bwd": (inputs.LLAMA70B_LAYER, ("fwd", "dx", "dw")),
    "llama7b_attn_proj_fwd": (inputs.LLAMA7B_ATTN_PROJ, ("fwd",)),
    "llama7b_ffn_down_bwd": (inputs.LLAMA7B_FFN_DOWN, ("dx", "dw")),
    "llama70b_gate_proj_dx": (inputs.LLAMA70B_GATE, ("dx",)),
    "llama70b_q_proj_dw": (inputs.LLAMA70B_Q, ("dw",)),
}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="halo", choices=["halo", "reference"])
    ap.add_argument("--qtype", default="int8", choices=["int8", "e4m3"])
    ap.add_argument("--group", type=int, default=0, choices=[0, 64, 128],
                    help="group-wise scales along each GEMM's contraction dimension (0: one scale per row)")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every kernel from the host instead of replaying the captured step")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the tiny, rotate+quantise, Llama-7B and FP8 70B-layer measurements")
    ap.add_argument("--workload", default="llama70b_layer_fwd_bwd", choices=sorted(WORKLOADS),
                    help="the bench line uses the default; the single-GEMM cases serve profiling")
    ap.add_argument("--measure-peaks", action="store_true",
                    help="print 8-bit GEMM burst / sustained throughput (this library and cuBLAS) and exit")
    ap.add_argument("--rotq-shapes", action="store_true",
                    help="print rotate+quantise time per operand shape of the layer and exit")
    ap.add_argument("--rotq-shape", default=None, metavar="AXIS:RxC",
                    help="with --rotq-shapes: only this case, AXIS contig or dim0 (e.g. dim0:16384x4096)")
    args = ap.parse_args()
    if args.measure_peaks or args.rotq_shapes:
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        only = None
        if args.rotq_shape:
            ax, shape = args.rotq_shape.split(":")
            r, c = (int(v) for v in shape.split("x"))
            only = ("along_contiguous_dim" if ax == "contig" else "along_dim0", (r, c))
        print(json.dumps(measure_peaks() if args.measure_peaks else measure_rotq_shapes(only=only)), flush=True)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    shapes, kinds = WORKLOADS[args.workload]
    config = {"workload": args.workload, "tokens": shapes.tokens, "hidden": shapes.hidden,
              "ffn": shapes.ffn, "kv": shapes.kv, "gemms": len(shapes.gemms) * len(kinds), "block": BLK,
              "qtype": args.qtype, "l2": "inputs larger than L2 (no flush)", "parallelism": f"replicas{world}"}
    if args.impl != "reference":
        config["launch"] = "stream" if args.no_graph else "cuda_graph"
        if args.group:
            config["scale_group"] = args.group

    if args.impl == "reference":
        if rank != 0:
            return
        s = OracleSample()
        s.size_for(4.0)
        for _ in range(args.warmup):
            s.run()
        ops_total, t_total = 0, 0.0
        for _ in range(args.steps):
            ops, dt = s.run()
            ops_total += ops
            t_total += dt
        value = ops_total / t_total / 1e12
        cb = {"value": value, "unit": UNIT, "cores": s.oracle.num_threads(), "kind": "oracle",
              "sample": s.describe(t_total / max(args.steps, 1))}
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_total / max(args.steps, 1),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config, "cpu_baseline": cb,
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import hadamard_rotated_precision_halo_b200 as halo

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
    qtype = halo.HALO_Q_INT8 if args.qtype == "int8" else halo.HALO_Q_E4M3
    step = LayerStep(shapes, seed=4 + rank, device=device, qtype=qtype, kinds=kinds, group=args.group)
    torch.cuda.synchronize()

    for _ in range(max(args.warmup, 3)):
        step.run()
    torch.cuda.synchronize()
    st, site = halo.halo_device_error()
    if st != halo.HALO_OK:
        raise RuntimeError(f"device error after warm-up at site {site:#x}")

    # The step's launches captured once as a CUDA graph (same kernels, same
    # arguments); replaying it keeps the GPU fed through the stretches of
    # short kernels that per-launch host work (ctypes, tensor-map encoding)
    # cannot keep up with.  --no-graph launches every kernel from the host.
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step.run()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(graph):
            step.run()
        torch.cuda.synchronize()
        for _ in range(max(args.warmup, 3)):
            graph.replay()
        torch.cuda.synchronize()

    # Timed region: K steps (no events between launches).
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    per_step = step.launches_per_step()
    with ClockSampler(local) as clocks:
        start.record(stream)
        launches = 0
        for _ in range(args.steps):
            if graph is not None:
                graph.replay()
                launches += per_step
            else:
                launches += step.run()
        end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_total = max_over_ranks(start.elapsed_time(end), world, device)
    st, site = halo.halo_device_error()
    if st != halo.HALO_OK:
        raise RuntimeError(f"device error in the timed region at site {site:#x}")

    # Attribution: the same K steps again with a CUDA event before every launch
    # (same stream), for the per-kernel durations.
    events = []
    for _ in range(args.steps):
        step.run(events)
    torch.cuda.synchronize()
    gemm_ms, by_axis = step.attribute(events, args.steps)
    ms_instrumented = events[0].elapsed_time(events[-1]) / args.steps
    rotq_ms = by_axis[0][0] + by_axis[1][0] + by_axis[2][0]
    n_gemm = sum(1 for op in step.plan() if op[0] == "gemm") * args.steps

    ops_step = step.ops_per_step()
    ms_step = ms_total / args.steps
    value = job_throughput(ops_step, args.steps, world, ms_total)
    gemm_tops = step.gemm_ops() * args.steps / (gemm_ms * 1e-3) / 1e12
    rotq_gbs = step.rotq_bytes() * args.steps / (rotq_ms * 1e-3) / 1e9
    pk = peaks()
    region_s = ms_total * 1e-3
    peak8, peak_kind, peak8_burst, peak8_sus = gemm_peak(pk, region_s)
    sustained = peak_kind == "sustained"

    def gbs(axis):  # 3 B per element (bf16 in, code out); both axes from one read: 4 B
        return (4 if axis == 2 else 3) * by_axis[axis][1] / max(by_axis[axis][0] * 1e-3, 1e-12) / 1e9

    traffic_ok = (args.workload == "llama70b_layer_fwd_bwd" and args.qtype == "int8" and not args.group
                  and GEMM_TRAFFIC_SOURCE_SHA is not None and gemm_source_sha() == GEMM_TRAFFIC_SOURCE_SHA)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8" if qtype == halo.HALO_Q_INT8 else "e4m3",
            "data": "synthetic", "config": config,
            "gpu_launches": launches,
            "roofline": {"bound": "tensor", "kernel": "qgemm_grouped_kernel" if args.group else "qgemm_pair_kernel",
                         "achieved": gemm_tops, "peak": peak8, "unit": "TFLOP/s", "frac": gemm_tops / peak8,
                         "peak_kind": "sustained" if sustained else "burst",
                         "frac_burst": gemm_tops / peak8_burst, "frac_sustained": gemm_tops / peak8_sus,
                         "peak_burst": peak8_burst, "peak_sustained": peak8_sus,
                         "traffic": GEMM_TRAFFIC_BYTES_PER_LAUNCH_INT8_LAYER if traffic_ok else None,
                         "traffic_unit": "bytes per launch (DRAM read + write, ncu)",
                         "algorithmic_bytes_per_launch": step.gemm_bytes() / max(n_gemm // args.steps, 1),
                         "peak_note": f"2 x {pk['source']} bf16 dense (8-bit : bf16 = 2 : 1); "
                                      f"{'sustained' if sustained else 'burst'} for a {region_s:.2f} s timed region",
                         "launches": n_gemm, "avg_launch_ms": gemm_ms / max(n_gemm, 1)},
            "step_roofline": {"achieved": value / max(world, 1), "unit": "TFLOP/s", "peak": peak8,
                              "frac": value / max(world, 1) / peak8,
                              "frac_burst": value / max(world, 1) / peak8_burst,
                              "frac_sustained": value / max(world, 1) / peak8_sus, "target_frac": 0.60,
                              "note": "whole step per GPU, every rotate+quantise launch included"},
            "rotq": {"gbs": rotq_gbs, "peak_gbs": pk["hbm_gbs"], "frac": rotq_gbs / pk["hbm_gbs"],
                     "target_frac": 0.70,
                     "bytes_per_step": step.rotq_bytes(), "ms_per_step": rotq_ms / args.steps,
                     "along_contiguous_dim_gbs": gbs(0), "along_dim0_gbs": gbs(1),
                     "along_contiguous_dim_frac": gbs(0) / pk["hbm_gbs"], "along_dim0_frac": gbs(1) / pk["hbm_gbs"],
                     "along_contiguous_dim_ms_per_step": by_axis[0][0] / args.steps,
                     "along_dim0_ms_per_step": by_axis[1][0] / args.steps,
                     "both_axes_of_dy_gbs": gbs(2) if by_axis[2][1] else None,
                     "both_axes_of_dy_frac": gbs(2) / pk["hbm_gbs"] if by_axis[2][1] else None,
                     "both_axes_of_dy_ms_per_step": by_axis[2][0] / args.steps},
            "ms_per_step_instrumented": ms_instrumented,
            "clocks": clocks.summary()}

    if not args.no_e2e:
        # every rank runs its own replica end to end; the job's time is the slowest rank's
        e2e_steps = 4
        e2e_ms, h2d, d2h = e2e_run(step, steps=e2e_steps)
        e2e_ms = max_over_ranks(e2e_ms, world, device)
        if rank == 0:
            line["e2e"] = {"value": job_throughput(ops_step, 1, world, e2e_ms), "unit": UNIT,
                           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                           "steps": e2e_steps, "copies": "own stream per direction, overlapped with the kernels"}
    if (world == 1 and not args.no_other_configs and args.workload == "llama70b_layer_fwd_bwd"
            and not args.group and args.qtype == "int8"):
        line["configs"] = measure_other_configs(pk)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
