"""Benchmark of the Averis split NVFP4 linear layer (forward + dgrad).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl averis|reference]

One step = one forward and one dgrad pass of the Qwen3-0.6B fused-QKV
projection (X bf16 [8192, 1024], W [1024, 4096], dY bf16 [8192, 4096],
Philox stochastic rounding): column reduce, fold, split quantizer (+ mean
quantizer and rank-one row) and tcgen05 FP4 GEMM for each pass, eight kernel
launches.
The weight quantization is done once before timing (it runs once per weight
update, not per linear) and is reported on its own.

Metric: useful FLOPs 2*(2 l m n) per step / device time, TFLOP/s.  Device
time: CUDA events around K replays of a CUDA graph of the step, inputs
rotating over enough copies that they exceed the 126 MB L2; max over ranks.
Under torchrun each rank runs its own replica (weak scaling, no collective in
the data path: the layer needs none).  Prints one JSON line on rank 0.

--impl reference times the CPU oracle (the plain restatement of the method
that the tests compare against) on a bounded row sample of the same workload.
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L, M, N = 8192, 1024, 4096
WORKLOAD = "Qwen3-0.6B fused QKV projection, forward + dgrad: X bf16 [8192, 1024], W [1024, 4096], dY bf16 [8192, 4096], stochastic rounding"
METRIC = "Averis fwd+dgrad linear TFLOP/s (Qwen3-0.6B shapes); split-quant HBM GB/s"
FLOPS_PER_STEP = 2 * (2 * L * M * N)


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=4000)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="averis", choices=["averis", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-sample-rows", type=int, default=8192)
    p.add_argument("--cpu-sample-steps", type=int, default=2)
    p.add_argument("--copies", type=int, default=4, help="input copies rotated between steps")
    p.add_argument("--case", choices=["qkv"], default=None,
                   help="profiling case: the QKV step's kernels alone (weight quantization, then --steps Averis "
                        "and --steps vanilla fwd + dgrad steps, eager launches), no timing and no JSON line")
    return p.parse_args()


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []          # (monotonic time, csv line)
        self.window = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "5"],   # about 90 samples/s on a B200 host
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            # the timed region starts only once nvidia-smi is sampling
            t_end = time.monotonic() + 5.0
            while not self.lines and time.monotonic() < t_end and self.proc.poll() is None:
                time.sleep(0.01)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def region(self, t0, t1):
        """The timed region, in time.monotonic() seconds."""
        self.window = (t0, t1)
        # a region shorter than the sampling period still gets the next sample
        t_end = time.monotonic() + 1.0
        while self.proc is not None and time.monotonic() < t_end and not any(t > t1 for t, _ in self.lines):
            time.sleep(0.01)

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.t.join(timeout=2)

    def summary(self):
        """Median SM clock and active reasons over the samples taken inside the
        timed region; if the region was shorter than the sampling period, the
        first sample after it (labelled with samples_in_region = 0)."""
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = self.lines
        inside = lines
        if self.window is not None:
            t0, t1 = self.window
            inside = [(t, ln) for t, ln in lines if t0 <= t <= t1]
            if not inside:
                inside = [(t, ln) for t, ln in lines if t > t1][:1]
        n_inside = sum(1 for t, _ in inside if self.window is None or t <= self.window[1])
        for _, ln in inside:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) != 6:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[2:]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples_in_region": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples_in_region": n_inside}


# ---------------------------------------------------------------------------
# the 28-layer Qwen3-0.6B linear stack (beyond the timed step)
# ---------------------------------------------------------------------------
STACK_SHAPES = (("qkv", 1024, 4096), ("o_proj", 2048, 1024), ("gate_up", 1024, 6144), ("down", 3072, 1024))


def stack_timing(dev, stream, layers=28, tokens=32768, steps=3):
    """Forward + dgrad through the 4 linears of each of `layers` layers at
    `tokens` tokens, Averis and vanilla NVFP4, one CUDA graph of the whole
    stack per mode, replayed `steps` times.  Every layer has its own weights
    (N(0, 1/sqrt(m)), quantized once); the activations and output gradients
    of a shape are shared by the layers (drawn on the device, seeded):
    activations = per-column mean N(0, 0.5) with 1% of channels x20 + N(0, 1)
    (the down projection's input: silu(a) b with a, b ~ N(0.2, 1)); output
    gradients 1e-3 (N(0, 1) + per-column N(0, 0.3)).  SM clocks are sampled
    over the timed replays (tens of ms, so several samples fall inside)."""
    import torch
    from quantized_gemm_column_b200 import api
    g = torch.Generator(device=dev)
    g.manual_seed(20)
    acts, weights = [], []
    for name, m, n in STACK_SHAPES:
        if name == "down":
            a = torch.randn(tokens, m, generator=g, device=dev) + 0.2
            b = torch.randn(tokens, m, generator=g, device=dev) + 0.2
            X = (torch.nn.functional.silu(a) * b).to(torch.bfloat16)
            del a, b
        else:
            mu = torch.randn(m, generator=g, device=dev) * 0.5
            hot = torch.randperm(m, generator=g, device=dev)[: m // 100]
            mu[hot] *= 20.0
            X = (torch.randn(tokens, m, generator=g, device=dev) + mu).to(torch.bfloat16)
        D = ((torch.randn(tokens, n, generator=g, device=dev) + torch.randn(n, generator=g, device=dev) * 0.3)
             * 1e-3).to(torch.bfloat16)
        ws = api.workspace(tokens, max(m, n), max(m, n), dev)
        Y = torch.empty((tokens, n), dtype=torch.bfloat16, device=dev)
        dX = torch.empty((tokens, m), dtype=torch.bfloat16, device=dev)
        acts.append((X, D, ws, Y, dX))
    torch.cuda.synchronize(dev)                # drawn on the default stream, consumed on `stream`
    for _ in range(layers):
        per_layer = []
        for name, m, n in STACK_SHAPES:
            W = (torch.randn(m, n, generator=g, device=dev) / m ** 0.5).to(torch.bfloat16)
            w_fwd, w_dgrad = api.NVFP4Tensor(n, m, dev), api.NVFP4Tensor(m, n, dev)
            wq_ws = api.workspace(m, n, n, dev)
            torch.cuda.synchronize(dev)
            api.averis_quant_weight(W, w_fwd, w_dgrad, wq_ws, stream)
            torch.cuda.synchronize(dev)
            if api.averis_check_status(wq_ws, stream):
                raise RuntimeError("device status set by the stack's weight quantization")
            del W, wq_ws
            per_layer.append((w_fwd, w_dgrad))
        weights.append(per_layer)

    def stack(vanilla):
        for per_layer in weights:
            for (X, D, ws, Y, dX), (w_fwd, w_dgrad) in zip(acts, per_layer):
                if vanilla:
                    api.nvfp4_linear_fwd(X, w_fwd, "sr", 1, 0, Y, ws, stream=stream)
                    api.nvfp4_linear_dgrad(D, w_dgrad, "sr", 2, 0, dX, ws, stream=stream)
                else:
                    api.averis_linear_fwd(X, w_fwd, "sr", 1, 0, Y, ws, stream=stream)
                    api.averis_linear_dgrad(D, w_dgrad, "sr", 2, 0, dX, ws, stream=stream)

    torch.cuda.synchronize(dev)
    out, clocks = {}, {}
    for vanilla in (False, True):
        with torch.cuda.stream(stream):
            stack(vanilla)
            torch.cuda.synchronize(dev)
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                stack(vanilla)
            gr.replay()
            torch.cuda.synchronize(dev)
            with ClockSampler(dev.index if dev.index is not None else 0) as clk:
                t0 = time.monotonic()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for _ in range(steps):
                    gr.replay()
                b.record(stream)
                torch.cuda.synchronize(dev)
                clk.region(t0, time.monotonic())
            clocks["vanilla" if vanilla else "averis"] = clk.summary()
        out["vanilla_ms" if vanilla else "averis_ms"] = a.elapsed_time(b) / steps
        del gr
    for _, _, ws, _, _ in acts:
        if api.averis_check_status(ws, stream):
            raise RuntimeError("device status set by the stack timing")
    flops = sum(2.0 * tokens * m * n * 2 for _, m, n in STACK_SHAPES) * layers
    return {"layers": layers, "tokens": tokens, "shapes": {s[0]: [s[1], s[2]] for s in STACK_SHAPES},
            "weights": "distinct per layer", "launch": "one CUDA graph of the whole stack per mode",
            "averis_ms_per_step": out["averis_ms"], "vanilla_ms_per_step": out["vanilla_ms"],
            "averis_overhead_vs_vanilla": out["averis_ms"] / out["vanilla_ms"] - 1.0,
            "tflops": flops / (out["averis_ms"] * 1e-3) / 1e12,
            "clocks": clocks,
            "data": "synthetic, drawn on the device (seeded)"}


# ---------------------------------------------------------------------------
# the MoE variant (beyond the timed step)
# ---------------------------------------------------------------------------
def moe_timing(dev, stream, avg_us):
    """Forward and dgrad of one MoE linear: 64 experts, 4096 tokens routed to 8
    experts each (skewed counts), hidden 2048 -> 1024 per expert; the permuted
    buffer (151 MB) is larger than L2."""
    import torch
    from quantized_gemm_column_b200 import api, inputs
    counts, Xm, Wm, Dm = inputs.workload_moe()
    E, m, n = Wm.shape
    l_cap = Xm.shape[0]
    cnt = torch.tensor(counts, dtype=torch.int32, device=dev)
    w_fwd, w_dgrad = api.NVFP4Group(E * n, m, E, dev), api.NVFP4Group(E * m, n, E, dev)
    wq_ws = api.workspace(m, n, n, dev)
    Wd, Xd, Dd = Wm.to(dev), Xm.to(dev), Dm.to(dev)
    torch.cuda.synchronize(dev)                # copied on the default stream, consumed on `stream`
    api.averis_moe_quant_weights(Wd, w_fwd, w_dgrad, wq_ws, stream)
    mws = api.moe_workspace(l_cap, max(m, n), max(m, n), E, dev)
    Y = torch.empty((l_cap, n), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((l_cap, m), dtype=torch.bfloat16, device=dev)
    fwd = avg_us(lambda i: api.averis_moe_linear_fwd(Xd, cnt, w_fwd, "sr", 1 + i, 0, Y, mws, stream))
    dgr = avg_us(lambda i: api.averis_moe_linear_dgrad(Dd, cnt, w_dgrad, "sr", 1 + i, 0, dX, mws, stream))
    if api.averis_check_status(mws, stream) or api.averis_check_status(wq_ws, stream):
        raise RuntimeError("device status set by the MoE timing")
    del Wd
    tokens = sum(counts)
    flops = 2.0 * tokens * m * n
    return {"experts": E, "tokens_routed": tokens, "rows_padded": l_cap, "m": m, "n": n,
            "fwd_us": fwd, "dgrad_us": dgr, "tflops": 2 * flops / ((fwd + dgr) * 1e-6) / 1e12,
            "launches_per_pass": 5}


# ---------------------------------------------------------------------------
# the measured FP4 ceiling
# ---------------------------------------------------------------------------
def fp4_ceiling(dev, stream):
    """The dense block-scaled FP4 rate of this device, measured two ways: this
    library's MMA-only tcgen05 loop on every SM (the tensor pipe alone, no
    loads), and cuBLASLt's NVFP4 GEMM at 8192^3 through torch._scaled_mm (a
    library GEMM, loads included).  Each is the best of 3 timed runs."""
    import torch
    from quantized_gemm_column_b200 import api
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    ns = torch.zeros(sms, dtype=torch.int64, device=dev)
    ws = api.workspace(0, 64, 0, dev)
    iters = 20000
    best = None
    with torch.cuda.stream(stream):
        api.averis_probe_mma_rate(2000, ns, ws, stream)
        for _ in range(3):
            api.averis_probe_mma_rate(iters, ns, ws, stream)
            torch.cuda.synchronize(dev)
            t = 2.0 * 128 * 256 * 256 * iters * sms / (int(ns.max().item()) * 1e-9) / 1e12
            best = t if best is None else max(best, t)
    if api.averis_check_status(ws, stream):
        raise RuntimeError("device status set by the MMA-rate loop")
    out = {"mma_loop_tflops": best, "mma_loop": f"{sms} CTAs x {iters} stages of 4 MMAs (M128 N256 K64), constant operands"}
    try:
        n = 8192
        a = torch.randint(0, 256, (n, n // 2), dtype=torch.uint8, device=dev).view(torch.float4_e2m1fn_x2)
        b = torch.randint(0, 256, (n, n // 2), dtype=torch.uint8, device=dev).view(torch.float4_e2m1fn_x2)
        sa = (torch.rand(n * n // 16, device=dev) + 0.5).to(torch.float8_e4m3fn)
        sb = (torch.rand(n * n // 16, device=dev) + 0.5).to(torch.float8_e4m3fn)
        with torch.cuda.stream(stream):
            for _ in range(3):
                torch._scaled_mm(a, b.t(), sa, sb, out_dtype=torch.bfloat16)
            best = None
            for _ in range(3):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(10):
                    torch._scaled_mm(a, b.t(), sa, sb, out_dtype=torch.bfloat16)
                e1.record(stream)
                torch.cuda.synchronize(dev)
                t = 2.0 * n ** 3 / (e0.elapsed_time(e1) * 1e-3 / 10) / 1e12
                best = t if best is None else max(best, t)
        out["cublaslt_nvfp4_8192_tflops"] = best
        del a, b, sa, sb
    except Exception as exc:          # a torch without the NVFP4 path
        out["cublaslt_nvfp4_8192_tflops"] = None
        out["cublaslt_error"] = f"{type(exc).__name__}: {str(exc)[:120]}"
    return out


# ---------------------------------------------------------------------------
# one linear at full size: Averis vs vanilla, the split and the GEMMs
# ---------------------------------------------------------------------------
def linear_timing(dev, stream, avg_us, X, W, D, fp4_peak):
    """Forward + dgrad of one linear (X [l, m], W [m, n], dY [l, n]), stochastic
    rounding: Averis and vanilla step times, the two splits and the two GEMMs
    on their own, TFLOP/s, the Averis overhead and the GEMMs' fraction of the
    measured FP4 peak."""
    import torch
    from quantized_gemm_column_b200 import api
    l, m = X.shape
    n = W.shape[1]
    Xd, Wd, Dd = X.to(dev), W.to(dev), D.to(dev)
    w_fwd, w_dgrad = api.NVFP4Tensor(n, m, dev), api.NVFP4Tensor(m, n, dev)
    ws = api.workspace(l, max(m, n), max(m, n), dev)
    torch.cuda.synchronize(dev)
    api.averis_quant_weight(Wd, w_fwd, w_dgrad, ws, stream)
    Y = torch.empty((l, n), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((l, m), dtype=torch.bfloat16, device=dev)
    xr, dr = api.NVFP4Tensor(l, m, dev), api.NVFP4Tensor(l, n, dev)
    muq, dmuq = api.NVFP4Tensor(1, m, dev), api.NVFP4Tensor(1, n, dev)

    def averis(i):
        api.averis_linear_fwd(Xd, w_fwd, "sr", 1 + i, 0, Y, ws, stream=stream)
        api.averis_linear_dgrad(Dd, w_dgrad, "sr", 1 + i, 0, dX, ws, stream=stream)

    def vanilla(i):
        api.nvfp4_linear_fwd(Xd, w_fwd, "sr", 1 + i, 0, Y, ws, stream=stream)
        api.nvfp4_linear_dgrad(Dd, w_dgrad, "sr", 1 + i, 0, dX, ws, stream=stream)

    t_a = avg_us(averis)
    t_v = avg_us(vanilla)
    sq_x = avg_us(lambda i: api.averis_split_quant(Xd, "sr", 1, 0, False, None, muq, xr, None, ws, stream))
    sq_d = avg_us(lambda i: api.averis_split_quant(Dd, "sr", 1, 0, True, None, dmuq, dr, None, ws, stream))
    g_f = avg_us(lambda i: api.nvfp4_gemm(xr, w_fwd, None, Y, ws, stream))
    g_d = avg_us(lambda i: api.nvfp4_gemm(dr, w_dgrad, None, dX, ws, stream))
    if api.averis_check_status(ws, stream):
        raise RuntimeError("device status set by the linear timing")
    flops = 2.0 * 2 * l * m * n
    gemm_tf = flops / ((g_f + g_d) * 1e-6) / 1e12
    del Xd, Wd, Dd, Y, dX, xr, dr
    return {"l": l, "m": m, "n": n, "averis_us": t_a, "vanilla_us": t_v,
            "averis_overhead_vs_vanilla": t_a / t_v - 1.0, "tflops": flops / (t_a * 1e-6) / 1e12,
            "split_quant_us": {"X": sq_x, "dY": sq_d}, "gemm_us": {"fwd": g_f, "dgrad": g_d},
            "gemm_tflops": gemm_tf, "gemm_frac_fp4_peak": gemm_tf / fp4_peak}


# ---------------------------------------------------------------------------
# the mean-strength sweep: the pages' effect measured on this library's output
# ---------------------------------------------------------------------------
E2M1_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def dequantize(q, dev):
    """value(code) * value(scale) * g_dec of a device NVFP4 tensor, fp32 on the
    device (codes two per byte, element 2k low; scales in the 128 x 4 atom
    layout).  A reporting aid of this script."""
    import torch
    R, K = q.rows, q.K
    lut = torch.tensor(E2M1_VALUES, dtype=torch.float32, device=dev)
    c = q.codes.to(torch.int64)
    vals = torch.stack([lut[c & 15], lut[c >> 4]], dim=-1).reshape(R, K)
    r = torch.arange(R, device=dev)[:, None]
    cb = torch.arange(K // 16, device=dev)[None, :]
    off = ((r // 128) * (K // 64) + cb // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + cb % 4
    sc = q.scales[off].view(torch.float8_e4m3fn).to(torch.float32)
    return vals * sc.repeat_interleave(16, dim=1) * q.g_dec.float()


def sweep_metrics(dev, stream, avg_us, rows_checked=256):
    """The mean-strength sweep (X [16384, 2048] = c 1 mu^T + rank-4 spike +
    N(0, 1), W [2048, 2048]) at c in {0, 0.5, 2, 8, 32}, stochastic rounding.
    Per c: entries over t = 3 and 4 (sigma of the Gaussian tail = 1) in X and
    in the residual X - 1 mu; the FP4 reconstruction error ||deq - X||_F /
    ||X||_F of vanilla Q4(X) and of Averis 1 deq(mu_bar) + deq(X_bar_R); the
    forward output's error against the fp64 product X W on sampled rows; and
    the Averis and vanilla forward times (split + GEMM)."""
    import torch
    from quantized_gemm_column_b200 import api, inputs
    out = []
    for c in inputs.WORKLOADS[3]["mean_scales"]:
        X, W = inputs.workload3(c)
        l, m = X.shape
        n = W.shape[1]
        Xd, Wd = X.to(dev), W.to(dev)
        w_fwd, w_dgrad = api.NVFP4Tensor(n, m, dev), api.NVFP4Tensor(m, n, dev)
        ws = api.workspace(l, max(m, n), max(m, n), dev)
        torch.cuda.synchronize(dev)
        api.averis_quant_weight(Wd, w_fwd, w_dgrad, ws, stream)
        mu = torch.empty(m, dtype=torch.float32, device=dev)
        xr, muq, xv = api.NVFP4Tensor(l, m, dev), api.NVFP4Tensor(1, m, dev), api.NVFP4Tensor(l, m, dev)
        api.averis_split_quant(Xd, "sr", 7, 0, False, mu, muq, xr, None, ws, stream)
        api.nvfp4_quant(Xd, "sr", 7, 0, False, xv, ws, stream)
        Ya = torch.empty((l, n), dtype=torch.bfloat16, device=dev)
        Yv = torch.empty((l, n), dtype=torch.bfloat16, device=dev)
        t_a = avg_us(lambda i: api.averis_linear_fwd(Xd, w_fwd, "sr", 7, 0, Ya, ws, stream=stream))
        t_v = avg_us(lambda i: api.nvfp4_linear_fwd(Xd, w_fwd, "sr", 7, 0, Yv, ws, stream=stream))
        if api.averis_check_status(ws, stream):
            raise RuntimeError("device status set by the sweep")
        with torch.cuda.stream(stream):
            x = Xd.float()
            xres = x - mu[None, :]
            over = {f"t{t}": {"X": int((x.abs() > t).sum().item()), "X_R": int((xres.abs() > t).sum().item())}
                    for t in (3, 4)}
            nx = torch.linalg.vector_norm(x).item()
            err_v = torch.linalg.vector_norm(dequantize(xv, dev) - x).item() / nx
            rec_a = dequantize(xr, dev) + dequantize(muq, dev)
            err_a = torch.linalg.vector_norm(rec_a - x).item() / nx
            del rec_a, xres
            rows = torch.randperm(l, generator=torch.Generator().manual_seed(5))[:rows_checked].to(dev)
            ref = Xd[rows].double() @ Wd.double()
            nref = torch.linalg.vector_norm(ref).item()
            gerr_a = torch.linalg.vector_norm(Ya[rows].double() - ref).item() / nref
            gerr_v = torch.linalg.vector_norm(Yv[rows].double() - ref).item() / nref
            torch.cuda.synchronize(dev)
        out.append({"c": c, "over_threshold": over, "elements": l * m,
                    "fp4_recon_rel_err": {"vanilla": err_v, "averis": err_a},
                    "gemm_rel_err_vs_fp64_xw": {"vanilla": gerr_v, "averis": gerr_a, "rows": rows_checked},
                    "fwd_us": {"averis": t_a, "vanilla": t_v}})
        del Xd, Wd, x, Ya, Yv, xr, xv
    return {"l": 16384, "m": 2048, "n": 2048, "rounding": "philox-sr", "per_c": out}


# ---------------------------------------------------------------------------
# CPU oracle baseline
# ---------------------------------------------------------------------------
def oracle_step(x, d, w_fwd_q, w_dgrad_q):
    """One forward + dgrad of the Averis linear in the oracle."""
    import oracle
    oracle.averis_linear_reference(x, w_fwd_q, "sr", seed=1, offset=0)
    oracle.averis_linear_reference(d, w_dgrad_q, "sr", seed=2, offset=0, grad=True)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_operands(rows):
    import oracle
    from quantized_gemm_column_b200 import inputs
    X, W, D = inputs.workload1()
    x = inputs.bf16_as_f32(X)[:rows]
    d = inputs.bf16_as_f32(D)[:rows]
    w_fwd_q, w_dgrad_q = oracle.quant_weight(inputs.bf16_as_f32(W))
    return x, d, w_fwd_q, w_dgrad_q


def cpu_baseline(rows, steps=1):
    x, d, wf, wd = oracle_operands(rows)
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle_step(x, d, wf, wd)
    dt = (time.perf_counter() - t0) / steps
    flops = 2 * (2 * rows * M * N)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"first {rows} of {L} tokens of X and dY (column mean, split, NVFP4 SR "
                      f"quantization and fp64 product of the sample), {steps} fwd+dgrad passes of "
                      f"{dt:.1f} s each"}


REF_WARMUP_S, REF_TIMED_S = 20.0, 120.0


def run_reference(args, rank, world):
    if rank != 0:
        return
    rows = 128
    x, d, wf, wd = oracle_operands(rows)
    # the oracle takes ~0.4 s a step (it decodes the weight every call): warm-up and timed steps
    # stop at a wall-clock budget so that a run with the GPU arm's step count still ends in minutes
    t0 = time.perf_counter()
    warm = 0
    while warm < args.warmup and (warm == 0 or time.perf_counter() - t0 < REF_WARMUP_S):
        oracle_step(x, d, wf, wd)
        warm += 1
    t0 = time.perf_counter()
    timed = 0
    while timed < args.steps and (timed == 0 or time.perf_counter() - t0 < REF_TIMED_S):
        oracle_step(x, d, wf, wd)
        timed += 1
    dt = (time.perf_counter() - t0) / timed
    value = 2 * (2 * rows * M * N) / dt / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": timed, "steps_requested": args.steps, "warmup": warm, "warmup_requested": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 product of e2m1 x e4m3 operands",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "l": L, "m": M, "n": N, "rounding": "philox-sr",
                   "parallelism": "single host process (rank 0)", "sample_rows": rows},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"first {rows} of {L} tokens per step, {timed} timed steps "
                                   f"(at most {REF_TIMED_S:.0f} s of steps)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# measured DRAM traffic (ncu), valid only for the kernel sources it was taken on
# ---------------------------------------------------------------------------
KERNEL_SOURCES = ["colreduce.cu", "quant.cu", "quant_common.cuh", "split_fused.cu", "gemm.cu", "gemm2.cu", "gemm3.cu", "pair.cuh",
                  "device.cuh", "internal.h"]
TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "traffic_qkv_step.json")


def kernel_digest():
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "quantized_gemm_column_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(key):
    """DRAM bytes per step of a kernel group ("split-quant" or "gemm") from the
    committed ncu capture (profiles/traffic_qkv_step.json), or None if it is
    missing or was taken on other kernel sources."""
    try:
        with open(TRAFFIC_PROFILE) as fh:
            rec = json.load(fh)
        if rec.get("digest") != kernel_digest():
            return None
        return int(rec["bytes_per_step"][key])
    except (OSError, KeyError, ValueError, TypeError):
        return None


# ---------------------------------------------------------------------------
# multi-rank plumbing (replicas; the only collective is this timing reduction)
# ---------------------------------------------------------------------------
def max_over_ranks(values, device):
    """Element-wise maximum of `values` over all ranks (identity on one rank).
    Every rank must call it at the same point; it runs outside the timed region."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_value(flops_per_step, world, step_ms):
    """Whole-job throughput (TFLOP/s): every rank runs its own step of
    flops_per_step; the slowest rank's step time counts."""
    return flops_per_step * world / (step_ms * 1e-3) / 1e12


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------
def run_case(args):
    """The QKV step's launches alone, for ncu captures: the weight
    quantization once, then args.warmup + args.steps Averis steps and as many
    vanilla steps (eager launches on one stream, inputs rotating over
    args.copies copies); the device status is checked at the end."""
    import torch
    from quantized_gemm_column_b200 import api, inputs
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    api.load()
    X0, W0, D0 = inputs.workload1()
    copies = max(1, args.copies)
    Xs = [X0.to(dev) for _ in range(copies)]
    Ds = [D0.to(dev) for _ in range(copies)]
    Wd = W0.to(dev)
    w_fwd, w_dgrad = api.NVFP4Tensor(N, M, dev), api.NVFP4Tensor(M, N, dev)
    ws = api.workspace(L, N, N, dev)
    Y = torch.empty((L, N), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((L, M), dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize(dev)
    api.averis_quant_weight(Wd, w_fwd, w_dgrad, ws)
    for i in range(args.warmup + args.steps):
        api.averis_linear_fwd(Xs[i % copies], w_fwd, "sr", 1 + i, 0, Y, ws)
        api.averis_linear_dgrad(Ds[i % copies], w_dgrad, "sr", 1 + i, 0, dX, ws)
    for i in range(args.warmup + args.steps):
        api.nvfp4_linear_fwd(Xs[i % copies], w_fwd, "sr", 1 + i, 0, Y, ws)
        api.nvfp4_linear_dgrad(Ds[i % copies], w_dgrad, "sr", 1 + i, 0, dX, ws)
    st = api.averis_check_status(ws)
    if st:
        raise RuntimeError(f"device status {st} in the profiling case")


def run_gpu(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from quantized_gemm_column_b200 import api, inputs

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    api.load()

    # inputs: `copies` replicas of (X, dY) so the rotating working set exceeds L2
    X0, W0, D0 = inputs.workload1(seed_tag=rank)
    copies = max(1, args.copies)
    Xs = [X0.to(dev) for _ in range(copies)]
    Ds = [D0.to(dev) for _ in range(copies)]
    Wd = W0.to(dev)
    w_fwd, w_dgrad = api.NVFP4Tensor(N, M, dev), api.NVFP4Tensor(M, N, dev)
    ws = api.workspace(L, N, N, dev)
    Y = torch.empty((L, N), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((L, M), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.Stream(dev)
    torch.cuda.synchronize(dev)                # staged on the default stream, consumed on `stream`

    def step(i, s=None):
        api.averis_linear_fwd(Xs[i % copies], w_fwd, "sr", 1 + i, 0, Y, ws, stream=s)
        api.averis_linear_dgrad(Ds[i % copies], w_dgrad, "sr", 1 + i, 0, dX, ws, stream=s)

    def vanilla_step(i, s=None):
        api.nvfp4_linear_fwd(Xs[i % copies], w_fwd, "sr", 1 + i, 0, Y, ws, stream=s)
        api.nvfp4_linear_dgrad(Ds[i % copies], w_dgrad, "sr", 1 + i, 0, dX, ws, stream=s)

    with torch.cuda.stream(stream):
        # weight quantization (once per weight update), timed alone
        api.averis_quant_weight(Wd, w_fwd, w_dgrad, ws, stream=stream)
        torch.cuda._sleep(20_000_000)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(10):
            api.averis_quant_weight(Wd, w_fwd, w_dgrad, ws, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        wq_us = e0.elapsed_time(e1) * 1e3 / 10
        for i in range(2):
            step(i, stream)
            vanilla_step(i, stream)
        torch.cuda.synchronize(dev)
    st = api.averis_check_status(ws, stream)
    if st:
        raise RuntimeError(f"device status {st} during warm-up")

    # CUDA graphs: one per input copy for the Averis step and the vanilla step
    graphs, vgraphs, launch = [], [], "cuda-graph"
    try:
        for i in range(copies):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                step(i, stream)
            graphs.append(g)
            vg = torch.cuda.CUDAGraph()
            with torch.cuda.graph(vg, stream=stream):
                vanilla_step(i, stream)
            vgraphs.append(vg)
    except Exception as exc:   # capture unsupported: time eager launches instead
        graphs, vgraphs, launch = [], [], f"eager ({type(exc).__name__})"
        torch.cuda.synchronize(dev)

    def replay(i, vanilla=False):
        if graphs:
            (vgraphs if vanilla else graphs)[i % copies].replay()
        else:
            (vanilla_step if vanilla else step)(i, stream)

    def timed(n, vanilla=False):
        with torch.cuda.stream(stream):
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize(dev)
            torch.cuda._sleep(5_000_000)            # let the host run ahead of the device
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for i in range(n):
                replay(i, vanilla)
            b.record(stream)
            torch.cuda.synchronize(dev)
            if world > 1:
                dist.barrier()
            return a.elapsed_time(b)                # ms

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            replay(i)
            replay(i, True)
        torch.cuda.synchronize(dev)

    with ClockSampler(local_rank) as clk:
        t0 = time.monotonic()
        ms = timed(args.steps)
        ms_van = timed(args.steps, vanilla=True)
        clk.region(t0, time.monotonic())
    clocks = clk.summary()
    st = api.averis_check_status(ws, stream)
    if st:
        raise RuntimeError(f"device status {st} in the timed region")

    ms, ms_van = max_over_ranks([ms, ms_van], dev)
    step_ms = ms / args.steps
    value = job_value(FLOPS_PER_STEP, world, step_ms)

    # per-step distribution (beside the headline): each replay bracketed by its
    # own events, warm (back to back) and with L2 flushed before every step
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # 256 MiB > 126 MB of L2

    def step_distribution(n, vanilla=False, cold=False):
        pairs = []
        with torch.cuda.stream(stream):
            for i in range(3):
                replay(i, vanilla)
            torch.cuda.synchronize(dev)
            for i in range(n):
                if cold:
                    flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                replay(i, vanilla)
                b.record(stream)
                pairs.append((a, b))
            torch.cuda.synchronize(dev)
        us = sorted(a.elapsed_time(b) * 1e3 for a, b in pairs)
        q = lambda f: us[min(len(us) - 1, int(round(f * (len(us) - 1))))]
        return {"median_us": q(0.5), "p10_us": q(0.1), "p90_us": q(0.9), "steps": n}

    n_dist = 200
    dist_steps = {"averis": {"warm": step_distribution(n_dist), "cold_l2": step_distribution(n_dist, cold=True)},
                  "vanilla": {"warm": step_distribution(n_dist, True),
                              "cold_l2": step_distribution(n_dist, True, cold=True)}}
    del flush

    # sustained: the Averis step replayed back to back for about two seconds
    # (long enough to meet the power cap), SM clocks sampled inside the region
    n_sus = max(args.steps, int(2.0 / (step_ms * 1e-3)))
    with torch.cuda.stream(stream):
        torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clk_sus:
        t0 = time.monotonic()
        ms_sus = timed(n_sus)
        clk_sus.region(t0, time.monotonic())
    sus_step_ms = ms_sus / n_sus
    sustained = {"steps": n_sus, "ms_per_step": sus_step_ms,
                 "tflops": FLOPS_PER_STEP / (sus_step_ms * 1e-3) / 1e12, "clocks": clk_sus.summary()}

    # per-kernel-group timing (same stream, events around n launches each)
    xr = api.NVFP4Tensor(L, M, dev)
    dr = api.NVFP4Tensor(L, N, dev)
    muq, dmuq = api.NVFP4Tensor(1, M, dev), api.NVFP4Tensor(1, N, dev)

    def avg_us(fn, n=20):
        with torch.cuda.stream(stream):
            for i in range(3):
                fn(i)
            torch.cuda.synchronize(dev)
            torch.cuda._sleep(5_000_000)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for i in range(n):
                fn(i)
            b.record(stream)
            torch.cuda.synchronize(dev)
        return a.elapsed_time(b) * 1e3 / n

    sq_x = avg_us(lambda i: api.averis_split_quant(Xs[i % copies], "sr", 1, 0, False, None, muq, xr, None, ws, stream))
    sq_d = avg_us(lambda i: api.averis_split_quant(Ds[i % copies], "sr", 1, 0, True, None, dmuq, dr, None, ws, stream))
    # the one-kernel split (same bits), for comparison with the two-kernel chain above
    fs_x = avg_us(lambda i: api.averis_split_quant_fused(Xs[i % copies], "sr", 1, 0, False, None, muq, xr, ws, stream))
    fs_d = avg_us(lambda i: api.averis_split_quant_fused(Ds[i % copies], "sr", 1, 0, True, None, dmuq, dr, ws, stream))
    g_f = avg_us(lambda i: api.nvfp4_gemm(xr, w_fwd, None, Y, ws, stream))
    g_d = avg_us(lambda i: api.nvfp4_gemm(dr, w_dgrad, None, dX, ws, stream))
    gemm_tflops = 2 * L * M * N * 2 / ((g_f + g_d) * 1e-6) / 1e12

    # the weight gradient dW = X^T dY (beyond the timed fwd + dgrad step):
    # two token-axis splits, the rank-one factors and the GEMM, fp32 dW
    wws = api.wgrad_workspace(L, M, N, dev)
    dW = torch.empty((M, N), dtype=torch.float32, device=dev)
    wg_a = avg_us(lambda i: api.averis_linear_wgrad(Xs[i % copies], Ds[i % copies], "sr", 1, 0, dW, wws, stream))
    wg_v = avg_us(lambda i: api.nvfp4_linear_wgrad(Xs[i % copies], Ds[i % copies], "sr", 1, 0, dW, wws, stream))
    Lp = api.padded_tokens(L)
    xt_q, dt_q = api.NVFP4Tensor(M, Lp, dev), api.NVFP4Tensor(N, Lp, dev)
    sqt_x = avg_us(lambda i: api.averis_split_quant_t(Xs[i % copies], "sr", 1, 0, False, None, muq, xt_q, ws, stream))
    sqt_d = avg_us(lambda i: api.averis_split_quant_t(Ds[i % copies], "sr", 1, 0, True, None, dmuq, dt_q, ws, stream))
    g_w = avg_us(lambda i: api.averis_wgrad_gemm(xt_q, dt_q, muq, dmuq, L, dW, wws, stream))
    if api.averis_check_status(wws, stream) or api.averis_check_status(ws, stream):
        raise RuntimeError("device status set by the weight-gradient timing")
    wgrad = {"dW": f"fp32 [{M}, {N}], contraction over {L} tokens", "averis_us": wg_a, "vanilla_us": wg_v,
             "averis_overhead_vs_vanilla": wg_a / wg_v - 1.0,
             "tflops": 2 * L * M * N / (wg_a * 1e-6) / 1e12,
             "split_quant_t_us": {"X": sqt_x, "dY": sqt_d}, "gemm_us": g_w,
             "gemm_tflops": 2 * L * M * N / (g_w * 1e-6) / 1e12}

    moe = moe_timing(dev, stream, avg_us)
    fp4 = fp4_ceiling(dev, stream)
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        pass
    bf16_peak = peaks.get("bf16_tflops", 1590.0)
    fp4_nominal = 4.0 * bf16_peak          # nominal dense FP4 : BF16 ratio 9 : 2.25
    fp4_peak = fp4["mma_loop_tflops"] or fp4_nominal
    fp4["bf16x4_nominal_tflops"] = fp4_nominal
    # the FFN projections of the Qwen3-0.6B layer at 16384 tokens, one linear at a time
    from quantized_gemm_column_b200 import inputs
    gX = inputs.to_bf16(inputs.spiked_activations(inputs.rng_for(2, 1), 16384, 1024, rank=4,
                                                  s=(16.0, 8.0, 6.0, 4.0), n_hot=10))
    gW = inputs.to_bf16(inputs.weight(inputs.rng_for(2, 2), 1024, 6144))
    gD = inputs.to_bf16(inputs.output_gradient(inputs.rng_for(2, 3), 16384, 6144))
    ffn = {"gate_up": linear_timing(dev, stream, avg_us, gX, gW, gD, fp4_peak)}
    del gX, gW, gD
    dXin, dWin, dDin = inputs.workload2_down()
    ffn["down"] = linear_timing(dev, stream, avg_us, dXin, dWin, dDin, fp4_peak)
    del dXin, dWin, dDin
    sweep = sweep_metrics(dev, stream, avg_us)
    stack = stack_timing(dev, stream)

    # split-quant algorithmic bytes: read the input twice (reduce, quantize),
    # write codes (1/2 byte per element) and scales (1/16 byte per element)
    def sq_bytes(rows, K):
        return rows * K * (2 * 2 + 0.5 + 1.0 / 16)
    sq_gbs = (sq_bytes(L, M) + sq_bytes(L, N)) / ((sq_x + sq_d) * 1e-6) / 1e9

    hbm_peak = peaks.get("hbm_gbs", 6650.0)
    peak_src = "measured" if peaks else "fallback"

    # dominant kernel group by time share of the step
    gemm_share = (g_f + g_d) / (step_ms * 1e3)
    if gemm_share >= 0.5:
        roof = {"bound": "tensor", "kernel": "gemm2_nvfp4_kernel (fwd + dgrad)",
                "achieved": gemm_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
                "frac": gemm_tflops / fp4_peak, "traffic": measured_traffic("gemm"),
                "traffic_unit": "DRAM bytes per step (fwd + dgrad launches)",
                "peak_source": "measured: this device's MMA-only tcgen05 FP4 loop",
                "peak_bf16x4_nominal": fp4_nominal}
    else:
        roof = {"bound": "hbm", "kernel": "colreduce_kernel + fold_kernel + quant_kernel (split-quant, X and dY)",
                "achieved": sq_gbs, "peak": hbm_peak, "unit": "GB/s", "frac": sq_gbs / hbm_peak,
                "traffic": measured_traffic("split-quant"),
                "traffic_unit": "DRAM bytes per step (6 launches: reduce, fold and quantize, X and dY)",
                "algorithmic_bytes_per_step": sq_bytes(L, M) + sq_bytes(L, N),
                "peak_source": f"{peak_src} HBM copy"}

    # end to end through the public API with host buffers: every step copies
    # its inputs in from pinned host memory and its outputs back; the copies of
    # neighbouring steps overlap the kernels (an upload stream, the compute
    # stream, a download stream; inputs and outputs double-buffered)
    Xh = [X0.pin_memory(), X0.clone().pin_memory()]
    Dh = [D0.pin_memory(), D0.clone().pin_memory()]
    Yh = [torch.empty((L, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    dXh = [torch.empty((L, M), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    Xe, De = [Xs[0], Xs[1 % copies]], [Ds[0], Ds[1 % copies]]
    Ye = [Y, torch.empty_like(Y)]
    dXe = [dX, torch.empty_like(dX)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "comp", "out")}

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(ev["comp"][b])          # step i-2 has read this input buffer
            Xe[b].copy_(Xh[b], non_blocking=True)
            De[b].copy_(Dh[b], non_blocking=True)
            ev["in"][b].record(up)
        stream.wait_event(ev["in"][b])
        if i >= 2:
            stream.wait_event(ev["out"][b])           # step i-2's outputs have left this buffer
        api.averis_linear_fwd(Xe[b], w_fwd, "sr", 1 + i, 0, Ye[b], ws, stream=stream)
        api.averis_linear_dgrad(De[b], w_dgrad, "sr", 1 + i, 0, dXe[b], ws, stream=stream)
        ev["comp"][b].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(ev["comp"][b])
            Yh[b].copy_(Ye[b], non_blocking=True)
            dXh[b].copy_(dXe[b], non_blocking=True)
            ev["out"][b].record(down)

    e2e_steps = max(3, min(args.steps, 20))
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    a, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    up.wait_event(a)
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_stream(down)
    stream.wait_stream(up)
    b_ev.record(stream)
    torch.cuda.synchronize(dev)
    b = b_ev
    e2e_ms = max_over_ranks([a.elapsed_time(b) / e2e_steps], dev)[0]
    e2e_val = job_value(FLOPS_PER_STEP, world, e2e_ms)
    h2d = (X0.numel() + D0.numel()) * 2
    d2h = (Y.numel() + dX.numel()) * 2
    if api.averis_check_status(ws, stream):
        raise RuntimeError("device status set by the end-to-end run")

    if rank != 0:
        return
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        cpu = cpu_baseline(args.cpu_sample_rows, args.cpu_sample_steps)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e2m1 x e2m1 (e4m3 block scales) -> fp32 accumulate",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "l": L, "m": M, "n": N, "rounding": "philox-sr",
                   "parallelism": f"replicas x{world}" if world > 1 else "single gpu",
                   "launch": launch,
                   "l2": f"inputs rotate over {copies} copies of (X, dY) = "
                         f"{copies * (L * M + L * N) * 2 / 2**20:.0f} MiB > 126 MB L2"},
        "split_quant_gbs": sq_gbs,
        "split_quant_us": {"X": sq_x, "dY": sq_d},
        "split_quant_fused_us": {"X": fs_x, "dY": fs_d},
        "gemm_us": {"fwd": g_f, "dgrad": g_d}, "gemm_tflops": gemm_tflops,
        "wgrad": wgrad,
        "moe": moe,
        "stack": stack,
        "gemm_frac_fp4_peak": gemm_tflops / fp4_peak,
        "fp4_ceiling": fp4,
        "ffn": ffn,
        "sweep": sweep,
        "vanilla_ms_per_step": ms_van / args.steps,
        "averis_overhead_vs_vanilla": (ms / ms_van) - 1.0,
        "weight_quant_us": wq_us,
        "roofline": roof,
        "step_us_distribution": dist_steps,
        "sustained": sustained,
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                   "reasons": clocks["reasons"], "samples_in_region": clocks["samples_in_region"]},
        "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms,
                "copies": "pinned host <-> device every step, overlapping the neighbouring steps' kernels "
                          "(upload, compute and download streams; double-buffered)"},
        # per step: column reduce, fold, quantizer and GEMM, for the forward and for the dgrad
        "gpu_launches": 8 * args.steps,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    for g in graphs + vgraphs:
        del g


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.case is not None:
        run_case(args)
        return
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
