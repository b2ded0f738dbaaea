"""Benchmark of the 4-bit linear layer on B200: one step = the forward and backward
passes of every projection of a Llama-3.1-8B transformer layer (QKV, O, gate, up,
down) on 8192 tokens, each pass rotated (H16), quantised (MXFP4) and multiplied on
the FP4 tensor cores:

    per projection: dual-layout quantise of X, W and dY (3 kernels),
                    Fprop Y = X W^T (bf16 out), Dgrad dX = dY W (bf16 out),
                    Wgrad dW = dY^T X (fp32 out)  -> 3 GEMM kernels
    with N > 1 ranks: data parallel over tokens (8192 per rank), dW all-reduced
    (NCCL) per projection, overlapped with the next projection.

The quantisation of projection p+1 runs on a second stream beside the GEMMs of
projection p (--side-stream 1, the default), filling the SMs their last tile wave
leaves idle; per-kernel rooflines are then timed on the same steps run on one stream.

Prints ONE JSON line (rank 0). `value` is the step's GEMM FLOPs divided by the step
time (quantisation included), summed over ranks. Inputs are synthetic, seeded, and
resident in HBM before the timed region; the step's working set (~4 GB) is far
larger than L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fp4|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FP4 GEMM TFLOPS (fprop/dgrad/wgrad) + H16-quantize GB/s, % of B200 roofline"
FP4_OVER_BF16 = 4.0  # nominal dense FP4 : BF16 tensor throughput (9 : 2.25 PFLOP/s)
FP8_OVER_BF16 = 2.0  # nominal dense FP8 : BF16 (4.5 : 2.25 PFLOP/s), for the MXFP8 comparator
DATASHEET_TFLOPS = {"fp4": 9000.0, "fp8": 4500.0}  # B200 dense tensor peaks (HGX datasheet)
FORMATS = {"mxfp4": 0, "nvfp4": 1, "mxfp8": 2}
PEAK_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
WORKLOAD = ("llama3.1-8b layer fwd+bwd: qkv 6144x4096, o 4096x4096, gate/up 14336x4096, "
            "down 4096x14336; 8192 tokens/rank; MXFP4 + H16")


WORKLOAD_GPT3 = ("gpt3-175b layer fwd+bwd: qkv 36864x12288, o 12288x12288, fc1 49152x12288, "
                 "fc2 12288x49152; 4096 tokens/rank")


def layer_table(a):
    """(projections (name, N, K), tokens, X outlier factor) of the workload."""
    from fp4_block_scaled_deterministic_b200 import synthetic
    if a.workload == "gpt3":
        return synthetic.GPT3_LAYERS, synthetic.GPT3_TOKENS, 100.0
    return synthetic.LLAMA_LAYERS, 8192, 50.0


def workload_name(a) -> str:
    """WORKLOAD for the default run; the same layer with the format / rotation / quantiser
    variant actually run otherwise."""
    if (a.workload == "llama" and a.format == "mxfp4" and a.hadamard == 16 and a.variant == "none"
            and getattr(a, "next_layer_quant", "none") == "none"):
        return WORKLOAD
    tag = f"{a.format.upper()} + " + (f"H{a.hadamard}" if a.hadamard else "no rotation")
    if a.variant != "none":
        tag += f" + {a.variant} quantiser variant"
    if getattr(a, "next_layer_quant", "none") != "none":
        tag += f" + Y quantised for the next layer ({a.next_layer_quant})"
    base = WORKLOAD_GPT3 if a.workload == "gpt3" else WORKLOAD.rsplit(";", 1)[0]
    return base + "; " + tag


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["fp4", "reference"], default="fp4")
    ap.add_argument("--format", choices=list(FORMATS), default="mxfp4",
                    help="mxfp8 = the FP8 comparator (E4M3, E8M0 scale per 32) on the same step")
    ap.add_argument("--hadamard", type=int, default=16, choices=[0, 16, 32])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=20.0,
                    help="oracle seconds of the CPU baseline (half on one thread, half on all)")
    ap.add_argument("--cpu-budget", type=float, default=None,
                    help="reference arm: oracle seconds per step (default: fills ~2 minutes)")
    ap.add_argument("--proj", default="qkv,o,gate,up,down",
                    help="comma-separated subset of the layer's projections (profiling cases)")
    ap.add_argument("--workload", choices=["llama", "gpt3"], default="llama",
                    help="gpt3: the GPT-3 175B layer shapes on 4096 tokens (a parity config, "
                         "measured for the record; the headline line is the Llama layer)")
    ap.add_argument("--library-compare", action="store_true",
                    help="GEMM only: this library's block-scaled GEMM against the library kernel "
                         "torch runs for the same format (torch.nn.functional.scaled_mm) on the "
                         "layer's GEMM shapes, same operands; one JSON line per shape + totals")
    ap.add_argument("--sweep", action="store_true",
                    help="quantise-only bandwidth sweep (one JSON line per case) instead of the step")
    ap.add_argument("--side-stream", type=int, default=1, choices=[0, 1],
                    help="1: quantise the next projection on a second stream beside the GEMMs "
                         "(per-kernel rooflines then come from the same steps on one stream)")
    ap.add_argument("--quant-batch", type=int, default=1, choices=[0, 1],
                    help="1: quantise each projection's X, W and dY in one batched launch "
                         "(fp4_quantize_dual_batch); 0: one launch per tensor")
    ap.add_argument("--gemm-group", type=int, default=1, choices=[0, 1],
                    help="1: a projection's Fprop, Dgrad and Wgrad GEMMs in one launch "
                         "(fp4_gemm_group; fp4_gemm_group_quant with --next-layer-quant "
                         "fused); 0: one launch per GEMM")
    ap.add_argument("--next-layer-quant", choices=["none", "standalone", "fused"], default="none",
                    help="also quantise each Fprop output Y row-wise (MXFP4, same rotation) for "
                         "the next layer: by a separate quantise launch after the GEMM, or in "
                         "the GEMM's epilogue (fp4_gemm_group_quant; fp4_gemm_quant with "
                         "--gemm-group 0)")
    ap.add_argument("--variant", choices=["none", "sr", "rht", "sr+rht", "amax"], default="none",
                    help="quantiser variant: stochastic rounding, randomised Hadamard signs, "
                         "both, or (NVFP4) a supplied tensor amax instead of the amax pass")
    a = ap.parse_args()
    a.warmup = max(3, a.warmup)
    if a.variant == "amax" and a.format != "nvfp4":
        ap.error("--variant amax needs --format nvfp4")
    if a.next_layer_quant != "none" and a.format != "mxfp4":
        ap.error("--next-layer-quant quantises Y as MXFP4: it needs --format mxfp4")
    return a


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d, "measured"
    return dict(PEAK_FALLBACK), "fallback"


# ---------------------------------------------------------------- clocks sampler
class Clocks:
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.sw_power_cap,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown")

    def __init__(self, dev: int):
        self.dev, self.proc, self.lines = dev, None, []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ("sw_power_cap", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")
        for ln in self.lines:
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 6:
                continue
            try:
                sm.append(float(p[0]))
                mx.append(float(p[1]))
            except ValueError:
                continue
            for n, v in zip(names, p[2:6]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


class NvmlClocks:
    """SM clock and clock-event reasons read through NVML every few milliseconds, so
    that windows of a few hundred milliseconds (the per-kernel timing pass, the timed
    region) get tens of samples; window(t0, t1) summarises those in [t0, t1] (host
    perf_counter seconds). Reads only: nothing is set."""
    REASONS = (("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"))

    def __init__(self, dev: int, period_s: float = 0.005):
        self.dev, self.period, self.samples, self.ok = dev, period_s, [], False
        self.stop_flag = threading.Event()

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(self.dev)
            self.bits = {n: getattr(pynvml, c) for n, c in self.REASONS}
            self.ok = True
        except Exception:  # no NVML: the nvidia-smi sampler still reports
            return
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()

    def _run(self):
        nv = self.nv
        while not self.stop_flag.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                break
            self.samples.append((time.perf_counter(), mhz, rs))
            time.sleep(self.period)

    def stop(self):
        self.stop_flag.set()
        if self.ok:
            self.t.join(timeout=2)

    def window(self, t0: float, t1: float):
        w = [(m, r) for t, m, r in self.samples if t0 <= t <= t1]
        if not w:
            return None
        mhz = sorted(m for m, _ in w)
        reasons = sorted(n for n, b in self.bits.items() if any(r & b for _, r in w))
        return {"sm_mhz_median": statistics.median(mhz), "sm_mhz_min": mhz[0],
                "sm_mhz_max": mhz[-1], "samples": len(w), "reasons": reasons}


# ---------------------------------------------------------------- workload
class LlamaLayer:
    """Inputs, quantised operands and outputs of every projection, all on the device."""

    def __init__(self, device, fmt, hn, tokens=8192, seed=0, names=None, variant="none",
                 side_stream=False, layers=None, outlier_mult=50.0, w_seed=0, next_quant="none",
                 quant_batch=True, gemm_group=True):
        import fp4_block_scaled_deterministic_b200 as fp4
        from fp4_block_scaled_deterministic_b200 import synthetic
        self.fp4, self.fmt, self.hn, self.M = fp4, fmt, hn, tokens
        self.variant = variant
        self.next_quant = next_quant
        # the plain quantiser takes a projection's three tensors in one batched launch
        self.quant_batch = quant_batch and variant == "none"
        self.gemm_group = gemm_group
        self.qstream = torch.cuda.Stream(device) if side_stream else None
        self.projs = []
        g = torch.Generator(device=device)
        for i, (name, N, K) in enumerate(layers or synthetic.LLAMA_LAYERS):
            if names is not None and name not in names:
                continue
            X = synthetic.normal(tokens, K, 1.0, seed=seed + i, outlier_frac=0.001,
                                 outlier_mult=outlier_mult, device=device)
            W = synthetic.normal(N, K, 0.02, seed=w_seed + 100 + i, device=device)
            dY = synthetic.heavy_tailed_grad(tokens, N, 1e-3, seed=seed + 200 + i, device=device)
            p = {"name": name, "N": N, "K": K, "X": X, "W": W, "dY": dY}
            for key, (r, c) in (("X", (tokens, K)), ("W", (N, K)), ("dY", (tokens, N))):
                p[key + "_row"] = self._qbuf(r, c, device)
                p[key + "_col"] = self._qbuf(c, r, device)
                p[key + "_ts"] = torch.zeros(4, dtype=torch.float32, device=device)
            p["Y"] = torch.empty(tokens, N, dtype=torch.bfloat16, device=device)
            if next_quant != "none":  # Y quantised row-wise (along N) for the next layer
                p["Yq"] = self._qbuf(tokens, N, device)
            p["dX"] = torch.empty(tokens, K, dtype=torch.bfloat16, device=device)
            p["dW"] = torch.empty(N, K, dtype=torch.float32, device=device)
            self.projs.append(p)
        del g
        if variant == "amax":
            # the supplied amax is that of an earlier quantisation of the same tensor: run
            # one plain quantisation now; its {amax_row, amax_col} (ts[2:4]) stay in place
            for p in self.projs:
                for key, (r, c) in self._operands(p):
                    row, col, ts = p[key + "_row"], p[key + "_col"], p[key + "_ts"]
                    st = fp4.fp4_quantize_dual(p[key], row[0], row[1], col[0], col[1], ts, r, c,
                                               fmt, hn, torch.cuda.current_stream().cuda_stream)
                    assert st == 0
        self.gemms_done, self.quant_done = [], []
        self.opts = {}
        for p in self.projs:
            # batched quantisation: one fp4_quant_item per operand, built once
            p["qitems"] = (fp4.QuantItem * 3)(*[
                fp4.QuantItem(p[key].data_ptr(), p[key + "_row"][0].data_ptr(),
                              p[key + "_row"][1].data_ptr(), p[key + "_col"][0].data_ptr(),
                              p[key + "_col"][1].data_ptr(),
                              p[key + "_ts"].data_ptr() if fmt == 1 else None, r, c)
                for key, (r, c) in self._operands(p)])
            # the GEMMs of the projection in one fp4_gemm_group launch, built once:
            # Fprop (member 0; with the fused epilogue it also quantises Y), Dgrad, Wgrad
            ts = (lambda k, i: p[k + "_ts"][i:i + 1].data_ptr()) if fmt == 1 else (lambda k, i: None)
            M, N, K = tokens, p["N"], p["K"]
            descs = [(p["X_row"], p["W_row"], "X", "W", 0, 0, p["Y"], M, N, K, 1),
                     (p["dY_row"], p["W_col"], "dY", "W", 0, 1, p["dX"], M, K, N, 1),
                     (p["dY_col"], p["X_col"], "dY", "X", 1, 1, p["dW"], N, K, M, 0)]
            p["gdescs"] = (fp4.GemmDesc * len(descs))(*[
                fp4.GemmDesc(a[0].data_ptr(), a[1].data_ptr(), ts(ka, ia), b[0].data_ptr(),
                             b[1].data_ptr(), ts(kb, ib), out.data_ptr(), m, n, k, od)
                for a, b, ka, kb, ia, ib, out, m, n, k, od in descs])
            for key, _ in self._operands(p):
                o = None
                if variant == "amax":
                    o = fp4.QuantOpts(p[key + "_ts"].data_ptr() + 8, 0, 0, 0, 0)
                elif variant != "none":
                    o = fp4.QuantOpts(None, int("sr" in variant), int("rht" in variant),
                                      0x5EED0000 + seed, 0x51600000 + seed)
                self.opts[(p["name"], key)] = o
        for _ in self.projs:
            for lst in (self.gemms_done, self.quant_done):
                ev = torch.cuda.Event()
                ev.record(torch.cuda.current_stream(device))
                lst.append(ev)

    def _operands(self, p):
        return (("X", (self.M, p["K"])), ("W", (p["N"], p["K"])), ("dY", (self.M, p["N"])))

    def _qbuf(self, r, c, device):
        f = self.fp4
        return (torch.empty(r, c if self.fmt == 2 else c // 2, dtype=torch.uint8, device=device),
                torch.empty(f.fp4_scales_bytes(r, c, self.fmt), dtype=torch.uint8, device=device))

    def flops(self):
        return sum(3 * 2.0 * self.M * p["N"] * p["K"] for p in self.projs)

    def quant_elems(self):
        return sum(self.M * p["K"] + p["N"] * p["K"] + self.M * p["N"] for p in self.projs)

    def bytes_in(self):
        return sum(t.numel() * t.element_size() for p in self.projs for t in (p["X"], p["W"], p["dY"]))

    def bytes_out(self):
        return sum(t.numel() * t.element_size() for p in self.projs for t in (p["Y"], p["dX"], p["dW"]))

    def gemm_launches(self):
        """GEMM launches of a projection: one group or three."""
        return 1 if self.gemm_group else 3

    def launches_per_step(self):
        # NVFP4 adds the amax pass (plus a memset) unless the amax is supplied
        per_q = 1 if self.fmt != 1 or self.variant == "amax" else 2
        q_launches = per_q if self.quant_batch else 3 * per_q
        return len(self.projs) * (q_launches + self.gemm_launches() +
                                  (self.next_quant == "standalone"))

    def step(self, stream, timers=None, allreduce=None, overlap=None, inputs_ready=None,
             outputs_free=None):
        """One fwd+bwd pass over every projection. timers: dict kind -> list of event
        pairs to record around each quantise / GEMM launch. overlap: quantise on the
        side stream (default: when the layer has one). inputs_ready[i] / outputs_free[i]:
        events the quantisation / the GEMMs of projection i wait for (the end-to-end
        copies); self.quant_done[i] and self.gemms_done[i] are recorded after them."""
        f, fmt, hn = self.fp4, self.fmt, self.hn
        if overlap is None:
            overlap = self.qstream is not None
        s = stream.cuda_stream
        pending = []

        def timed(kind, fn, on=None):
            on = stream if on is None else on
            if timers is None:
                return fn()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(on)
            r = fn()
            e1.record(on)
            timers[kind].append((e0, e1))
            return r

        def quantise(p, qstream):
            i = self.projs.index(p)
            if inputs_ready is not None:
                qstream.wait_event(inputs_ready[i])
            qs = qstream.cuda_stream
            if self.quant_batch:
                st = timed("quant", lambda: f.lib().fp4_quantize_dual_batch(
                    p["qitems"], 3, fmt, hn, qs), qstream)
                assert st == 0, f.status_string(st)
                return
            for key, (r, c) in self._operands(p):
                row, col, ts = p[key + "_row"], p[key + "_col"], p[key + "_ts"]
                opts = self.opts[(p["name"], key)]
                if opts is None:
                    st = timed("quant", lambda: f.fp4_quantize_dual(
                        p[key], row[0], row[1], col[0], col[1], ts if fmt == 1 else None, r, c,
                        fmt, hn, qs), qstream)
                else:
                    st = timed("quant", lambda: f.fp4_quantize_dual_opts(
                        p[key], row[0], row[1], col[0], col[1], ts if fmt == 1 else None, r, c,
                        fmt, hn, opts, qs), qstream)
                assert st == 0, f.status_string(st)

        # With a side stream the quantisation of projection p+1 runs beside the GEMMs of
        # projection p (it fills the SMs their last tile wave leaves idle). Events order
        # each GEMM after its operands' quantisation, and each quantisation after the
        # previous step's GEMMs that read the buffers it overwrites.
        side = self.qstream if overlap else None
        if side is not None:
            start = torch.cuda.Event()
            start.record(stream)          # inputs written on the main stream (e2e copies)
            side.wait_event(start)
            ready = []
            for i, p in enumerate(self.projs):
                side.wait_event(self.gemms_done[i])
                quantise(p, side)
                self.quant_done[i].record(side)
                ready.append(self.quant_done[i])
        for i, p in enumerate(self.projs):
            if side is None:
                quantise(p, stream)
                self.quant_done[i].record(stream)
            else:
                stream.wait_event(ready[i])
            if outputs_free is not None:
                stream.wait_event(outputs_free[i])
            tsx, tsw, tsy = p["X_ts"], p["W_ts"], p["dY_ts"]
            nv = fmt == 1
            M, N, K = self.M, p["N"], p["K"]
            if self.gemm_group:
                # Fprop, Dgrad and Wgrad in one launch; with the fused epilogue the Fprop's
                # epilogue also quantises Y (member 0 of the group)
                gd = p["gdescs"]
                if self.next_quant == "fused":
                    yq = p["Yq"]
                    st = timed("gemm", lambda: f.lib().fp4_gemm_group_quant(
                        gd, len(gd), fmt, 0, yq[0].data_ptr(), yq[1].data_ptr(), hn, s))
                else:
                    st = timed("gemm", lambda: f.lib().fp4_gemm_group(gd, len(gd), fmt, s))
                assert st == 0, f.status_string(st)
                if self.next_quant == "standalone":  # Q_row(Y) by a separate launch
                    st = timed("quant_y", lambda: f.fp4_quantize(
                        p["Y"], p["Yq"][0], p["Yq"][1], None, M, N, fmt, hn, 0, s))
                    assert st == 0
                self.gemms_done[i].record(stream)
                if allreduce is not None:
                    pending.append(allreduce(p["dW"]))
                continue
            # Fprop: Y[M][N] = X_row . W_row^T
            if self.next_quant == "fused":  # and Q_row(Y) from the same epilogue
                st = timed("gemm", lambda: f.fp4_gemm_quant(
                    p["X_row"][0], p["X_row"][1], None, p["W_row"][0], p["W_row"][1], None,
                    p["Y"], p["Yq"][0], p["Yq"][1], M, N, K, fmt, hn, s))
            else:
                st = timed("gemm", lambda: f.fp4_gemm(
                    p["X_row"][0], p["X_row"][1], tsx[0:1] if nv else None, p["W_row"][0],
                    p["W_row"][1], tsw[0:1] if nv else None, p["Y"], M, N, K, fmt, 1, s))
            assert st == 0
            if self.next_quant == "standalone":  # Q_row(Y) by a separate launch
                st = timed("quant_y", lambda: f.fp4_quantize(
                    p["Y"], p["Yq"][0], p["Yq"][1], None, M, N, fmt, hn, 0, s))
                assert st == 0
            # Dgrad: dX[M][K] = dY_row . W_col^T  (contraction over N)
            st = timed("gemm", lambda: f.fp4_gemm(
                p["dY_row"][0], p["dY_row"][1], tsy[0:1] if nv else None, p["W_col"][0],
                p["W_col"][1], tsw[1:2] if nv else None, p["dX"], M, K, N, fmt, 1, s))
            assert st == 0
            # Wgrad: dW[N][K] = dY_col . X_col^T  (contraction over the tokens)
            st = timed("gemm", lambda: f.fp4_gemm(
                p["dY_col"][0], p["dY_col"][1], tsy[1:2] if nv else None, p["X_col"][0],
                p["X_col"][1], tsx[1:2] if nv else None, p["dW"], N, K, M, fmt, 0, s))
            assert st == 0
            self.gemms_done[i].record(stream)
            if allreduce is not None:
                pending.append(allreduce(p["dW"]))
        for w in pending:
            w.wait()


def gemm_flops_of(layer):
    """Flops of each GEMM launch of one step, in launch order."""
    per = []
    for p in layer.projs:
        one = 2.0 * layer.M * p["N"] * p["K"]
        per += [one] * 3 if not layer.gemm_group else [3 * one]
    return per


# ---------------------------------------------------------------- CPU baseline
def host_facts() -> dict:
    """The host the CPU baseline ran on: logical CPUs, the affinity mask of this
    process, and the CPU model."""
    model = None
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                model = ln.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    aff = sorted(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else []
    runs, start = [], None
    for i, c in enumerate(aff):  # compress the mask to ranges, e.g. "0-63,128-191"
        if start is None:
            start = c
        if i + 1 == len(aff) or aff[i + 1] != c + 1:
            runs.append(f"{start}-{c}" if c != start else f"{c}")
            start = None
    return {"cpu_count": os.cpu_count(), "affinity": ",".join(runs),
            "affinity_cpus": len(aff), "cpu_model": model}


def host_threads() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


def cpu_oracle_rate(seconds_budget: float, fmt: int, hn: int, layers=None, tokens: int = 8192,
                    outlier_mult: float = 50.0, threads: int = 1):
    """Time the oracle on a bounded sample of the same step: dual quantisation of a
    row slice of every operand and a sample of GEMM outputs of every pass, on
    `threads` host threads (1 = the serial build). Returns (extrapolated seconds per
    full step, description, threads used)."""
    import numpy as np
    import oracle
    from fp4_block_scaled_deterministic_b200 import synthetic
    oracle.build()
    threads = oracle.set_threads(threads)
    layers = layers or synthetic.LLAMA_LAYERS
    M = tokens
    rows = 64
    n_ent = 48
    q_time, q_elems, g_time, g_macs = 0.0, 0, 0.0, 0
    t_start = time.perf_counter()
    rounds = 0
    # repeat the per-projection sample until the time budget is used (at least once)
    while rounds == 0 or time.perf_counter() - t_start < seconds_budget:
        for i, (name, N, K) in enumerate(layers):
            X = synthetic.normal(rows * 2, K, 1.0, seed=i + 10 * rounds, outlier_frac=0.001,
                                 outlier_mult=outlier_mult)
            W = synthetic.normal(rows * 2, K, 0.02, seed=100 + i + 10 * rounds)
            t0 = time.perf_counter()
            xq = oracle.quantize(X, fmt, hn, oracle.ROW)
            oracle.quantize(X, fmt, hn, oracle.COL)
            wq = oracle.quantize(W, fmt, hn, oracle.ROW)
            oracle.quantize(W, fmt, hn, oracle.COL)
            q_time += time.perf_counter() - t0
            q_elems += 2 * X.numel() + 2 * W.numel()
            rng = np.random.default_rng(2 + rounds)
            ms, ns = rng.integers(0, rows * 2, n_ent), rng.integers(0, rows * 2, n_ent)
            t0 = time.perf_counter()
            oracle.gemm_entries(xq[:3], wq[:3], fmt, ms, ns)
            g_time += time.perf_counter() - t0
            g_macs += n_ent * K
        rounds += 1
    # full step: dual quantisation of X, W, dY of each projection, and 3 GEMMs
    step_elems, step_macs = 0, 0
    for name, N, K in layers:
        step_elems += 2 * (M * K + N * K + M * N)
        step_macs += 3 * M * N * K
    t_step = q_time / q_elems * step_elems + g_time / g_macs * step_macs
    oracle.set_threads(1)
    desc = (f"oracle (scalar C, {threads} thread{'s' if threads > 1 else ''}"
            f"{', OpenMP over rows and entries' if threads > 1 else ''}): {rounds} rounds of "
            f"dual quantisation of {rows * 2}-row "
            f"slices of X and W of each projection and {n_ent} GEMM outputs per projection "
            f"({q_elems} elements, {g_macs} MACs, {q_time + g_time:.1f} s of oracle time), "
            f"extrapolated linearly to the full step")
    return t_step, desc, threads


# ---------------------------------------------------------------- reference arm
def run_reference(a):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    fmt = FORMATS[a.format]
    layers, tokens, omult = layer_table(a)
    flops = sum(3 * 2.0 * tokens * N * K for _, N, K in layers)
    budget = min(20.0, max(2.0, 120.0 / (a.steps + a.warmup))) if a.cpu_budget is None \
        else a.cpu_budget
    threads = host_threads()
    for _ in range(a.warmup):
        cpu_oracle_rate(min(1.0, budget), fmt, a.hadamard, layers, tokens, omult, threads)
    ts = []
    desc = ""
    cores = threads
    t0 = time.perf_counter()
    for _ in range(a.steps):
        t_step, desc, cores = cpu_oracle_rate(budget, fmt, a.hadamard, layers, tokens, omult,
                                              threads)
        ts.append(t_step)
    wall = time.perf_counter() - t0
    t_med = statistics.median(ts)
    value = flops / t_med / 1e12
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": t_med * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": workload_name(a), "format": a.format, "hadamard_n": a.hadamard,
                       "l2": "n/a (CPU)"},
            "extrapolated": True,
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": desc, "wall_s": wall, "extrapolated": True,
                             "host": host_facts()},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- traffic record
def recorded_traffic(kernel_key: str):
    """dram bytes per launch of the dominant kernel from the committed ncu summary,
    valid only while the kernel sources hash to the value recorded with it."""
    path = os.path.join(ROOT, "profiles", "gemm_llama_traffic.json")
    if not os.path.exists(path):
        return None
    try:
        rec = json.load(open(path))
    except ValueError:
        return None
    if rec.get("source_sha1") != kernel_source_hash():
        return None
    return rec.get("per_launch_bytes", {}).get(kernel_key)


def kernel_source_hash():
    """Hash of the GEMM sources' code: // comments, trailing blanks and empty lines are
    left out, so that an edit of a comment does not void the recorded counters."""
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "fp4_block_scaled_deterministic_b200", "csrc")
    for f in ("common.cuh", "gemm.cuh"):
        for line in open(os.path.join(csrc, f), encoding="utf-8"):
            code = line.split("//", 1)[0].rstrip()
            if code:
                h.update(code.encode() + b"\n")
    return h.hexdigest()


# ---------------------------------------------------------------- quantise-only sweep
def run_sweep(a, dev):
    """Quantise-only bandwidth sweep: tensors of 2^p elements with rows of L elements,
    single (ROW, COL) and dual layouts; algorithmic GB/s per launch against measured HBM.
    One JSON line per case."""
    import fp4_block_scaled_deterministic_b200 as fp4
    from fp4_block_scaled_deterministic_b200 import synthetic
    fmt = FORMATS[a.format]
    pk, pk_kind = peaks()
    stream = torch.cuda.current_stream(dev)
    code_b = 1.0 if fmt == 2 else 0.5
    scale_b = 1 / 16 if fmt == 1 else 1 / 32
    for p in (24, 28, 30):
        for L in (4096, 14336, 49152):
            x = synthetic.sweep_tensor(p, L, seed=p, device=dev)
            rows, cols = x.shape
            ts = torch.zeros(4, dtype=torch.float32, device=dev) if fmt == 1 else None
            rq = fp4._alloc_q(rows, cols, fmt, dev)
            cq = fp4._alloc_q(cols, rows, fmt, dev)
            for mode in ("row", "col", "dual"):
                def launch():
                    if mode == "dual":
                        st = fp4.fp4_quantize_dual(x, rq[0], rq[1], cq[0], cq[1], ts, rows, cols,
                                                   fmt, a.hadamard, stream.cuda_stream)
                    else:
                        q = rq if mode == "row" else cq
                        st = fp4.fp4_quantize(x, q[0], q[1], ts, rows, cols, fmt, a.hadamard,
                                              fp4.ROW if mode == "row" else fp4.COL,
                                              stream.cuda_stream)
                    assert st == 0
                for _ in range(3):
                    launch()
                torch.cuda.synchronize(dev)
                n = 20 if p < 30 else 8
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(n):
                    launch()
                e1.record(stream)
                torch.cuda.synchronize(dev)
                ms = e0.elapsed_time(e1) / n
                outs = 2 if mode == "dual" else 1
                bpe = 2.0 + outs * (code_b + scale_b) + (2.0 if fmt == 1 else 0.0)
                gbs = rows * cols * bpe / (ms * 1e-3) / 1e9
                print(json.dumps({"sweep": "quantise", "elements": rows * cols, "p": p,
                                  "shape": [rows, cols], "format": a.format,
                                  "hadamard_n": a.hadamard, "mode": mode, "ms": ms,
                                  "gbs": gbs, "bytes_per_elem": bpe,
                                  "frac_hbm": gbs / pk["hbm_gbs"], "peak_source": pk_kind}),
                      flush=True)
            del x, rq, cq
            torch.cuda.empty_cache()
    assert fp4.fp4_check_status() == 0


def library_gemm(fmt, a, sa, ta, b, sb, tb):
    """torch's library block-scaled GEMM for `fmt` on this library's buffers, C = A B^T in
    bf16, as a callable; None where torch offers none. Codes [rows][K/2] (E2M1 pairs) or
    [rows][K] (E4M3); scales in the 32x4x4 swizzled atoms this library writes: E8M0 per 32
    (MX) or E4M3 per 16 under the fp32 tensor scales ta, tb (NVFP4)."""
    F = torch.nn.functional
    if not (hasattr(F, "scaled_mm") and hasattr(F, "ScalingType")
            and hasattr(torch, "float4_e2m1fn_x2")):
        return None
    ST, SW = F.ScalingType, F.SwizzleType
    if fmt == 1:
        a4, b4 = a.view(torch.float4_e2m1fn_x2), b.view(torch.float4_e2m1fn_x2).t()
        sa8, sb8 = sa.view(torch.float8_e4m3fn), sb.view(torch.float8_e4m3fn)
        for sw in ([SW.SWIZZLE_32_4_4, SW.NO_SWIZZLE], [SW.SWIZZLE_32_4_4]):
            def call(sw=sw):
                return F.scaled_mm(a4, b4, [sa8, ta], [ST.BlockWise1x16, ST.TensorWise],
                                   [sb8, tb], [ST.BlockWise1x16, ST.TensorWise],
                                   swizzle_a=sw, swizzle_b=sw, output_dtype=torch.bfloat16)
            try:
                call()
                return call
            except (RuntimeError, TypeError, ValueError):
                continue
        return None
    dt = torch.float8_e4m3fn if fmt == 2 else torch.float4_e2m1fn_x2
    a_, b_ = a.view(dt), b.view(dt).t()
    sa8, sb8 = sa.view(torch.float8_e8m0fnu), sb.view(torch.float8_e8m0fnu)

    def call():
        return F.scaled_mm(a_, b_, sa8, ST.BlockWise1x32, sb8, ST.BlockWise1x32,
                           swizzle_a=SW.SWIZZLE_32_4_4, swizzle_b=SW.SWIZZLE_32_4_4,
                           output_dtype=torch.bfloat16)
    try:
        call()
        return call
    except (RuntimeError, TypeError, ValueError):
        return None


def gemm_shapes(layers, tokens):
    """(label, M, N, K) of the layer's Fprop, Dgrad and Wgrad GEMMs, as the step runs them."""
    out = []
    for name, n, k in layers:
        out += [(f"{name}.fprop", tokens, n, k), (f"{name}.dgrad", tokens, k, n),
                (f"{name}.wgrad", n, k, tokens)]
    return out


def run_library_compare(a, dev):
    """This library's block-scaled GEMM against the kernel torch runs for the same format
    (torch.nn.functional.scaled_mm) on the layer's GEMM shapes. Both get the same random
    codes and scales (the scale layout is shared) and write bf16; each launch is timed
    alone after a 256 MB L2 flush, CUDA events on the launching stream. One JSON line per
    shape and one with the totals (flops over summed time) and whether every bf16 output
    was bit-identical."""
    import fp4_block_scaled_deterministic_b200 as fp4
    fmt = FORMATS[a.format]
    layers, tokens, _ = layer_table(a)
    wanted = [p.strip() for p in a.proj.split(",")]
    layers = [t for t in layers if t[0] in wanted] or layers
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(2)

    def timed(fn, n=10, warm=3):
        for _ in range(warm):
            fn()
        torch.cuda.synchronize(dev)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n)]
        for e0, e1 in ev:
            flush.fill_(1)
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        return sum(x.elapsed_time(y) for x, y in ev) / n

    def operand(rows, k):
        codes = torch.randint(0, 256, (rows, k if fmt == 2 else k // 2), dtype=torch.uint8,
                              device=dev, generator=gen)
        if fmt == 2:  # no E4M3 NaN codes
            codes[(codes & 0x7F) == 0x7F] -= 1
        lo, hi = (0x30, 0x50) if fmt == 1 else (122, 131)  # E4M3 / E8M0 scale bytes
        sc = torch.randint(lo, hi, (fp4.fp4_scales_bytes(rows, k, fmt),), dtype=torch.uint8,
                           device=dev, generator=gen)
        return codes, sc

    ta = torch.tensor([0.75], dtype=torch.float32, device=dev)
    tb = torch.tensor([1.3125], dtype=torch.float32, device=dev)
    tot = {"ours": [0.0, 0.0], "library": [0.0, 0.0]}
    all_equal, available = True, True
    for label, m, n, k in gemm_shapes(layers, tokens):
        A, As = operand(m, k)
        B, Bs = operand(n, k)
        C = torch.empty(m, n, dtype=torch.bfloat16, device=dev)
        nv = fmt == 1

        def ours():
            st = fp4.fp4_gemm(A, As, ta if nv else None, B, Bs, tb if nv else None, C, m, n, k,
                              fmt, fp4.OUT_BF16, stream.cuda_stream)
            assert st == 0, fp4.status_string(st)
        flops = 2.0 * m * n * k
        ms = timed(ours)
        rec = {"library_compare": a.format, "gemm": label, "mnk": [m, n, k],
               "ours_tflops": flops / ms / 1e9}
        tot["ours"][0] += flops
        tot["ours"][1] += ms
        lib = library_gemm(fmt, A, As, ta, B, Bs, tb)
        if lib is None:
            available = False
        else:
            ms2 = timed(lib)
            rec["library_tflops"] = flops / ms2 / 1e9
            tot["library"][0] += flops
            tot["library"][1] += ms2
            ours()
            ref = lib()
            torch.cuda.synchronize(dev)
            rec["bf16_bit_identical"] = bool(torch.equal(C.view(torch.int16),
                                                         ref.contiguous().view(torch.int16)))
            all_equal = all_equal and rec["bf16_bit_identical"]
            del ref
        print(json.dumps(rec), flush=True)
        del A, As, B, Bs, C
        torch.cuda.empty_cache()
    out = {"library_compare": a.format, "total": True, "gemms": len(gemm_shapes(layers, tokens)),
           "ours_tflops": tot["ours"][0] / tot["ours"][1] / 1e9,
           "library": "torch.nn.functional.scaled_mm" if available else None}
    if available:
        out["library_tflops"] = tot["library"][0] / tot["library"][1] / 1e9
        out["ratio"] = out["ours_tflops"] / out["library_tflops"]
        out["bf16_bit_identical_all"] = all_equal
    print(json.dumps(out), flush=True)
    assert fp4.fp4_check_status() == 0


# ---------------------------------------------------------------- main
def spawn_ranks(a) -> int:
    """`--gpus N` (N > 1) started as a plain process: re-launch this command as N ranks
    of one node through torch.distributed.run (one process per GPU, rendezvous on
    127.0.0.1), and return its exit status. Fails loudly when fewer than N GPUs are
    visible."""
    import socket
    have = torch.cuda.device_count()
    if have < a.gpus:
        print(f"bench.py: --gpus {a.gpus} needs {a.gpus} visible CUDA devices, found {have}",
              file=sys.stderr, flush=True)
        return 2
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={a.gpus}", "--master-addr=127.0.0.1", f"--master-port={port}",
           os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    a = parse()
    if a.impl == "reference":
        return run_reference(a)
    if a.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(spawn_ranks(a))
    if a.gpus != int(os.environ.get("WORLD_SIZE", "1")):
        print(f"bench.py: --gpus {a.gpus} but WORLD_SIZE={os.environ.get('WORLD_SIZE', '1')}",
              file=sys.stderr, flush=True)
        sys.exit(2)
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    import fp4_block_scaled_deterministic_b200 as fp4
    fp4.lib()  # fails loudly if the library is missing
    fmt = FORMATS[a.format]
    if a.sweep:
        return run_sweep(a, dev)
    if a.library_compare:
        return run_library_compare(a, dev)
    layers, tokens, omult = layer_table(a)
    all_names = [n for n, _, _ in layers]
    names = [n.strip() for n in a.proj.split(",") if n.strip() in all_names] or all_names
    # data parallel: every rank holds the same W (replicated weights) and its own tokens
    layer = LlamaLayer(dev, fmt, a.hadamard, tokens=tokens, seed=1000 * rank, names=names,
                       variant=a.variant, side_stream=bool(a.side_stream), layers=layers,
                       outlier_mult=omult, w_seed=0, next_quant=a.next_layer_quant,
                       quant_batch=bool(a.quant_batch), gemm_group=bool(a.gemm_group))
    stream = torch.cuda.current_stream(dev)
    from fp4_block_scaled_deterministic_b200 import dp
    allreduce = (lambda t: dp.allreduce_wgrad(t, async_op=True)) if world > 1 else None

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])
        torch.cuda.synchronize(dev)

    for _ in range(a.warmup):
        layer.step(stream, None, allreduce)
    barrier()
    assert fp4.fp4_check_status() == 0

    timers = {"quant": [], "gemm": [], "quant_y": []}
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    nvml = NvmlClocks(local)
    nvml.start()
    win_pass = None
    if a.side_stream:
        # Per-kernel durations for the rooflines come from the same steps run on one
        # stream, where no kernel shares the SMs; the step time below overlaps them.
        for _ in range(a.warmup):
            layer.step(stream, None, allreduce, overlap=False)
        barrier()
        tp0 = time.perf_counter()
        for _ in range(a.steps):
            layer.step(stream, timers, allreduce, overlap=False)
        barrier()
        win_pass = (tp0, time.perf_counter())
        for _ in range(a.warmup):
            layer.step(stream, None, allreduce)
        barrier()
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    barrier()
    tt0 = time.perf_counter()
    e0.record(stream)
    for _ in range(a.steps):
        layer.step(stream, None if a.side_stream else timers, allreduce)
    e1.record(stream)
    barrier()
    tt1 = time.perf_counter()
    clk = clocks.stop()
    nvml.stop()
    if win_pass is None:
        win_pass = (tt0, tt1)
    clk_fine = {"timed_region": nvml.window(tt0, tt1),
                "kernel_timing_pass": nvml.window(*win_pass),
                "source": "NVML every 5 ms (reads only)"} if nvml.ok else None
    ms = dp.max_over_ranks(e0.elapsed_time(e1), dev)
    status = fp4.fp4_check_status()
    if status != 0:
        raise RuntimeError(f"device status {fp4.status_string(status)}")

    flops_step = layer.flops()
    value = flops_step * world / (ms / a.steps * 1e-3) / 1e12
    gemm_ms = [x.elapsed_time(y) for x, y in timers["gemm"]]
    quant_ms = [x.elapsed_time(y) for x, y in timers["quant"]]
    per_launch_flops = gemm_flops_of(layer) * a.steps
    gemm_tflops = sum(per_launch_flops) / (sum(gemm_ms) * 1e-3) / 1e12
    amax_pass = fmt == 1 and a.variant != "amax"
    code_b = 1.0 if fmt == 2 else 0.5                   # bytes per code
    scale_b = 1 / 16 if fmt == 1 else 1 / 32            # scale bytes per element
    bpe = 2.0 + 2 * (code_b + scale_b) + (2.0 if amax_pass else 0.0)
    q_bytes = layer.quant_elems() * bpe * a.steps
    quant_gbs = q_bytes / (sum(quant_ms) * 1e-3) / 1e9

    pk, pk_kind = peaks()
    ratio = FP8_OVER_BF16 if fmt == 2 else FP4_OVER_BF16
    # the GEMM is timed launch by launch in a sub-second loop: the burst bf16 figure x the
    # nominal FP4 (FP8) : BF16 ratio; the datasheet dense peak and the sustained figure
    # are reported beside it
    peak_fp4 = pk["bf16_tflops"] * ratio
    sheet = DATASHEET_TFLOPS["fp8" if fmt == 2 else "fp4"]
    avg_launch_ms = sum(gemm_ms) / len(gemm_ms)
    avg_flops = sum(per_launch_flops) / len(per_launch_flops)
    traffic = (recorded_traffic(("mxfp4" if fmt == 0 else "nvfp4")
                                + ("_group" if layer.gemm_launches() == 1 else ""))
               if a.workload == "llama" and a.hadamard == 16 and len(names) == len(all_names)
               else None)
    # the GEMM rate referred to the maximum SM clock, from the clocks sampled while the
    # per-launch times were taken (time x median MHz / max MHz)
    at_max_clock = None
    if clk_fine and clk_fine["kernel_timing_pass"] and clk.get("sm_max_mhz"):
        at_max_clock = (gemm_tflops * clk["sm_max_mhz"]
                        / clk_fine["kernel_timing_pass"]["sm_mhz_median"])
    roof = {"bound": "tensor", "achieved": gemm_tflops, "peak": peak_fp4, "unit": "TFLOP/s",
            "achieved_at_max_sm_clock": at_max_clock,
            "frac": gemm_tflops / peak_fp4, "traffic": traffic,
            "frac_datasheet": gemm_tflops / sheet, "peak_datasheet": sheet,
            "frac_sustained": gemm_tflops / (pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
                                             * ratio),
            "kernel": "gemm_fp4_pair_kernel (tcgen05 block-scaled "
                      f"{'MXFP8, kind::mxf8f6f4' if fmt == 2 else 'FP4'}, CTA pairs"
                      + ("; a projection's Fprop, Dgrad and Wgrad per launch)"
                         if layer.gemm_launches() == 1 else ")"),
            "per_launch": {"avg_flops": avg_flops, "avg_ms": avg_launch_ms,
                           "median_ms": statistics.median(gemm_ms),
                           "launches": len(gemm_ms)},
            "achieved_at_median_launch": (
                statistics.median([f / (t * 1e-3) / 1e12 for f, t in zip(per_launch_flops, gemm_ms)])),
            "timing": ("CUDA events around each launch over the timed steps" if not a.side_stream
                       else "CUDA events around each launch over the same number of steps run "
                            "on one stream just before the overlapped timed region"),
            "peak_source": f"{pk_kind}: bf16_tflops (burst) x {ratio} (nominal "
                           f"{'FP8' if fmt == 2 else 'FP4'}:BF16); frac_datasheet against the "
                           f"B200 dense {'FP8' if fmt == 2 else 'FP4'} datasheet peak"}
    qroof = {"bound": "hbm", "achieved": quant_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
             "frac": quant_gbs / pk["hbm_gbs"], "bytes_per_elem": bpe,
             "kernel": ("quantize_kernel dual layout, "
                        + ("X, W, dY of a projection per launch" if layer.quant_batch
                           else "one tensor per launch")), "launches": len(quant_ms),
             "avg_ms": sum(quant_ms) / len(quant_ms), "median_ms": statistics.median(quant_ms),
             "peak_source": f"{pk_kind}: hbm_gbs"}

    out = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
           "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms / a.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp8_e4m3" if fmt == 2 else "fp4_e2m1",
           "data": "synthetic",
           "dw_reduction": (dp.REDUCTION if world > 1 else None),
           "config": {"workload": workload_name(a) if len(names) == len(all_names) else
                      f"subset {','.join(names)} of: {workload_name(a)}",
                      "format": a.format, "hadamard_n": a.hadamard, "variant": a.variant,
                      "next_layer_quant": a.next_layer_quant,
                      "quant_launch": ("one batched launch per projection (X, W, dY)"
                                       if layer.quant_batch else "one launch per tensor"),
                      "gemm_launch": (("one fp4_gemm_group_quant launch per projection (Fprop "
                                       "with Y quantised in its epilogue, Dgrad, Wgrad)"
                                       if layer.next_quant == "fused" else
                                       "one fp4_gemm_group launch per projection (Fprop, "
                                       "Dgrad, Wgrad)")
                                      if layer.gemm_group else "one launch per GEMM"),
                      "streams": 2 if a.side_stream else 1,
                      "tokens_per_rank": layer.M,
                      "l2": f"inputs larger than L2 ({(layer.bytes_in() + layer.bytes_out()) / 1e9:.1f} GB per step)",
                      "parallelism": f"dp{world}"},
           "gemm_tflops": gemm_tflops, "quantize_gbs": quant_gbs,
           "roofline": roof, "roofline_quantize": qroof, "clocks": clk, "clocks_nvml": clk_fine,
           "gpu_launches": layer.launches_per_step() * a.steps}
    if a.next_layer_quant != "none":
        qy = [x.elapsed_time(y) for x, y in timers["quant_y"]]
        out["next_layer_quant"] = {
            "mode": a.next_layer_quant,
            "what": "each Fprop output Y quantised row-wise (MXFP4, same rotation) for the next "
                    "layer, by a separate launch (standalone) or in the GEMM epilogue (fused)",
            "standalone_launch_avg_ms": (sum(qy) / len(qy)) if qy else None}

    # end to end through the C ABI from pinned host buffers (inputs H2D, outputs D2H)
    if not a.no_e2e:
        host_in = [[t.cpu().pin_memory() for t in (p["X"], p["W"], p["dY"])] for p in layer.projs]
        host_out = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                     for t in (p["Y"], p["dX"], p["dW"])] for p in layer.projs]
        barrier()

        # Copies run on their own streams, per projection: the inputs of projection i
        # arrive while earlier projections compute, and its outputs leave while later
        # ones compute (PCIe carries both directions at once). Events keep every copy
        # ordered with the kernels that read or overwrite the same buffers.
        h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        n = len(layer.projs)
        in_ready = [torch.cuda.Event() for _ in range(n)]
        out_free = [torch.cuda.Event() for _ in range(n)]
        for ev in out_free:
            ev.record(stream)

        def e2e_step():
            for i, (p, hin) in enumerate(zip(layer.projs, host_in)):
                h2d.wait_event(layer.quant_done[i])  # last step's readers of these inputs
                with torch.cuda.stream(h2d):
                    p["X"].copy_(hin[0], non_blocking=True)
                    p["W"].copy_(hin[1], non_blocking=True)
                    p["dY"].copy_(hin[2], non_blocking=True)
                in_ready[i].record(h2d)
            layer.step(stream, None, allreduce, inputs_ready=in_ready, outputs_free=out_free)
            if allreduce is not None:
                d2h.wait_stream(stream)  # dW is final only after its all-reduce
            for i, (p, hout) in enumerate(zip(layer.projs, host_out)):
                d2h.wait_event(layer.gemms_done[i])
                with torch.cuda.stream(d2h):
                    hout[0].copy_(p["Y"], non_blocking=True)
                    hout[1].copy_(p["dX"], non_blocking=True)
                    hout[2].copy_(p["dW"], non_blocking=True)
                out_free[i].record(d2h)
            stream.wait_event(out_free[n - 1])  # the step ends when its last output is home
            stream.wait_stream(d2h)

        e2e_step()
        barrier()
        e0.record(stream)
        for _ in range(a.steps):
            e2e_step()
        e1.record(stream)
        barrier()
        ems = dp.max_over_ranks(e0.elapsed_time(e1), dev)
        out["e2e"] = {"value": flops_step * world / (ems / a.steps * 1e-3) / 1e12,
                      "unit": "TFLOP/s", "h2d_bytes_per_step": layer.bytes_in(),
                      "d2h_bytes_per_step": layer.bytes_out(), "ms_per_step": ems / a.steps}
    else:
        out["e2e"] = None

    if (rank == 0 and world == 1 and not a.no_cpu_baseline and a.workload == "llama"
            and len(names) == len(all_names)):
        t1, desc1, _ = cpu_oracle_rate(a.cpu_seconds / 2, fmt, a.hadamard, threads=1)
        tn, descn, cores = cpu_oracle_rate(a.cpu_seconds / 2, fmt, a.hadamard,
                                           threads=host_threads())
        out["cpu_baseline"] = {"value": flops_step / tn / 1e12, "unit": "TFLOP/s",
                               "cores": cores, "kind": "oracle", "sample": descn,
                               "extrapolated": True, "host": host_facts(),
                               "single_thread": {"value": flops_step / t1 / 1e12,
                                                 "cores": 1, "sample": desc1}}
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
