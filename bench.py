"""Benchmark of the quantized DiT linear layer on B200.

One step = one pass of the whole path over one batch of synthetic FLUX-shaped
input: dynamic activation quantization, block-scaled tcgen05 GEMM and fused
epilogue, for every layer of the workload.  The default (headline) workload
is the largest FLUX shape, the CFG-batched parallel-block linear1
(M = 2 x 16896 tokens, K = 3072, N = 21504, split bias / GELU epilogue) in its
FP8 and its NVFP4 variant, one layer each on their own inputs; the line also
carries a shorter measurement of every other FLUX configuration ("sweep").

Metric: TFLOP/s of the quantized linear layers (2*M*N*K per GEMM / step
time).  Timing: W warm-up steps, then exactly K steps between CUDA events on
the launching stream, bracketed by barrier + synchronize; max over ranks.
Input sets rotate and every set is larger than the 126 MB L2, so no step
reads operands that an earlier step left in L2.

Per kernel, after the timed steps (same inputs, CUDA events on the launching
stream):
  * roofline: each GEMM alone in a loop of at least 50 launches over the
    rotating sets -> algorithmic 2*M*N*K / mean launch time, against the
    measured bf16 peak times the nominal FP8 (x2) / FP4 (x4) ratio;
  * quant_roofline: each activation quantization alone in a loop over enough
    copies of its input that one pass reads more than twice the L2 -> the
    algorithmic bytes / mean call time, against the measured copy bandwidth.

Multi-GPU (torchrun): every rank runs the same per-GPU workload on its own
tokens (weak scaling, no data-path collective); value = all ranks' FLOPs /
max-over-ranks time.

--impl reference times the CPU oracle (the reference arm of this method) on
the host cores, on a bounded row sample of every layer per step.
"""
import argparse
import dataclasses
import hashlib
import json
import os
import re
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import WORKLOADS, make_inputs  # noqa: E402

DEFAULT_WORKLOAD = "cfg_linear1"
# the other FLUX configurations, measured after the headline in the default run
SWEEP = ("flux_qkv_fp8", "flux_mlp_fp8", "flux2k_swiglu_nvfp4", "tiny_fp8", "flux_qkv_w8a16")
L2_BYTES = 126 * 2 ** 20
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# nominal dense tensor-core ratios to bf16 (FP8 4.5 / 2.25 PF, FP4 9 / 2.25 PF)
NOMINAL_RATIO = {"fp8": 2.0, "nvfp4": 4.0, "w8a16": 1.0}  # w8a16 runs bf16 MMAs
GEMM_SOURCES = ["precision_gemm_qlinear_b200/csrc/gemm.cu", "precision_gemm_qlinear_b200/csrc/codec.cuh",
                "precision_gemm_qlinear_b200/csrc/ptx.cuh",
                "precision_gemm_qlinear_b200/csrc/internal.h"]
MIN_GEMM_LAUNCHES = 50


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--no-sweep", action="store_true",
                    help="measure only --workload (no other configurations)")
    ap.add_argument("--sweep-steps", type=int, default=100)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--sets", type=int, default=0, help="input rotation sets (0 = auto)")
    ap.add_argument("--fuse-quant", action="store_true",
                    help="NVFP4 -> NVFP4 layer boundaries: the producing GEMM writes the next "
                         "layer's quantized input (previous step's observed amax)")
    ap.add_argument("--gemm-ms", type=float, default=300.0,
                    help="target duration of each GEMM-only timing loop")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override M of every layer (smaller captures for profiling only)")
    return ap.parse_args(argv)


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def strip_comments(src):
    """C/C++ source without comments, trailing blanks or blank lines, so that
    the fingerprint below changes with the code only (the kernel sources hold
    no comment markers inside string literals)."""
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(ln.rstrip() for ln in src.splitlines() if ln.strip())


def gemm_source_sha(root=None):
    """Fingerprint of the GEMM kernel's code (comments excluded)."""
    h = hashlib.sha256()
    for p in GEMM_SOURCES:
        with open(os.path.join(root or ROOT, p)) as f:
            h.update(strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload, layer_index, M):
    """DRAM bytes (read + write) per launch of a GEMM from the committed ncu
    summaries (profiles/traffic.json), if the kernel's code has not changed
    since the capture.  A capture of a smaller M is scaled to this M by the
    ratio of the launch's algorithmic bytes (recorded with the capture)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None, None
    with open(path) as f:
        d = json.load(f)
    e = d.get(f"{workload}:{layer_index}")
    if not e or e.get("source_sha") != gemm_source_sha():
        return None, None
    b = float(e["dram_bytes_per_launch"])
    if e.get("M") and e["M"] != M:
        b *= float(e["algorithmic_bytes_full"]) / float(e["algorithmic_bytes_captured"])
    return int(b), e.get("capture")


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, index, period=0.02):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self.ok = False
        self.period = period
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        reasons = [k for k, v in self.REASONS.items() if self.reasons & v and k != "gpu_idle"]
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples)}


def with_tokens(wl, tokens):
    """The workload with every layer's M replaced (0 = unchanged)."""
    if not tokens:
        return wl
    layers = tuple(dataclasses.replace(l, M=int(tokens)) for l in wl.layers)
    return dataclasses.replace(wl, name=f"{wl.name}@M={tokens}", layers=layers)


def base_name(wl):
    return wl.name.split("@", 1)[0]


# ------------------------------------------------------- multi-rank helpers

def rank_seed(rank: int) -> int:
    """Weak scaling over tokens: every rank quantizes and multiplies its own
    tokens (seed = rank), against the same weights (seed 0)."""
    return int(rank)


def max_over_ranks(ms: float, world: int, device=None) -> float:
    """Max of a per-rank device time over all ranks (the job's time)."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_tflops(flops_per_step: float, world: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: the FLOPs of every rank over the slowest rank's time."""
    return flops_per_step * world * steps / (max_ms / 1e3) / 1e12


# --------------------------------------------------------------------- ours

def to_dev(a, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)


class Model:
    """The workload's layers with NSETS rotated copies of inputs and weights.

    Set 0 holds the seeded inputs of the workload (seed `seed` for the
    tokens, 0 for the weights).  With distinct=False the other sets are
    device copies of set 0 (separate memory, same values: what matters for
    the rotation is that no set is in L2 when it is reused); with
    distinct=True each set draws its own inputs and weights.

    fuse=True: at every NVFP4 -> NVFP4 layer boundary (Nout % 256 == 0) the
    producing GEMM writes the next layer's quantized input itself
    (qlinear_forward_nvfp4_out), against the tensor amax the same boundary
    observed on the previous step (another input set); a calibration pass of
    the unfused path provides the first values."""

    def __init__(self, wl, dev, seed, nsets, fuse=False, distinct=False):
        import torch
        import precision_gemm_qlinear_b200 as ql
        self.wl, self.dev = wl, dev
        self.sets = []
        base = {}  # set 0's device inputs, copied for the other sets
        for s in range(nsets):
            layers = []
            for li, layer in enumerate(wl.layers):
                if s == 0 or distinct:
                    inp = make_inputs(layer, seed=seed * 1000 + s if distinct else seed,
                                      layer_index=li, w_seed=s if distinct else 0)
                    dev_in = {}
                    for k, v in inp.items():
                        if v is None:
                            dev_in[k] = None
                        elif k in ("rope_cos", "rope_sin"):
                            dev_in[k] = torch.from_numpy(v).to(dev)
                        else:
                            dev_in[k] = to_dev(v, dev)
                    if s == 0:
                        base[li] = dev_in
                else:
                    dev_in = {k: (None if v is None else v.clone()) for k, v in base[li].items()}
                lay = ql.QLinear(layer.fmt, layer.epi, dev_in["w"], dev_in["bias"],
                                 split_col=layer.split_col)
                codes, scales = lay.act_buffers(layer.M, dev)
                d = dict(lay=lay, codes=codes, scales=scales,
                         out=torch.empty((layer.M, lay.Nout), dtype=torch.bfloat16, device=dev))
                for k in ("x", "gate", "residual", "rope_cos", "rope_sin"):
                    if k in dev_in:
                        d[k] = dev_in[k]
                if layer.epi == "qkv_norm_rope":
                    lay.set_qk_norm(dev_in["q_norm"], dev_in["k_norm"])
                layers.append(d)
            self.sets.append(layers)
        base.clear()  # the bf16 master weights: quantized into each layer's workspace
        L = wl.layers
        self.fused = [False] + [
            fuse and L[j].chained and L[j - 1].fmt == "nvfp4" and L[j].fmt == "nvfp4" and
            L[j - 1].Nout % 256 == 0 for j in range(1, len(L))]
        if fuse and not any(self.fused):
            raise ValueError(f"{wl.name}: no NVFP4 -> NVFP4 boundary to fuse")
        torch.cuda.synchronize()
        if any(self.fused):
            for s in range(nsets):   # calibration: the unfused path fills every observed amax
                self.run_layers(self.sets[s], None, unfused=True)
            torch.cuda.synchronize()

    def amax_of(self, layers, j):
        """Device fp32 view of the observed tensor amax stored in the tail of
        layer j's activation scales of one input set."""
        import torch
        layer = self.wl.layers[j]
        nsf = ((layer.M + 127) // 128) * ((layer.K + 255) // 256) * 4 * 512
        return layers[j]["scales"][nsf + 4:nsf + 8].view(torch.float32)

    def inputs_of(self, layers, i):
        """bf16 input of layer i: its own x, or the previous layer's output."""
        return layers[i - 1]["out"] if self.wl.layers[i].chained else layers[i]["x"]

    def run_layers(self, layers, stream, gemm_events=None, amax_from=None, unfused=False,
                   x_override=None):
        """quantize + GEMM + epilogue of every layer over one input set.
        x_override: {layer index: bf16 input} replacing a layer's own x."""
        for i, d in enumerate(layers):
            lay = d["lay"]
            x = (x_override or {}).get(i)
            if x is None:
                x = self.inputs_of(layers, i)
            fused_in = self.fused[i] and not unfused
            fused_out = i + 1 < len(layers) and self.fused[i + 1] and not unfused
            w16 = self.wl.layers[i].fmt == "w8a16"  # activations stay bf16: x is the operand
            if not fused_in and not w16:
                lay.quantize(x, d["codes"], d["scales"], stream)
            codes = x if w16 else d["codes"]
            if gemm_events is not None:
                gemm_events[i][0].record(stream)
            self.gemm(i, layers, codes, stream, amax_from, fused_out)
            if gemm_events is not None:
                gemm_events[i][1].record(stream)

    def gemm(self, i, layers, codes, stream, amax_from=None, fused_out=False):
        """The GEMM + epilogue of layer i on one input set."""
        d, M = layers[i], self.wl.layers[i].M
        lay = d["lay"]
        if fused_out:
            nd = layers[i + 1]
            lay.forward_nvfp4_out(codes, d["scales"], M, self.amax_of(amax_from, i + 1),
                                  nd["codes"], nd["scales"], d.get("residual"), d.get("gate"),
                                  stream)
        elif "rope_cos" in d:
            lay.forward_rope(codes, d["scales"], M, d["rope_cos"], d["rope_sin"], d["out"], stream)
        else:
            lay.forward_codes(codes, d["scales"], M, d["out"], d.get("residual"), d.get("gate"),
                              stream)

    def step(self, s, stream, gemm_events=None):
        """Enqueue one pass of the path over input set s."""
        n = len(self.sets)
        self.run_layers(self.sets[s % n], stream, gemm_events, amax_from=self.sets[(s - 1) % n])

    def launches_per_step(self):
        n = 0
        for j, layer in enumerate(self.wl.layers):
            if not self.fused[j] and layer.fmt != "w8a16":
                n += 1 if layer.fmt == "fp8" else 2   # the quantize kernels
            n += 1                                     # the GEMM
        return n

    def close(self):
        for s in self.sets:
            for d in s:
                d["lay"].close()
        self.sets = []


def quant_bytes(layer) -> int:
    """Algorithmic HBM bytes of one activation quantization of `layer`'s input."""
    mk = layer.M * layer.K
    if layer.fmt == "fp8":
        return mk * 2 + mk + layer.M * 4                # read x, write codes, row scales
    return mk * 2 + mk * 2 + mk // 2 + mk // 16 + 16    # amax pass, read x, codes, block scales


def gemm_bytes(layer) -> int:
    """Algorithmic HBM bytes of one GEMM launch: both operands with their
    scales read once, the output written once (plus the residual read)."""
    M, N, K, Nout = layer.M, layer.N, layer.K, layer.Nout
    if layer.fmt == "nvfp4":
        b = M * K // 2 + N * K // 2 + (M + N) * K // 16
    elif layer.fmt == "w8a16":
        b = M * K * 2 + N * K + N * 4
    else:
        b = M * K + N * K + (M + N) * 4
    b += M * Nout * 2
    if layer.epi == "bias_gated_residual":
        b += M * Nout * 2
    return b


def _timed_loop(stream, fn, target_ms, min_calls, max_calls=5000):
    """Mean duration (ms) of fn(i) over a loop sized to about target_ms,
    CUDA events on `stream` around the whole loop (after 3 untimed calls)."""
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for i in range(3):
            fn(i)
        e0.record(stream)
        fn(3)
        e1.record(stream)
    stream.synchronize()
    one = max(e0.elapsed_time(e1), 1e-3)
    n = int(min(max_calls, max(min_calls, target_ms / one)))
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(n):
            fn(4 + i)
        e1.record(stream)
    stream.synchronize()
    return e0.elapsed_time(e1) / n, n


def gemm_roofline(model, stream, peaks, peak_src, target_ms):
    """Each layer's GEMM (+ fused epilogue) timed alone over the rotating
    sets (their activation codes were written by the timed steps)."""
    import torch
    out = []
    nsets = len(model.sets)
    dev = torch.device(model.dev)
    dev_index = dev.index if dev.index is not None else 0
    for j, layer in enumerate(model.wl.layers):
        w16 = layer.fmt == "w8a16"
        fused_out = j + 1 < len(model.wl.layers) and model.fused[j + 1]

        def run(i, j=j, w16=w16, fused_out=fused_out):
            layers = model.sets[i % nsets]
            codes = model.inputs_of(layers, j) if w16 else layers[j]["codes"]
            model.gemm(j, layers, codes, stream, amax_from=model.sets[(i - 1) % nsets],
                       fused_out=fused_out)
        with ClockSampler(dev_index, period=0.01) as cs:
            ms, n = _timed_loop(stream, run, target_ms, MIN_GEMM_LAUNCHES)
        achieved = layer.flops / (ms / 1e3) / 1e12
        sustained = ms * n > 1000.0
        bf16 = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
        peak = bf16 * NOMINAL_RATIO[layer.fmt]
        peak_sus = peaks["bf16_tflops_sustained"] * NOMINAL_RATIO[layer.fmt]
        traffic, capture = profiled_traffic(base_name(model.wl), j, layer.M)
        out.append({
            "layer": j, "kernel": f"qgemm_kernel<{layer.fmt},{layer.epi}>", "bound": "tensor",
            "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "frac_vs_sustained": round(achieved / peak_sus, 4),
            "traffic": traffic, "traffic_capture": capture,
            "algorithmic_bytes": gemm_bytes(layer), "gemm_ms": round(ms, 5), "launches": n,
            "clocks": cs.summary(),
            "fused_nvfp4_out": bool(fused_out),
            "peak_source": f"{peak_src} bf16 {'sustained' if sustained else 'burst'} x "
                           f"{NOMINAL_RATIO[layer.fmt]:g} (nominal {layer.fmt}/bf16 ratio)"})
    return out


def quant_roofline(model, stream, peaks, peak_src, target_ms=100.0):
    """The quantize kernel(s) of every layer timed alone, rotating over
    enough copies of the layer's input (and output buffers) that one pass
    moves more than twice the L2: every call reads x from HBM."""
    import torch
    out = []
    for j, layer in enumerate(model.wl.layers):
        if model.fused[j] or layer.fmt == "w8a16":
            continue  # quantized by the previous layer's epilogue / not quantized at all
        d0 = model.sets[0][j]
        x0 = model.inputs_of(model.sets[0], j)
        ncopies = min(1024, max(2, int(np.ceil(2 * L2_BYTES / quant_bytes(layer))) + 1))
        bufs = [(x0, d0["codes"], d0["scales"])]
        for _ in range(ncopies - 1):
            c, s = d0["lay"].act_buffers(layer.M, x0.device)
            bufs.append((x0.clone(), c, s))

        def run(i, bufs=bufs, lay=d0["lay"]):
            x, c, s = bufs[i % len(bufs)]
            lay.quantize(x, c, s, stream)
        us = _timed_loop(stream, run, target_ms, 20, 4000)[0] * 1e3
        gbs = quant_bytes(layer) / (us * 1e-6) / 1e9
        out.append({"layer": j, "kernel": "quant_fp8_rows" if layer.fmt == "fp8"
                    else "tensor_amax+quant_nvfp4", "bound": "hbm", "us": round(us, 2),
                    "bytes": quant_bytes(layer), "achieved": round(gbs, 1),
                    "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(gbs / peaks["hbm_gbs"], 4), "input_copies": len(bufs),
                    "peak_source": f"{peak_src} copy bandwidth"})
        del bufs
        torch.cuda.empty_cache()
    return out


class OracleLayer:
    """The oracle's path for one layer: weights quantized once (untimed), then
    quantize + GEMM + epilogue over a slice of activation rows."""

    def __init__(self, layer, inp, x):
        import oracle
        self.o, self.layer, self.inp, self.x = oracle, layer, inp, x
        if layer.fmt in ("fp8", "w8a16"):
            self.qw, self.sw = oracle.quant_fp8_rows(inp["w"])
        else:
            self.qw, self.sfw, self.gw = oracle.quant_nvfp4(inp["w"])
            self.amax = oracle.tensor_amax(x)  # the tensor amax is over the whole input

    def gemm(self, r0, rows):
        o, L, xs = self.o, self.layer, self.x[r0:r0 + rows]
        if L.fmt == "fp8":
            qa, sa = o.quant_fp8_rows(xs)
            return o.gemm_fp8(qa, sa, self.qw, self.sw)
        if L.fmt == "w8a16":
            return o.gemm_w8a16(xs, self.qw, self.sw)
        qa, sfa, ga = o.quant_nvfp4(xs, amax=self.amax)
        return o.gemm_nvfp4(qa, sfa, ga, self.qw, self.sfw, self.gw)

    def run(self, r0, rows):
        o, L, inp = self.o, self.layer, self.inp
        y = self.gemm(r0, rows)
        if L.epi == "qkv_norm_rope":
            return o.qkv_norm_rope(y, inp["bias"], inp["q_norm"], inp["k_norm"],
                                   inp["rope_cos"][r0:r0 + rows], inp["rope_sin"][r0:r0 + rows])
        res = inp.get("residual")
        return o.epilogue(L.epi, y, bias=inp["bias"], split_col=L.split_col,
                          residual=None if res is None else res[r0:r0 + rows],
                          gate=inp.get("gate"))


def oracle_layers(wl):
    """One OracleLayer per layer of the workload (a chained layer's input is a
    bf16 stand-in of the same shape: the oracle's time does not depend on
    the values)."""
    out = []
    for li, layer in enumerate(wl.layers):
        inp = make_inputs(layer, seed=0, layer_index=li)
        x = inp.get("x")
        if x is None:
            x = make_inputs(dataclasses.replace(layer, chained=False), seed=0, layer_index=li)["x"]
        out.append(OracleLayer(layer, inp, x))
    return out


def cpu_baseline(wl, seconds):
    """Time the oracle (as it stands) on a bounded row sample of every layer
    of the workload; returns TFLOP/s-equivalent and a description."""
    ols = oracle_layers(wl)  # weights quantized once, untimed

    def run(rows):
        t0 = time.perf_counter()
        for ol in ols:
            ol.run(0, rows)
        return time.perf_counter() - t0

    Mmin = min(l.M for l in wl.layers)
    probe = 4
    t = run(probe)
    while t < 0.5 and probe < Mmin:
        probe = min(Mmin, probe * 4)
        t = run(probe)
    rows = int(max(1, min(Mmin, probe * seconds / max(t, 1e-6))))
    dt = run(rows) if rows != probe else t
    flops = sum(2.0 * rows * l.N * l.K for l in wl.layers)
    return flops / dt / 1e12, rows, dt, ols[0].o.num_threads()


def measure(wl, args, dev, rank, world, steps, warmup, peaks, peak_src, e2e=False):
    """Time one workload: K steps of the whole path, then the per-kernel
    loops.  Returns the workload's result dict (rank 0 fields)."""
    import torch
    import torch.distributed as dist

    per_set = 0
    for layer in wl.layers:
        kb = layer.K // 2 if layer.fmt == "nvfp4" else layer.K
        per_set += layer.M * layer.K * 2 + layer.N * kb + layer.M * layer.Nout * 2
    nsets = args.sets or max(2, int(np.ceil(2 * L2_BYTES / per_set)) + 1)
    model = Model(wl, dev, seed=rank_seed(rank), nsets=nsets, fuse=args.fuse_quant)
    stream = torch.cuda.Stream(device=dev)
    flops_step = float(wl.flops)

    with torch.cuda.stream(stream):
        for i in range(warmup):
            model.step(i, stream)
    stream.synchronize()
    for s in model.sets:
        for d in s:
            st = d["lay"].check(stream)
            if st != 0:
                raise RuntimeError(f"{wl.name}: device error during warm-up: status {st}")

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    with sampler:
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for i in range(steps):
                model.step(warmup + i, stream)
            ev1.record(stream)
        stream.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    total_ms = ev0.elapsed_time(ev1)
    for s in model.sets:
        for d in s:
            st = d["lay"].check(stream)
            if st != 0:
                raise RuntimeError(f"{wl.name}: device error during timing: status {st}")
    max_ms = max_over_ranks(total_ms, world, dev)
    res = {"workload": wl.name, "desc": wl.note,
           "layers": [dict(fmt=l.fmt, M=l.M, K=l.K, N=l.N, epi=l.epi) for l in wl.layers],
           "value": round(weak_scaling_tflops(flops_step, world, steps, max_ms), 2),
           "unit": "TFLOP/s", "steps": steps, "ms_per_step": round(max_ms / steps, 5),
           "clocks": sampler.summary(), "sets": nsets,
           "set_mb": round(per_set / 2 ** 20, 1),
           "gpu_launches": model.launches_per_step() * steps,
           "fused_quant": [j for j, f in enumerate(model.fused) if f]}
    # the quantize kernels first, after a pause: a sustained GEMM loop holds
    # the SM clock down at the power cap, and these short HBM-bound kernels
    # also need SM cycles for their conversions
    time.sleep(1.0)
    with ClockSampler(dev.index if dev.index is not None else 0) as qs:
        res["quant_roofline"] = quant_roofline(model, stream, peaks, peak_src)
    res["quant_clocks"] = qs.summary()
    with ClockSampler(dev.index if dev.index is not None else 0) as gs:
        res["gemm_roofline"] = gemm_roofline(model, stream, peaks, peak_src, args.gemm_ms)
    res["gemm_clocks"] = gs.summary()
    if e2e:
        res["e2e"] = run_e2e(model, stream, dev, args, world, flops_step)
    model.close()
    del model
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def main_ours(args):
    import torch
    import torch.distributed as dist

    rank, local_rank, world = dist_env()
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    wl = with_tokens(WORKLOADS[args.workload], args.tokens)
    head = measure(wl, args, dev, rank, world, args.steps, args.warmup, peaks, peak_src,
                   e2e=not args.no_e2e)
    sweep = []
    if not args.no_sweep and args.workload == DEFAULT_WORKLOAD and not args.tokens:
        for name in SWEEP:
            sweep.append(measure(WORKLOADS[name], args, dev, rank, world, args.sweep_steps,
                                 max(3, args.warmup // 2), peaks, peak_src, e2e=False))

    cpu = None
    if not args.no_cpu and world == 1 and rank == 0:
        v, rows, dt, cores = cpu_baseline(wl, args.cpu_seconds)
        cpu = {"value": round(v, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": f"{rows} rows of each of the {len(wl.layers)} layer(s) of {wl.name} "
                         f"({', '.join(f'{l.fmt} {l.M}x{l.K}x{l.N}' for l in wl.layers)}), "
                         f"quantize + GEMM + epilogue, {dt:.1f} s"}

    if rank == 0:
        # the dominant kernel: the GEMM with the largest time per step
        gr = head["gemm_roofline"]
        dom = max(gr, key=lambda r: r["gemm_ms"])
        roofline = dict(dom)
        roofline["gemm_share"] = round(sum(r["gemm_ms"] for r in gr) / head["ms_per_step"], 4)
        fmts = sorted(set(l.fmt for l in wl.layers))
        line = {
            "metric": "quantized DiT linear TFLOP/s at FLUX shapes",
            "value": head["value"], "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "+".join({"fp8": "fp8", "nvfp4": "nvfp4", "w8a16": "bf16"}[f] for f in fmts)
                     + " (fp32 accumulate)",
            "data": "synthetic (seeded FLUX-shaped activations and random-init weights)",
            "config": {"workload": wl.name, "desc": wl.note, "layers": head["layers"],
                       "global_tokens": wl.layers[0].M * world, "parallelism": f"replicas{world}",
                       "fused_quant": head["fused_quant"],
                       "l2": f"inputs rotate over {head['sets']} sets ({head['set_mb']:.0f} MB "
                             "each, > 126 MB L2): no set is L2-resident when reused"},
            "roofline": roofline,
            "roofline_by_layer": gr,
            "quant_roofline": head["quant_roofline"],
            "cpu_baseline": cpu,
            "e2e": head.get("e2e"),
            "gpu_launches": head["gpu_launches"],
            "clocks": head["clocks"],
            "gemm_loop_clocks": head["gemm_clocks"],
            "quant_loop_clocks": head["quant_clocks"],
            "sweep": sweep,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_e2e(model, stream, dev, args, world, flops_step):
    """Same metric through the public API with host buffers: every step copies
    its activations in from pinned host memory, runs quantize + GEMM +
    epilogue, and copies its results out to pinned host memory.  Steps are
    pipelined the way a serving loop would run them: uploads on one stream,
    layers on the compute stream, readbacks on a third, two device buffer sets
    alternating, so step i+1's upload and step i-1's readback overlap step i's
    kernels.  The timed region runs from the first upload to the last readback."""
    import torch
    nb = min(2, len(model.sets))
    L = model.wl.layers
    ins = [i for i, l in enumerate(L) if not l.chained]                      # uploaded
    outs = [i for i in range(len(L)) if i + 1 >= len(L) or not L[i + 1].chained]  # read back
    x_host = {i: model.sets[0][i]["x"].cpu().pin_memory() for i in ins}
    out_host = [{i: torch.empty(tuple(model.sets[0][i]["out"].shape), dtype=torch.bfloat16)
                 .pin_memory() for i in outs} for _ in range(nb)]
    s_up, s_down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    up_done = [ev() for _ in range(nb)]
    comp_done = [ev() for _ in range(nb)]
    down_done = [ev() for _ in range(nb)]
    step_bytes_out = sum(t.numel() * 2 for t in out_host[0].values())
    steps = max(3, min(args.steps, 50, int(4e10 // max(1, step_bytes_out))))
    started = [False] * nb

    def one(i):
        j = i % nb
        layers = model.sets[j]
        if started[j]:
            s_up.wait_event(comp_done[j])        # step i-nb has consumed its inputs
        with torch.cuda.stream(s_up):
            for li in ins:
                layers[li]["x"].copy_(x_host[li], non_blocking=True)
        up_done[j].record(s_up)
        stream.wait_event(up_done[j])
        if started[j]:
            stream.wait_event(down_done[j])      # step i-nb's results have left
        model.run_layers(layers, stream, amax_from=model.sets[(j + 1) % len(model.sets)])
        comp_done[j].record(stream)
        s_down.wait_event(comp_done[j])
        with torch.cuda.stream(s_down):
            for li in outs:
                out_host[j][li].copy_(layers[li]["out"], non_blocking=True)
        down_done[j].record(s_down)
        started[j] = True

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    for i in range(steps):
        one(3 + i)
    s_up.wait_stream(s_down)
    e1.record(s_up)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    return {"value": round(weak_scaling_tflops(flops_step, world, steps, ms), 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(sum(t.numel() * 2 for t in x_host.values())),
            "d2h_bytes_per_step": int(step_bytes_out), "steps": steps,
            "pipelined": "upload, compute and readback streams, two buffer sets"}


# ---------------------------------------------------------------- reference

def main_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return
    import oracle
    wl = WORKLOADS[args.workload]
    ols = oracle_layers(wl)
    per_row = sum(2.0 * l.N * l.K for l in wl.layers)
    Mmin = min(l.M for l in wl.layers)
    # bounded per-step row sample so that warm-up + steps finish in a few minutes
    budget_s = 150.0 / max(1, args.steps + args.warmup)

    def gemm_rows(rows):
        t0 = time.perf_counter()
        for ol in ols:
            ol.gemm(0, rows)
        return time.perf_counter() - t0

    probe = 1
    t1 = gemm_rows(probe)
    while t1 < 0.5 and probe < Mmin:  # size the per-step sample from a timed probe
        probe = min(Mmin, probe * 4)
        t1 = gemm_rows(probe)
    rows = int(max(1, min(Mmin, probe * budget_s / max(t1, 1e-6))))

    def step(i):
        for ol in ols:
            r0 = (i * rows) % max(1, ol.layer.M - rows + 1)
            ol.run(r0, rows)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = time.perf_counter() - t0
    value = per_row * rows * args.steps / dt / 1e12
    cores = oracle.num_threads()
    fmts = sorted(set(l.fmt for l in wl.layers))
    line = {
        "impl": "reference", "metric": "quantized DiT linear TFLOP/s at FLUX shapes",
        "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded FLUX-shaped activations and random-init weights)",
        "config": {"workload": wl.name, "desc": wl.note, "formats": fmts,
                   "layers": [dict(fmt=l.fmt, M=l.M, K=l.K, N=l.N, epi=l.epi) for l in wl.layers]},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"{rows} rows of each layer per step (quantize + GEMM + "
                                   "epilogue)"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        main_reference(a)
    else:
        main_ours(a)
