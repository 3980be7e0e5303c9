#!/usr/bin/env python
"""Benchmark of the blockwise-FP8 linear layer at Qwen3-1.7B shapes on B200.

One step = the 28-layer linear sweep of one micro-batch (2 x 4096 = 8192
tokens): for every layer, for each of the four linears (fused QKV
[4096, 2048], o_proj [2048, 2048], gate_up [12288, 2048], down [2048, 6144])

    forward   quantize X (1x128 row-wise + along-token, one read)
              quantize W (128x128 blocks + transposed codes)
              fprop      Y  = X W^T
    backward  quantize dY (row-wise + along-token)          (layers in reverse)
              dgrad      dX = dY W
              wgrad      dW = dY^T X

i.e. every step of the hot path, 672 launches and 69.27 TFLOP of GEMM work
per step, all through the C ABI (libfp8blk.so).  Inputs are seeded synthetic
tensors with the shapes and value distributions of the sweep (per layer
17.8 GB / 28 = 637 MB of bf16 inputs; 17.8 GB per step, far above the 126 MB
L2, so no flush is needed between steps).

Reported (one JSON line on rank 0):
  value      GEMM TFLOP per step x steps / device time of the timed steps,
             inputs resident in HBM; each timed step replays a captured CUDA
             graph of the step's 672 launches (kernels launched with
             programmatic dependent launch, so one's prologue overlaps the
             previous one's tail); per-kernel times come from three extra
             replays of graphs with an event-record node between every two
             launches, run after the timed region;
  e2e        the same metric with inputs in pinned host memory and results
             copied back: per layer, host->device copy of X, W, dY, the 24
             launches, device->host copy of Y, dX, dW, pipelined on three
             streams (host ring of 4 layers' buffers reused across the 28);
  roofline   for the kernel with the largest share of device time;
  cpu_baseline  the CPU oracle, as it stands, on a bounded row sample.

--impl reference times the CPU oracle alone (the reference arm of this
build): each step computes a bounded row sample of the step's 12 GEMM
shapes; rank 0 only.

Multi-GPU (torchrun): every rank runs the whole step on its own micro-batch
(data-parallel replicas, no collective on the data path); the timing is the
maximum over ranks and value counts the work of all ranks.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "blockwise-FP8 linear TFLOPS at Qwen3-1.7B shapes; % of B200 dense FP8 peak"
UNIT = "TFLOPS"
FP8_DENSE_SPEC_TFLOPS = 4500.0          # NVIDIA B200 dense FP8 (no sparsity)
FP8_PER_BF16 = 2.0                      # nominal dense FP8 : BF16 rate
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TOKENS = 8192
LAYERS = 28
# DRAM bytes of one captured launch per kernel kind (dram__bytes_read.sum +
# dram__bytes_write.sum from `ncu --set full`), with the launch they belong to.
# Valid only for the kernels they were taken on; the profiles/ summaries give
# the commands.  Remove an entry when its kernel changes.
NCU_TRAFFIC_BYTES_PER_LAUNCH: dict = {
    "gemm_rowblock": (204918016.0, "gate_up fprop 8192x12288x2048 (algorithmic 243.3 MB); kernel of commit 64d796a"),
    "gemm_outer": (176350976.0, "gate_up wgrad 12288x2048x8192, split schedule (algorithmic 167.8 MB plus the "
                                "partial sums); kernel of commit 64d796a"),
    "quant_act": (358906112.0, "gate_up gradient 8192x12288, both layouts (algorithmic 408.9 MB); kernel of "
                               "commit 968e0c3"),
}


def parse():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=LAYERS, help="layers per step (28 = the full sweep)")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target length of the oracle sample")
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="--impl reference: oracle work of all warm-up and timed steps together")
    ap.add_argument("--graphs", type=int, default=8, help="distinct captured step graphs")
    ap.add_argument("--no-ceiling", action="store_true", help="skip the FP8 library ceiling measurement")
    ap.add_argument("--no-split", action="store_true",
                    help="GEMMs without a workspace: whole tiles only, no split schedule")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the per-launch timing of the fused SwiGLU producer and the FP32 main-grad wgrad")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ workload

def linear_shapes():
    from blockwise_fp8_pretraining_b200 import synthetic as syn

    return list(syn.LAYER_LINEARS)


def step_gemm_flops(layers: int) -> float:
    return layers * sum(3 * 2.0 * TOKENS * n * k for _, n, k in linear_shapes())


class Sweep:
    """Device buffers and the launch list of one step."""

    def __init__(self, layers: int, device, seed_base: int, no_split: bool = False):
        import torch

        from blockwise_fp8_pretraining_b200 import synthetic as syn

        self.torch = torch
        self.layers = layers
        self.device = device
        T = TOKENS
        e = lambda shape, dt: torch.empty(shape, dtype=dt, device=device)
        u8, f32, bf = torch.uint8, torch.float32, torch.bfloat16
        self.shared = {}
        for name, n, k in linear_shapes():
            self.shared[name] = {
                "xq": e((T, k), u8), "sx": e((k // 128, T), f32), "wq": e((n, k), u8),
                "y": e((T, n), bf), "dyq": e((T, n), u8), "sdy": e((n // 128, T), f32),
                "dyqT": e((n, T), u8), "sdyT": e((T // 128, n), f32),
                "dx": e((T, k), bf), "dw": e((n, k), bf),
            }
        # GEMM workspace: shapes whose last wave of tiles would leave CTA
        # pairs idle run the split schedule (all launches share one stream)
        import blockwise_fp8_pretraining_b200 as fp8

        self.ws = fp8.fp8_gemm_workspace(device)
        self.ws_arg = (ctypes.c_void_p(self.ws.data_ptr()), ctypes.c_size_t(self.ws.numel()))
        if no_split:
            self.ws_arg = (ctypes.c_void_p(0), ctypes.c_size_t(0))
        self.layer = []
        for l in range(layers):
            gen = torch.Generator(device=device)
            gen.manual_seed(seed_base + l)
            inputs = syn.layer(seed_base + l, device=device, gen=gen)
            per = {}
            for name, n, k in linear_shapes():
                per[name] = dict(inputs[name])
                per[name].update({
                    "xqT": e((k, T), u8), "sxT": e((T // 128, k), f32),
                    "wqT": e((k, n), u8), "sw": e((n // 128, k // 128), f32),
                })
            self.layer.append(per)
        torch.cuda.synchronize()

    # A launch: (kind, c function name, argument builder taking the stream
    # handle and returning the ctypes argument tuple, flop, algorithmic bytes)
    def _launches_linear(self, per, sh, name, n, k, phase):
        out = self._launches_linear_unlabeled(per, sh, name, n, k, phase)
        labels = {"fp8_quantize_act_1x128": "quantize act", "fp8_quantize_weight_128x128": "quantize weight",
                  "fp8_block_gemm_fprop": "fprop", "fp8_block_gemm_dgrad": "dgrad", "fp8_block_gemm_wgrad": "wgrad"}
        return [(kind, fname, argf, flop, nbytes, f"{name} {labels[fname]}" +
                 (" (dY)" if fname == "fp8_quantize_act_1x128" and phase == "bwd" else ""))
                for kind, fname, argf, flop, nbytes in out]

    def _launches_linear_unlabeled(self, per, sh, name, n, k, phase):
        T = TOKENS
        P = lambda t: ctypes.c_void_p(t.data_ptr())
        ws = self.ws_arg
        out = []
        if phase == "fwd":
            x, w = per["x"], per["w"]
            out.append(("quant_act", "fp8_quantize_act_1x128",
                        lambda s, x=x: (P(x), T, k, 3, P(sh["xq"]), P(sh["sx"]), P(per["xqT"]), P(per["sxT"]), s),
                        0.0, T * k * (2 + 1 + 1 + 8 / 128)))
            out.append(("quant_weight", "fp8_quantize_weight_128x128",
                        lambda s, w=w: (P(w), n, k, P(sh["wq"]), P(per["sw"]), P(per["wqT"]), s),
                        0.0, n * k * (2 + 1 + 1) + 4 * (n // 128) * (k // 128)))
            out.append(("gemm_rowblock", "fp8_block_gemm_fprop",
                        lambda s: (P(sh["xq"]), P(sh["sx"]), P(sh["wq"]), P(per["sw"]), P(sh["y"]), T, n, k, *ws, s),
                        2.0 * T * n * k, T * k + n * k + 2 * T * n))
        else:
            dy = per["dy"]
            out.append(("quant_act", "fp8_quantize_act_1x128",
                        lambda s, dy=dy: (P(dy), T, n, 3, P(sh["dyq"]), P(sh["sdy"]), P(sh["dyqT"]), P(sh["sdyT"]), s),
                        0.0, T * n * (2 + 1 + 1 + 8 / 128)))
            out.append(("gemm_rowblock", "fp8_block_gemm_dgrad",
                        lambda s: (P(sh["dyq"]), P(sh["sdy"]), P(per["wqT"]), P(per["sw"]), P(sh["dx"]), T, n, k, *ws, s),
                        2.0 * T * n * k, T * n + n * k + 2 * T * k))
            out.append(("gemm_outer", "fp8_block_gemm_wgrad",
                        lambda s: (P(sh["dyqT"]), P(sh["sdyT"]), P(per["xqT"]), P(per["sxT"]), P(sh["dw"]), n, k, T, *ws, s),
                        2.0 * T * n * k, T * n + T * k + 2 * n * k))
        return out

    def launches(self):
        shapes = linear_shapes()
        out = []
        for l in range(self.layers):
            for name, n, k in shapes:
                out += self._launches_linear(self.layer[l][name], self.shared[name], name, n, k, "fwd")
        for l in reversed(range(self.layers)):
            for name, n, k in reversed(shapes):
                out += self._launches_linear(self.layer[l][name], self.shared[name], name, n, k, "bwd")
        return out


def extra_launches(sweep):
    """Launches of the kernels outside the step's sweep, on the step's own
    buffers (after it has run): the fused SwiGLU producer on every layer's
    gate_up fprop output (H's codes for the down projection without H in
    memory); the RMSNorm row statistic and the fused RMSNorm producer on
    every layer's qkv and gate_up input, taken as the norm's input (X's
    codes without X in memory); and the wgrad of every linear accumulated
    into FP32 main gradients."""
    import torch

    T = TOKENS
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    out = []
    if not hasattr(sweep, "norm_gamma"):
        gen = torch.Generator(device=sweep.device)
        gen.manual_seed(4321)
        hidden = dict((name, k) for name, _, k in linear_shapes())["qkv"]
        sweep.norm_gamma = (1.0 + 0.1 * torch.randn(hidden, generator=gen, device=sweep.device)).to(torch.bfloat16)
        sweep.norm_rstd = torch.empty(T, dtype=torch.float32, device=sweep.device)
    gam, rstd = sweep.norm_gamma, sweep.norm_rstd
    for l in range(sweep.layers):
        for name in ("qkv", "gate_up"):
            per, sh = sweep.layer[l][name], sweep.shared[name]
            k = per["x"].shape[1]
            out.append(("rmsnorm_rstd", "fp8_rmsnorm_rstd",
                        lambda s, per=per, k=k: (P(per["x"]), T, k, ctypes.c_float(1e-6), P(rstd), s),
                        0.0, T * k * 2 + T * 4, f"{name} rmsnorm rstd"))
            out.append(("rmsnorm_quant_fused", "fp8_rmsnorm_quantize_1x128",
                        lambda s, per=per, sh=sh, k=k: (P(per["x"]), T, k, P(rstd), P(gam), 3, P(sh["xq"]),
                                                        P(sh["sx"]), P(per["xqT"]), P(per["sxT"]), s),
                        0.0, T * k * (2 + 1 + 1 + 8 / 128) + T * 4 + k * 2, f"{name} fused rmsnorm producer"))
    ffn = dict((name, n) for name, n, _ in linear_shapes())["gate_up"] // 2
    gu, dn = sweep.shared["gate_up"], sweep.shared["down"]
    for l in range(sweep.layers):
        per = sweep.layer[l]["down"]
        out.append(("swiglu_quant_fused", "fp8_swiglu_quantize_1x128",
                    lambda s, per=per: (P(gu["y"]), T, ffn, 3, P(dn["xq"]), P(dn["sx"]), P(per["xqT"]),
                                        P(per["sxT"]), s),
                    0.0, T * ffn * (2 * 2 + 1 + 1 + 8 / 128), "fused SwiGLU producer"))
    if not hasattr(sweep, "main_grad"):
        sweep.main_grad = {name: torch.zeros((n, k), dtype=torch.float32, device=sweep.device)
                           for name, n, k in linear_shapes()}
    for l in range(sweep.layers):
        for name, n, k in linear_shapes():
            sh, per, mg = sweep.shared[name], sweep.layer[l][name], sweep.main_grad[name]
            out.append(("gemm_outer_accum_f32", "fp8_block_gemm_wgrad_accum_f32",
                        lambda s, sh=sh, per=per, mg=mg, n=n, k=k: (P(sh["dyqT"]), P(sh["sdyT"]), P(per["xqT"]),
                                                                   P(per["sxT"]), P(mg), n, k, T,
                                                                   *sweep.ws_arg, s),
                        2.0 * T * n * k, T * n + T * k + 2 * 4 * n * k, f"{name} wgrad accumulate"))
    return out


def run_launches(lib, launches, stream_handle, events=None):
    s = ctypes.c_void_p(stream_handle)
    for i, (_, fname, argf, *_rest) in enumerate(launches):
        if events is not None:
            events[i].record()
        st = getattr(lib, fname)(*argf(s))
        if st != 0:
            raise RuntimeError(f"{fname} returned status {st}: {lib.fp8_last_cuda_error().decode()}")
    if events is not None:
        events[len(launches)].record()


# -------------------------------------------------------------------- clocks

REJECT_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def clock_rejects(clk: dict) -> bool:
    """Whether the timing rules reject a timed region by its clock record: a
    hardware or thermal slowdown was active, or the SM clock sat well below
    its maximum with no reason reported (a clock lock left behind).  Such a
    region is measured once more.  sw_power_cap alone is normal under load."""
    reasons = clk.get("reasons") or []
    if any(r in REJECT_REASONS for r in reasons):
        return True
    sm, smax = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    return bool(sm and smax and not reasons and sm < 0.8 * smax)


def nvidia_smi_id(local_rank: int, visible) -> str:
    """The `nvidia-smi -i` identifier of this rank's GPU: the local rank's
    entry of CUDA_VISIBLE_DEVICES (an index or a UUID, both of which
    nvidia-smi accepts), else the local rank itself."""
    if visible is None or not visible.strip():
        return str(local_rank)
    ids = [v.strip() for v in visible.split(",") if v.strip()]
    return ids[local_rank] if local_rank < len(ids) else str(local_rank)


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu: str):
        self.gpu = gpu
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, power, reasons = [], [], [], set()
        for line in self.lines:
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                smax.append(float(p[2]))
                power.append(float(p[3]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, p[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------- FP8 library ceiling

CEILING_SHAPES = (("8192x8192x8192", 8192, 8192, 8192),
                  ("gate_up_fprop_8192x12288x2048", 8192, 12288, 2048))


def fp8_library_ceiling(device, reps: int = 20, warmup: int = 5):
    """TFLOPS of the library's E4M3 GEMM with one scale per tensor
    (torch._scaled_mm, a cuBLASLt kernel; no blockwise scales, no promotion)
    at 8192^3 and at the gate_up fprop shape, timed with CUDA events on the
    current stream, outside the timed region.  It is the measured ceiling
    beside which the blockwise kernels' TFLOPS are read, not a path of this
    library."""
    import torch

    out = {"kind": "torch._scaled_mm per-tensor E4M3 -> BF16 (cuBLASLt)", "reps": reps}
    clocks = ClockSampler(nvidia_smi_id(torch.cuda.current_device(), os.environ.get("CUDA_VISIBLE_DEVICES")))
    clocks.start()
    try:
        for label, m, n, k in CEILING_SHAPES:
            g = torch.Generator(device=device)
            g.manual_seed(7)
            a = torch.randn((m, k), device=device, generator=g).to(torch.float8_e4m3fn)
            b = torch.randn((n, k), device=device, generator=g).to(torch.float8_e4m3fn)
            one = torch.ones((), device=device, dtype=torch.float32)

            def run():
                return torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)

            for _ in range(warmup):
                run()
            torch.cuda.synchronize()
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record()
            for _ in range(reps):
                run()
            t1.record()
            torch.cuda.synchronize()
            ms = t0.elapsed_time(t1) / reps
            out[label] = {"tflops": 2.0 * m * n * k / (ms * 1e-3) / 1e12, "us": 1e3 * ms}
            del a, b
    except Exception as e:  # noqa: BLE001 - reported, not fatal
        out["error"] = f"{type(e).__name__}: {e}"[:300]
    out["clocks"] = clocks.stop()
    return out


def roofline_fracs(tflops: float, pk: dict, peak_kind: str, ceiling: dict | None) -> dict:
    """A GEMM's TFLOPS as a fraction of each denominator it is read against:
    the spec dense FP8 peak, twice the measured BF16 peaks (burst and
    sustained; the nominal FP8:BF16 ratio) and the measured FP8 library
    ceiling at 8192^3 and at the gate_up shape."""
    fr = {"spec_fp8_dense_4500": tflops / FP8_DENSE_SPEC_TFLOPS,
          f"2x_{peak_kind}_bf16_burst": tflops / (FP8_PER_BF16 * pk["bf16_tflops"]),
          f"2x_{peak_kind}_bf16_sustained": tflops / (FP8_PER_BF16 * pk["bf16_tflops_sustained"])}
    for label, _, _, _ in CEILING_SHAPES:
        v = (ceiling or {}).get(label)
        if v and v.get("tflops"):
            fr[f"fp8_library_{label}"] = tflops / v["tflops"]
    return fr


# ------------------------------------------------------------------ CPU oracle

def calibrate_rows(run_seconds, threads: int, seconds: float, max_rows: int = TOKENS) -> int:
    """Rows per GEMM for a sample that takes about `seconds`.

    The oracle parallelises over output rows, so a sample's time only grows
    with its rows once every thread has one: calibrate on multiples of the
    thread count, doubling until a run takes at least half a second, and fit
    time = a + b * rows through the last two runs.  `run_seconds(rows)`
    times one sample.  The result is a multiple of `threads` (at least one
    row per thread) and at most `max_rows`."""
    threads = max(1, int(threads))
    r = min(threads, max_rows)
    pts = [(r, run_seconds(r))]
    while pts[-1][1] < 0.5 and r < max_rows:
        r = min(max_rows, 2 * r)
        pts.append((r, run_seconds(r)))
    r2, t2 = pts[-1]
    slope, intercept = t2 / r2, 0.0
    if len(pts) >= 2:
        r1, t1 = pts[-2]
        if t2 > t1:
            slope = (t2 - t1) / (r2 - r1)
            intercept = max(0.0, t2 - slope * r2)
    rows = int((seconds - intercept) / slope) if seconds > intercept else 0
    rows = rows // threads * threads
    return max(min(threads, max_rows), min(max_rows, rows))


class OracleSample:
    """The CPU oracle's GEMMs on row samples of one layer's 12 GEMM shapes
    (fprop, dgrad and wgrad of qkv, o_proj, gate_up and down over the
    8192-token micro-batch).  The operands are generated and quantized by
    the oracle once, when the object is made; that is not timed."""

    def __init__(self, seed: int = 0):
        import oracle
        from blockwise_fp8_pretraining_b200 import synthetic as syn

        self.oracle = oracle
        lay = syn.layer(seed)
        self.prepared = []
        for name, n, k in syn.LAYER_LINEARS:
            t = lay[name]
            xb, wb, dyb = syn.bf16_bits(t["x"]), syn.bf16_bits(t["w"]), syn.bf16_bits(t["dy"])
            xq, sx = oracle.quantize_act_rowwise(xb)
            xqT, sxT = oracle.quantize_act_colwise(xb)
            wq, sw = oracle.quantize_weight(wb)
            dyq, sdy = oracle.quantize_act_rowwise(dyb)
            dyqT, sdyT = oracle.quantize_act_colwise(dyb)
            self.prepared.append((n, k, xq, sx, xqT, sxT, wq, sw, dyq, sdy, dyqT, sdyT))
        self.threads = oracle.num_threads()

    def run(self, rows: int):
        """The first `rows` output rows of each GEMM; returns (flop, seconds)."""
        import numpy as np

        orc = self.oracle
        flop = 0.0
        t0 = time.perf_counter()
        for (n, k, xq, sx, xqT, sxT, wq, sw, dyq, sdy, dyqT, sdyT) in self.prepared:
            r_tok = np.arange(rows)
            r_n = np.arange(min(rows, n))
            orc.gemm_fprop(xq, sx, wq, sw, rows=r_tok)
            orc.gemm_dgrad(dyq, sdy, wq, sw, rows=r_tok)
            orc.gemm_wgrad(dyqT, sdyT, xqT, sxT, rows=r_n)
            flop += 2.0 * rows * n * k * 2 + 2.0 * r_n.size * k * TOKENS
        return flop, time.perf_counter() - t0

    def rows_for(self, seconds: float) -> int:
        return calibrate_rows(lambda r: self.run(r)[1], self.threads, seconds)

    @staticmethod
    def describe(rows: int) -> str:
        return (f"oracle fprop+dgrad+wgrad of the 4 linears of one layer, first {rows} output rows each "
                f"(8192-token micro-batch; operands quantized by the oracle beforehand, untimed)")


# ------------------------------------------------------------------ reference

def run_reference(args, rank):
    if rank != 0:
        return 0
    import oracle

    oracle.build()
    sample = OracleSample()
    # size one step so that the warm-up and timed steps together take about
    # args.ref_seconds of oracle work
    rows = sample.rows_for(args.ref_seconds / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        sample.run(rows)
    total_flop = total_t = 0.0
    for _ in range(args.steps):
        flop, secs = sample.run(rows)
        total_flop += flop
        total_t += secs
    value = total_flop / total_t / 1e12
    desc = sample.describe(rows)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "CPU oracle on a row sample of the Qwen3-1.7B 28-layer linear sweep's "
                               "GEMM shapes (one layer's fprop/dgrad/wgrad of qkv, o_proj, gate_up, down)",
                   "tokens": TOKENS, "rows_per_gemm": rows},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": sample.threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------- ours

def max_over_ranks(ms: float, device, world: int) -> float:
    """The slowest rank's device time: every rank enters this collective once."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(ms)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, flop_step: float, steps: int, elapsed_ms: float) -> float:
    """Whole-job throughput: every rank ran `steps` steps of `flop_step` in at most `elapsed_ms`."""
    return world * flop_step * steps / (elapsed_ms * 1e-3) / 1e12


def summarize_kernels(launches, events_by_graph, pk, peak_kind):
    """Per kind: launches, total ms, share, and roofline numbers."""
    kinds = {}
    for events in events_by_graph:
        for i, (kind, fname, _, flop, nbytes, *_label) in enumerate(launches):
            ms = events[i].elapsed_time(events[i + 1])
            d = kinds.setdefault(kind, {"launches": 0, "ms": 0.0, "flop": 0.0, "bytes": 0.0})
            d["launches"] += 1
            d["ms"] += ms
            d["flop"] += flop
            d["bytes"] += nbytes
    total = sum(d["ms"] for d in kinds.values())
    for d in kinds.values():
        d["share"] = d["ms"] / total if total else 0.0
        d["avg_us"] = 1e3 * d["ms"] / d["launches"]
        d["tflops"] = d["flop"] / (d["ms"] * 1e-3) / 1e12 if d["flop"] else None
        d["gbs"] = d["bytes"] / (d["ms"] * 1e-3) / 1e9
    return kinds


def back_to_back(lib, launches, stream, pk, peak_kind, replays: int = 3):
    """Per kernel kind: the step's launches of that kind, in step order, in
    one CUDA graph with nothing between them (so each launch's start-up
    overlaps the previous launch's tail, as in the step), replayed after one
    warm-up replay; CUDA events around each replay on the launching stream.
    Returns kind -> launches, mean microseconds per launch and rate."""
    import torch

    out = {}
    for kind in sorted({l[0] for l in launches}):
        sel = [l for l in launches if l[0] == kind]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            run_launches(lib, sel, torch.cuda.current_stream().cuda_stream)
        g.replay()
        torch.cuda.synchronize()
        ms = 0.0
        with torch.cuda.stream(stream):
            for _ in range(replays):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                g.replay()
                e1.record()
                e1.synchronize()
                ms += e0.elapsed_time(e1)
        g.reset()
        us = 1e3 * ms / (replays * len(sel))
        flop = sum(l[3] for l in sel) / len(sel)
        nbytes = sum(l[4] for l in sel) / len(sel)
        d = {"launches": len(sel) * replays, "avg_us": round(us, 2)}
        if flop:
            d["tflops"] = round(flop / (us * 1e-6) / 1e12, 1)
            d["frac_of"] = {k: round(v, 4) for k, v in roofline_fracs(d["tflops"], pk, peak_kind, None).items()}
        else:
            d["gbs"] = round(nbytes / (us * 1e-6) / 1e9, 1)
            d["frac_of_hbm"] = round(d["gbs"] / pk["hbm_gbs"], 4)
        out[kind] = d
    return out


def summarize_labels(launches, events_by_graph):
    """Mean device time per launch of each (linear, pass) of the step."""
    acc = {}
    for events in events_by_graph:
        for i, (kind, fname, _, flop, nbytes, *label) in enumerate(launches):
            if not label:
                continue
            d = acc.setdefault(label[0], {"n": 0, "ms": 0.0, "flop": flop, "bytes": nbytes})
            d["n"] += 1
            d["ms"] += events[i].elapsed_time(events[i + 1])
    out = {}
    for lab, d in acc.items():
        us = 1e3 * d["ms"] / d["n"]
        out[lab] = {"avg_us": round(us, 2)}
        if d["flop"]:
            out[lab]["tflops"] = round(d["flop"] / (us * 1e-6) / 1e12, 1)
        else:
            out[lab]["gbs"] = round(d["bytes"] / (us * 1e-6) / 1e9, 1)
    return out


def main_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import blockwise_fp8_pretraining_b200 as fp8

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=device)
    lib = fp8.load()
    fp8.fp8_clear_error()
    pk, peak_kind = peaks()

    sweep = Sweep(args.layers, device, seed_base=1000 * rank, no_split=args.no_split)
    launches = sweep.launches()
    flop_step = step_gemm_flops(args.layers)

    # warm-up eagerly once (sets kernel attributes outside capture)
    stream = torch.cuda.Stream(device=device)
    with torch.cuda.stream(stream):
        run_launches(lib, launches, stream.cuda_stream)
    torch.cuda.synchronize()

    # Timed steps replay graphs of the bare launch sequence: the kernels are
    # launched with programmatic stream serialization, and an event-record
    # node between two kernels would take away their overlap.  The per-kernel
    # breakdown comes from separate graphs with an event-record node between
    # every two launches, replayed after the timed region.
    ngraphs = max(1, min(args.graphs, args.steps))
    graphs = []
    for _ in range(ngraphs):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            run_launches(lib, launches, torch.cuda.current_stream().cuda_stream)
        graphs.append(g)
    nprof = max(1, min(3, args.steps))
    prof_graphs, events_by_graph = [], []
    for _ in range(nprof):
        evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(launches) + 1)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            run_launches(lib, launches, torch.cuda.current_stream().cuda_stream, evs)
        prof_graphs.append(g)
        events_by_graph.append(evs)
    torch.cuda.synchronize()

    for w in range(args.warmup):
        graphs[w % ngraphs].replay()
    torch.cuda.synchronize()

    def timed_steps():
        clocks = ClockSampler(nvidia_smi_id(local_rank, os.environ.get("CUDA_VISIBLE_DEVICES")))
        clocks.start()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            t_start.record()
            for s in range(args.steps):
                graphs[s % ngraphs].replay()
            t_end.record()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        return t_start.elapsed_time(t_end), clocks.stop()

    local_ms, clk = timed_steps()
    # every rank takes the same decision (and the same collectives)
    if max_over_ranks(1.0 if clock_rejects(clk) else 0.0, device, world) > 0.0:
        rejected = clk
        local_ms, clk = timed_steps()
        clk["remeasured_after"] = {"sm_mhz": rejected["sm_mhz"], "reasons": rejected["reasons"]}
    elapsed_ms = max_over_ranks(local_ms, device, world)
    err = fp8.fp8_get_error()
    if err != 0:
        raise RuntimeError(f"device error word {err} after the timed region")

    # per-kernel breakdown (not timed as a whole)
    for g in prof_graphs:
        g.replay()
    torch.cuda.synchronize()
    kinds = summarize_kernels(launches, events_by_graph, pk, peak_kind)
    by_label = summarize_labels(launches, events_by_graph)
    for g in prof_graphs:
        g.reset()
    prof_graphs.clear()
    value = job_tflops(world, flop_step, args.steps, elapsed_ms)

    # ---- end-to-end through host buffers
    e2e = None
    if not args.no_e2e:
        for g in graphs:
            g.reset()
        graphs.clear()
        e2e = run_e2e(args, lib, sweep, device, world)
        e2e_ms = max_over_ranks(e2e.pop("_elapsed_ms"), device, world)
        e2e["value"] = job_tflops(world, flop_step, args.e2e_steps, e2e_ms)

    # ---- each kind's launches back to back (programmatic dependent launch
    # between them, as in the step), timed by events around whole replays
    b2b = back_to_back(lib, launches, stream, pk, peak_kind)

    # ---- kernels outside the step, per launch (after the timed region)
    extra = None
    if not args.no_extra:
        xl = extra_launches(sweep)
        with torch.cuda.stream(stream):
            run_launches(lib, xl, stream.cuda_stream)          # warm-up, sets attributes
        torch.cuda.synchronize()
        xevents, xgraphs = [], []
        for _ in range(3):
            evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(xl) + 1)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                run_launches(lib, xl, torch.cuda.current_stream().cuda_stream, evs)
            xgraphs.append(g)
            xevents.append(evs)
        for g in xgraphs:
            g.replay()
        torch.cuda.synchronize()
        xk = summarize_kernels(xl, xevents, pk, peak_kind)
        for g in xgraphs:
            g.reset()
        if fp8.fp8_get_error() != 0:
            raise RuntimeError("device error word set by the extra kernels")
        ffn_elems = TOKENS * 6144
        extra = {k: {"launches": d["launches"], "avg_us": round(d["avg_us"], 2),
                     "tflops": None if d["tflops"] is None else round(d["tflops"], 1),
                     "gbs": round(d["gbs"], 1)} for k, d in xk.items()}
        sq = extra.get("swiglu_quant_fused")
        if sq:
            sq["frac_of_hbm"] = round(sq["gbs"] / pk["hbm_gbs"], 4)
            sq["algorithmic_bytes_per_launch"] = ffn_elems * (4 + 2 + 8 / 128)
            # an unfused SwiGLU kernel writes H in bf16 and the quantizer reads it back
            sq["hbm_bytes_saved_per_layer_vs_unfused"] = ffn_elems * 4
            sq["input"] = "each layer's gate_up fprop output [8192, 12288] (gate | up), both layouts out"
        rq = extra.get("rmsnorm_quant_fused")
        if rq:
            rq["frac_of_hbm"] = round(rq["gbs"] / pk["hbm_gbs"], 4)
            rq["input"] = ("each layer's qkv and gate_up input [8192, 2048] as RMSNorm's input (rstd from "
                           "rmsnorm_rstd), both layouts out")
            # unfused: the norm reads x and writes y, the quantizer reads y; fused: x is read twice
            rq["hbm_bytes_saved_per_launch_vs_unfused"] = TOKENS * 2048 * 2
        oa = extra.get("gemm_outer_accum_f32")
        if oa:
            oa["note"] = "wgrad of every linear added into FP32 main gradients (vector-reduction epilogue)"

    # ---- measured FP8 library ceiling (outside every timed region)
    ceiling = None if args.no_ceiling else fp8_library_ceiling(device)

    # ---- roofline of the dominant kernel
    dom_kind = max(kinds, key=lambda k: kinds[k]["ms"])
    dom = kinds[dom_kind]
    fp8_peak = FP8_PER_BF16 * pk["bf16_tflops_sustained"]
    if dom["flop"]:
        roofline = {"bound": "tensor", "kernel": dom_kind, "achieved": dom["tflops"], "peak": fp8_peak,
                    "unit": "TFLOP/s", "frac": dom["tflops"] / fp8_peak,
                    "peak_source": f"{peak_kind} bf16 sustained x {FP8_PER_BF16:g} (nominal fp8:bf16)",
                    "frac_of_spec_fp8_4500": dom["tflops"] / FP8_DENSE_SPEC_TFLOPS,
                    "frac_of": roofline_fracs(dom["tflops"], pk, peak_kind, ceiling)}
    else:
        roofline = {"bound": "hbm", "kernel": dom_kind, "achieved": dom["gbs"], "peak": pk["hbm_gbs"],
                    "unit": "GB/s", "frac": dom["gbs"] / pk["hbm_gbs"], "peak_source": peak_kind}
    bd = b2b.get(dom_kind, {})
    if bd.get("tflops"):
        roofline["achieved_back_to_back"] = bd["tflops"]
        roofline["frac_back_to_back"] = bd["tflops"] / roofline["peak"]
    elif bd.get("gbs"):
        roofline["achieved_back_to_back"] = bd["gbs"]
        roofline["frac_back_to_back"] = bd["gbs"] / roofline["peak"]
    tr = NCU_TRAFFIC_BYTES_PER_LAUNCH.get(dom_kind)
    roofline["traffic"] = tr[0] if tr else None
    if tr:
        roofline["traffic_launch"] = tr[1]
    roofline["achieved_over"] = (f"{dom['launches']} {dom_kind} launches (mixed shapes) of {len(events_by_graph)} "
                                 "extra replays of the step with an event between every two launches")
    q_ms = sum(d["ms"] for k, d in kinds.items() if k.startswith("quant"))
    q_bytes = sum(d["bytes"] for k, d in kinds.items() if k.startswith("quant"))
    q_gbs = q_bytes / (q_ms * 1e-3) / 1e9 if q_ms else None
    q_b2b = [(k, d) for k, d in b2b.items() if k.startswith("quant")]
    q_b2b_gbs = None
    if q_b2b:
        tot_bytes = sum(sum(l[4] for l in launches if l[0] == k) for k, _ in q_b2b)
        tot_us = sum(d["avg_us"] * sum(1 for l in launches if l[0] == k) for k, d in q_b2b)
        q_b2b_gbs = tot_bytes / (tot_us * 1e-6) / 1e9
    roofline_quant = {"bound": "hbm", "kernel": "all quantizers", "achieved": q_gbs, "peak": pk["hbm_gbs"],
                      "achieved_back_to_back": q_b2b_gbs,
                      "frac_back_to_back": (q_b2b_gbs / pk["hbm_gbs"]) if q_b2b_gbs else None,
                      "unit": "GB/s", "frac": (q_gbs / pk["hbm_gbs"]) if q_gbs else None,
                      "peak_source": peak_kind,
                      "traffic": NCU_TRAFFIC_BYTES_PER_LAUNCH.get("quant_act", (None,))[0],
                      "traffic_launch": NCU_TRAFFIC_BYTES_PER_LAUNCH.get("quant_act", (None, None))[1]}

    # ---- CPU oracle baseline (rank 0, one GPU only)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        sample = OracleSample()
        rows = sample.rows_for(args.cpu_seconds)
        flop, secs = sample.run(rows)
        cpu = {"value": flop / secs / 1e12, "unit": UNIT, "cores": sample.threads, "kind": "oracle",
               "sample": sample.describe(rows) + f"; {secs:.1f} s"}

    if rank == 0:
        gemm_ms = sum(d["ms"] for k, d in kinds.items() if k.startswith("gemm"))
        gemm_flop = sum(d["flop"] for d in kinds.values())
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
            "data": "synthetic (seeded; Qwen3-1.7B linear shapes, N(0,1) activations with 1% x30 outlier "
                    "channels, SwiGLU down-proj inputs, N(0,0.02) weights, N(0,1e-3) output grads)",
            "config": {"workload": f"Qwen3-1.7B linear sweep, {args.layers} layers x (qkv, o_proj, gate_up, down) "
                                   "x (fprop, dgrad, wgrad) with blockwise E4M3 quantizers, one 8192-token "
                                   "micro-batch (2 x 4096)",
                       "tokens": TOKENS, "layers": args.layers, "gemm_tflop_per_step": flop_step / 1e12,
                       "launches_per_step": len(launches),
                       "gemm_schedule": ("whole 256x256 tiles (no workspace)" if args.no_split else
                                         "split (slab ranges per CTA pair) where the last wave of 256x256 tiles "
                                         "would leave >5% of pairs idle, K >= 32 slabs and the work is at least "
                                         f"{fp8.GEMM_SPLIT_MIN_WORK_DEFAULT} tile-slabs per pair; whole tiles "
                                         "elsewhere"),
                       "l2": "no flush: 17.8 GB of distinct inputs per step >> 126 MB L2",
                       "parallelism": f"dp{world} replicas, no data-path collective"},
            "pct_of_fp8_dense_peak": 100.0 * value / FP8_DENSE_SPEC_TFLOPS,
            "gemm_only_tflops": gemm_flop / (gemm_ms * 1e-3) / 1e12 if gemm_ms else None,
            "kernels": {k: {"launches": d["launches"], "share": round(d["share"], 4),
                            "avg_us": round(d["avg_us"], 2),
                            "tflops": None if d["tflops"] is None else round(d["tflops"], 1),
                            "gbs": round(d["gbs"], 1),
                            **({"frac_of": {f: round(v, 4) for f, v in
                                            roofline_fracs(d["tflops"], pk, peak_kind, ceiling).items()}}
                               if d["tflops"] else {})}
                        for k, d in kinds.items()},
            "per_linear": by_label,
            "kernels_back_to_back": b2b,
            "fp8_library_tflops": ceiling,
            "kernels_outside_step": extra,
            "roofline": roofline,
            "roofline_quantize": roofline_quant,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": len(launches) * args.steps,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_e2e(args, lib, sweep, device, world):
    """Inputs from pinned host memory, results back to pinned host memory,
    pipelined per layer on a copy-in, a compute and a copy-out stream."""
    import torch

    ring = 4
    shapes = linear_shapes()
    T = TOKENS
    # host ring: 4 layers' inputs (filled from the device copies) and outputs
    host_in, host_out = [], []
    for r in range(ring):
        src = sweep.layer[r % sweep.layers]
        host_in.append({name: {t: src[name][t].cpu().pin_memory() for t in ("x", "w", "dy")}
                        for name, _, _ in shapes})
        host_out.append({name: {"y": torch.empty((T, n), dtype=torch.bfloat16).pin_memory(),
                                "dx": torch.empty((T, k), dtype=torch.bfloat16).pin_memory(),
                                "dw": torch.empty((n, k), dtype=torch.bfloat16).pin_memory()}
                         for name, n, k in shapes})
    # device staging: two slots of inputs and outputs
    slots = []
    for _ in range(2):
        slot = {}
        for name, n, k in shapes:
            slot[name] = {"x": torch.empty((T, k), dtype=torch.bfloat16, device=device),
                          "w": torch.empty((n, k), dtype=torch.bfloat16, device=device),
                          "dy": torch.empty((T, n), dtype=torch.bfloat16, device=device),
                          "y": torch.empty((T, n), dtype=torch.bfloat16, device=device),
                          "dx": torch.empty((T, k), dtype=torch.bfloat16, device=device),
                          "dw": torch.empty((n, k), dtype=torch.bfloat16, device=device)}
        slots.append(slot)
    h2d_bytes = sweep.layers * sum(2 * (T * k + n * k + T * n) for _, n, k in shapes)
    d2h_bytes = h2d_bytes

    s_in, s_cmp, s_out = (torch.cuda.Stream(device=device) for _ in range(3))

    def layer_launches(l, slot):
        out = []
        for name, n, k in shapes:
            per = dict(sweep.layer[l][name])
            per.update({"x": slot[name]["x"], "w": slot[name]["w"], "dy": slot[name]["dy"]})
            sh = dict(sweep.shared[name])
            sh.update({"y": slot[name]["y"], "dx": slot[name]["dx"], "dw": slot[name]["dw"]})
            out += sweep._launches_linear(per, sh, name, n, k, "fwd")
            out += sweep._launches_linear(per, sh, name, n, k, "bwd")
        return out

    plans = [[layer_launches(l, slots[l % 2]) for l in range(sweep.layers)]]

    def one_step():
        in_ready = [torch.cuda.Event() for _ in range(sweep.layers)]
        done = [torch.cuda.Event() for _ in range(sweep.layers)]
        out_done = [torch.cuda.Event() for _ in range(sweep.layers)]
        for l in range(sweep.layers):
            slot = slots[l % 2]
            hin, hout = host_in[l % ring], host_out[l % ring]
            with torch.cuda.stream(s_in):
                if l >= 2:
                    s_in.wait_event(done[l - 2])
                for name, _, _ in shapes:
                    for t in ("x", "w", "dy"):
                        slot[name][t].copy_(hin[name][t], non_blocking=True)
                in_ready[l].record()
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(in_ready[l])
                if l >= 2:
                    s_cmp.wait_event(out_done[l - 2])
                run_launches(lib, plans[0][l], s_cmp.cuda_stream)
                done[l].record()
            with torch.cuda.stream(s_out):
                s_out.wait_event(done[l])
                for name, _, _ in shapes:
                    for t in ("y", "dx", "dw"):
                        hout[name][t].copy_(slot[name][t], non_blocking=True)
                out_done[l].record()

    one_step()                      # warm-up
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for _ in range(args.e2e_steps):
        s_in.wait_stream(s_out)
        one_step()
    s_out.wait_stream(s_cmp)
    end.record(s_out)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    flop = step_gemm_flops(sweep.layers) * args.e2e_steps
    return {"value": flop / (ms * 1e-3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": h2d_bytes,
            "d2h_bytes_per_step": d2h_bytes, "steps": args.e2e_steps,
            "ms_per_step": ms / args.e2e_steps,
            "path": "C ABI with pinned host buffers, H2D/compute/D2H pipelined per layer",
            "_elapsed_ms": ms}


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        # one process per GPU: N > 1 is launched by torchrun, which sets
        # WORLD_SIZE; anything else would time a different number of replicas
        # than the line reports
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; launch N > 1 GPUs with "
              f"python -m torch.distributed.run --nproc-per-node {args.gpus} bench.py --gpus {args.gpus}",
              file=sys.stderr)
        return 2
    if args.impl == "reference":
        return run_reference(args, rank)
    return main_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
