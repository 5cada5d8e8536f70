#!/usr/bin/env python
"""Benchmark of the blockwise-FP8 linear layer (quantize + GEMM) on B200.

One step = one pass of the whole hot path over the four linear layers of a
Qwen3-1.7B transformer block at M = 8192 tokens (micro-batch 2 x sequence 4096):
QKV (2048 -> 4096), O (2048 -> 2048), gate/up (2048 -> 12288), down (6144 -> 2048).
For each linear: fp8_quant_act_dual(X) (row-wise and token-wise copies from one read),
fp8_quant_weight(W), fprop; fp8_quant_act_dual(dY), dgrad; wgrad -- 24 kernel
launches, 2.47 TFLOP of GEMM work (--separate-quant: the four single-layout passes,
32 launches).  The wgrad of each linear runs on a second stream, concurrently with
its dgrad (both need only the quantized dY and the retained quantized X / weight), so
that the SMs one GEMM leaves idle in its last round of tiles take the other's
(--no-overlap: one stream).  The metric is TFLOP/s of the whole step (2MNK summed over
the 12 GEMMs, divided by the time of all quantizers and GEMMs); the kernel roofline
comes from a separate one-stream pass with every GEMM bracketed by events.

The line also carries "variant_e8m0": the same step with power-of-two (E8M0) scales,
applied by the tensor cores' block-scaled MMA (the MXFP8 form of the recipe;
--no-variant skips it).

--sweep: the micro-batch knee sweep of a 28-layer step (M = 4096 ... 32768 tokens,
one stream), one JSON line per M and one naming the knee.

Inputs are seeded synthetic BF16 tensors (X ~ N(0,1) with 1% outlier channels x20,
W ~ N(0,0.02), dY ~ N(0,1e-3)); 637 MB per step, larger than the 126 MB L2, so no
flush is needed between steps.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun (N > 1) each rank runs an independent replica (weak scaling): the path
shards by tokens with no exchange in the data path.  --dp-grad reduce-scatter adds the
data-parallel weight-gradient exchange: each linear's wgrad accumulates into an FP32
main gradient (fp8_gemm_wgrad_acc32), which is reduce-scattered by rows over NCCL on
the stream that computed it, overlapping the next linear's kernels.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "blockwise-FP8 linear TFLOP/s (quant+GEMM, M=8192) and % of B200 FP8 peak"
UNIT = "TFLOP/s"
TOKENS = 8192
LINEARS = [("qkv", 2048, 4096), ("o", 2048, 2048), ("gate_up", 2048, 12288), ("down", 6144, 2048)]
WORKLOAD = "qwen3-1.7b block linears (qkv, o, gate_up, down) fprop+dgrad+wgrad, M=8192"
STEP_FLOPS = sum(3 * 2 * TOKENS * din * dout for _, din, dout in LINEARS)
FP8_OVER_BF16 = 4.5 / 2.25  # nominal dense FP8 : BF16 tensor throughput on B200
NOMINAL_FP8_TFLOPS = 4500.0  # B200 dense FP8 tensor peak as NVIDIA states it
NOMINAL_HBM_GBS = 8000.0     # B200 HBM3e bandwidth as NVIDIA states it (DGX figure)
# algorithmic bytes per element: BF16 read + per layout (E4M3 code + FP32 scale / 128)
DUAL_BYTES = 2 + 2 * (1 + 4 / 128)
ACT_BYTES = 2 + 1 + 4 / 128
WEIGHT_BYTES = 2 + 1 + 4 / (128 * 128)  # one FP32 scale per 128x128 block


def config_dict(n, overlap=True, dp_grad=False):
    return {
        "schedule": ("each linear's wgrad on a second stream, concurrent with its dgrad"
                     if overlap else "one stream"),
        "workload": WORKLOAD,
        "tokens": TOKENS,
        "linears": {name: [din, dout] for name, din, dout in LINEARS},
        "passes": "fprop+dgrad+wgrad with all quantizers (X and dY quantized once into both layouts)",
        "step_gflop": round(STEP_FLOPS / 1e9, 3),
        "l2": "inputs larger than L2 (637 MB of BF16 inputs per step), no flush",
        "parallelism": (f"dp{n}, FP32 main-grad (wgrad_acc32) reduce-scatter over NCCL, "
                        "overlapped with the next linear" if dp_grad
                        else f"replicas x{n}" if n > 1 else "single GPU"),
    }


# --------------------------------------------------------------------- helpers

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def kernel_source_digest():
    """SHA-256 over the GEMM kernel sources: ncu traffic figures are only reported
    while the kernel they were taken on is unchanged."""
    import hashlib
    h = hashlib.sha256()
    for f in ("gemm.cu", "ptx.cuh"):
        with open(os.path.join(ROOT, "blockwise_fp8_linear_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic():
    """DRAM bytes per GEMM launch from the committed ncu summary, or None if the
    summary is missing or was taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", "gemm_dram_traffic_qwen3_block_m8192.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("gemm_source_sha256") != kernel_source_digest():
        return None
    return rec.get("dram_bytes_per_launch")


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def __enter__(self):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.file.flush()

    def summary(self):
        rows = []
        try:
            with open(self.file.name) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
        finally:
            os.unlink(self.file.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        loaded = [v for v in sm if v > 0.5 * (max(smax) if smax else 0)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------- our arm

class LayerWork:
    """Device buffers of one step and the launch sequence through the C ABI."""

    def __init__(self, dev, host_inputs, separate=False, scales="fp32"):
        import torch
        import blockwise_fp8_linear_b200 as fb
        self.fb = fb
        self.torch = torch
        self.separate = separate
        # scales: "fp32" (amax/448, promoted per block on the CUDA cores) or "e8m0" (power
        # of two, scale blocks applied by the block-scaled MMA)
        self.e8 = scales == "e8m0"
        self.launches_per_step = (8 if separate else 6) * len(LINEARS)
        self.lin = []
        for (name, din, dout), (X, W, dY) in zip(LINEARS, host_inputs):
            t = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
            if self.e8:  # scale blocks of 512 bytes per 128 rows x 128-deep block
                sc = lambda rows, red: torch.empty(rows // 128, (red // 128) * 512, dtype=torch.uint8,
                                                   device=dev)
                scales_ = {"sx": sc(TOKENS, din), "sw": sc(dout, din), "sdy": sc(TOKENS, dout),
                           "sdyt": sc(dout, TOKENS), "sxt": sc(din, TOKENS)}
            else:
                f32 = lambda r, c: torch.empty(r, c, dtype=torch.float32, device=dev)
                scales_ = {"sx": f32(din // 128, TOKENS), "sw": f32(dout // 128, din // 128),
                           "sdy": f32(dout // 128, TOKENS), "sdyt": f32(TOKENS // 128, dout),
                           "sxt": f32(TOKENS // 128, din)}
            d = {
                "name": name, "din": din, "dout": dout,
                "X": t(X).to(dev), "W": t(W).to(dev), "dY": t(dY).to(dev),
                "qx": torch.empty(TOKENS, din, dtype=torch.uint8, device=dev),
                "qw": torch.empty(dout, din, dtype=torch.uint8, device=dev),
                "qdy": torch.empty(TOKENS, dout, dtype=torch.uint8, device=dev),
                "qdyt": torch.empty(dout, TOKENS, dtype=torch.uint8, device=dev),
                "qxt": torch.empty(din, TOKENS, dtype=torch.uint8, device=dev),
                **scales_,
                "Y": torch.empty(TOKENS, dout, dtype=torch.bfloat16, device=dev),
                "dX": torch.empty(TOKENS, din, dtype=torch.bfloat16, device=dev),
                "dW": torch.empty(dout, din, dtype=torch.bfloat16, device=dev),
            }
            self.lin.append(d)
        self.h2d_bytes = sum(d[k].numel() * 2 for d in self.lin for k in ("X", "W", "dY"))
        self.d2h_bytes = sum(d[k].numel() * 2 for d in self.lin for k in ("Y", "dX", "dW"))

    def step(self, gemm_events=None, side=None, hooks=None, reducer=None, quant_events=None):
        """Enqueue one step on the current stream.  gemm_events: optional list that
        receives (start, end, flops) CUDA-event triples around each GEMM; quant_events:
        likewise (start, end, kind, shape, bytes) around each quantizer.  side: an
        optional second stream; each linear's wgrad then runs there, after the dY
        quantizer and concurrently with the dgrad (the two are independent given
        dY), and the current stream waits for it at the end of the step.
        hooks: optional object with before(i), inputs_read(i) and after(i, main, side)
        called around linear i (used by the end-to-end pipeline)."""
        fb, torch = self.fb, self.torch
        L = fb.lib()
        main = torch.cuda.current_stream()
        T = TOKENS

        def gemm(mode, a, sa, b, sb, out, M, N, K, stream=None):
            s = stream if stream is not None else main
            if gemm_events is not None:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(s)
            fn = L.fp8_gemm_blockwise_e8m0 if self.e8 else L.fp8_gemm_blockwise
            rc = fn(mode, a.data_ptr(), sa.data_ptr(), b.data_ptr(), sb.data_ptr(), out.data_ptr(),
                    M, N, K, s.cuda_stream)
            if rc:
                raise fb.Fp8bwError(rc, "fp8_gemm_blockwise")
            if gemm_events is not None:
                e1.record(s)
                gemm_events.append((e0, e1, 2 * M * N * K))

        st = main.cuda_stream
        e8 = self.e8
        q_act = L.fp8_quant_act_e8m0 if e8 else L.fp8_quant_act
        q_act_t = L.fp8_quant_act_t_e8m0 if e8 else L.fp8_quant_act_t
        q_dual = L.fp8_quant_act_dual_e8m0 if e8 else L.fp8_quant_act_dual
        q_weight = L.fp8_quant_weight_e8m0 if e8 else L.fp8_quant_weight

        def chk(rc, what):
            if rc:
                raise fb.Fp8bwError(rc, what)

        def quant(fn, args, kind, shape, nbytes):
            if quant_events is not None:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(main)
            chk(fn(*args), kind)
            if quant_events is not None:
                e1.record(main)
                quant_events.append((e0, e1, kind, shape, nbytes))

        for i, d in enumerate(self.lin):
            din, dout = d["din"], d["dout"]
            if hooks is not None:
                hooks.before(i)
            if self.separate:
                chk(q_act(d["X"].data_ptr(), T, din, d["qx"].data_ptr(), d["sx"].data_ptr(), st), "qa")
            else:  # X read once: row-wise copy for fprop, token-wise copy kept for wgrad
                quant(q_dual, (d["X"].data_ptr(), T, din, d["qx"].data_ptr(), d["sx"].data_ptr(),
                               d["qxt"].data_ptr(), d["sxt"].data_ptr(), st),
                      "quant_act_dual", (T, din), T * din * DUAL_BYTES)
            quant(q_weight, (d["W"].data_ptr(), dout, din, d["qw"].data_ptr(),
                             d["sw"].data_ptr(), None, st),
                  "quant_weight", (dout, din), dout * din * WEIGHT_BYTES)
            gemm(fb.FPROP, d["qx"], d["sx"], d["qw"], d["sw"], d["Y"], T, dout, din)
            if self.separate:
                chk(q_act(d["dY"].data_ptr(), T, dout, d["qdy"].data_ptr(), d["sdy"].data_ptr(), st), "qa")
            else:
                quant(q_dual, (d["dY"].data_ptr(), T, dout, d["qdy"].data_ptr(), d["sdy"].data_ptr(),
                               d["qdyt"].data_ptr(), d["sdyt"].data_ptr(), st),
                      "quant_act_dual", (T, dout), T * dout * DUAL_BYTES)
            if self.separate:
                chk(q_act_t(d["dY"].data_ptr(), T, dout, d["qdyt"].data_ptr(), d["sdyt"].data_ptr(), st), "qt")
                chk(q_act_t(d["X"].data_ptr(), T, din, d["qxt"].data_ptr(), d["sxt"].data_ptr(), st), "qt")
            if hooks is not None:
                hooks.inputs_read(i)
            if side is not None:
                ready = torch.cuda.Event()
                ready.record(main)
                side.wait_event(ready)
            gemm(fb.DGRAD, d["qdy"], d["sdy"], d["qw"], d["sw"], d["dX"], T, din, dout)
            if reducer is None:
                gemm(fb.WGRAD, d["qdyt"], d["sdyt"], d["qxt"], d["sxt"], d["dW"], dout, din, T,
                     stream=side)
            else:
                # data-parallel step: this rank's token reduction accumulates into the
                # FP32 main gradient, which is then summed over the ranks (reduce-scatter)
                ws = side if side is not None else main
                dw32 = d.setdefault("dW32", torch.empty(dout, din, dtype=torch.float32,
                                                        device=d["dW"].device))
                with torch.cuda.stream(ws):
                    dw32.zero_()
                chk(L.fp8_gemm_wgrad_acc32(d["qdyt"].data_ptr(), d["sdyt"].data_ptr(),
                                           d["qxt"].data_ptr(), d["sxt"].data_ptr(),
                                           dw32.data_ptr(), dout, din, T, ws.cuda_stream),
                    "wgrad_acc32")
                reducer.launch(i, dw32, ws)
            if hooks is not None:
                hooks.after(i, main, side if side is not None else main)
        if side is not None:
            done = torch.cuda.Event()
            done.record(side)
            main.wait_event(done)
        if reducer is not None:
            reducer.wait()


def make_inputs(rank=0):
    from blockwise_fp8_linear_b200 import synth
    out = []
    for i, (name, din, dout) in enumerate(LINEARS):
        wl = 10 + i
        X = synth.normal_bf16(TOKENS, din, 1.0, seed=synth.seed_for(wl, 0 + 10 * rank), outliers=True)
        W = synth.normal_bf16(dout, din, 0.02, seed=synth.seed_for(wl, 1))
        dY = synth.normal_bf16(TOKENS, dout, 1e-3, seed=synth.seed_for(wl, 2 + 10 * rank))
        out.append((X, W, dY))
    return out


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """Max of a per-rank number over all ranks (the slowest rank's time)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def gemm_summary(gemm_events, work):
    """Mean device time and TFLOP/s of each of the step's 12 GEMMs (linear x mode) over
    the one-stream pass (events in launch order: per linear fprop, dgrad, wgrad)."""
    names = [(d["name"], m) for d in work.lin for m in ("fprop", "dgrad", "wgrad")]
    acc = {}
    for j, (e0, e1, f) in enumerate(gemm_events):
        key = names[j % len(names)]
        t, ff, n = acc.get(key, (0.0, 0.0, 0))
        acc[key] = (t + e0.elapsed_time(e1), ff + f, n + 1)
    return [{"gemm": f"{k[0]}_{k[1]}", "us": round(1e3 * t / n, 2),
             "tflops": round(ff / (t * 1e-3) / 1e12, 1)} for k, (t, ff, n) in acc.items()]


def quant_kernel_rows(dev, quant_rows, hbm_peak, steps):
    rows = []
    for r in quant_rows:
        shape = tuple(r["shape"])
        per_elem = DUAL_BYTES if r["kernel"] == "quant_act_dual" else WEIGHT_BYTES
        us = quant_stream_us(dev, r["kernel"], shape)
        gbs = shape[0] * shape[1] * per_elem / (us * 1e-6) / 1e9
        rows.append({"kernel": r["kernel"], "shape": list(shape), "launches_per_step":
                     r["launches"] // max(1, steps), "us": round(us, 2),
                     "gbs": round(gbs, 1), "frac": round(gbs / hbm_peak, 4),
                     "frac_of_nominal": round(gbs / NOMINAL_HBM_GBS, 4),
                     "in_step_us": r["us"]})
    return rows


def quant_summary(quant_events):
    """GB/s of each quantizer kind and shape (algorithmic bytes / mean device time)."""
    acc = {}
    for e0, e1, kind, shape, nbytes in quant_events:
        key = (kind, tuple(shape))
        t, b, n = acc.get(key, (0.0, 0.0, 0))
        acc[key] = (t + e0.elapsed_time(e1), b + nbytes, n + 1)
    return [{"kernel": k, "shape": list(shp), "launches": n, "us": round(1e3 * t / n, 2),
             "gbs": round(b / (t * 1e-3) / 1e9, 1)} for (k, shp), (t, b, n) in sorted(acc.items())]


L2_BYTES = 126 * 2 ** 20  # B200 L2


def quant_stream_us(dev, kind, shape):
    """Device time per launch of one quantizer kind and shape, launched back to back
    through the C ABI as in the step (programmatic dependent launch lets each launch's
    prologue overlap the previous one's tail).  Inputs and outputs rotate over enough
    copies to exceed twice the L2, so every launch reads its BF16 input from HBM; the
    event-bracketed in-step time also carries the launch gap that the brackets force."""
    import torch
    import blockwise_fp8_linear_b200 as fb
    L = fb.lib()
    st = torch.cuda.current_stream().cuda_stream
    R, C = shape
    n = max(2, -(-2 * L2_BYTES // (R * C * 2)))
    g = torch.Generator(device=dev).manual_seed(1)
    u8 = lambda r, c: torch.empty(r, c, dtype=torch.uint8, device=dev)
    f32 = lambda r, c: torch.empty(r, c, dtype=torch.float32, device=dev)
    bufs = []
    for _ in range(n):
        x = torch.randn(R, C, device=dev, generator=g).to(torch.bfloat16)
        if kind == "quant_act_dual":
            bufs.append((x, u8(R, C), f32(C // 128, R), u8(C, R), f32(R // 128, C)))
        else:
            bufs.append((x, u8(R, C), f32(R // 128, C // 128)))

    def launch(i):
        b = [t.data_ptr() for t in bufs[i]]
        if kind == "quant_act_dual":
            rc = L.fp8_quant_act_dual(b[0], R, C, b[1], b[2], b[3], b[4], st)
        else:
            rc = L.fp8_quant_weight(b[0], R, C, b[1], b[2], None, st)
        if rc:
            raise fb.Fp8bwError(rc, kind)

    for i in range(n):
        launch(i)
    reps = max(4 * n, 40)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for k in range(reps):
        launch(k % n)
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / reps
    del bufs
    torch.cuda.empty_cache()
    return us


def single_fprop_latency(dev, reps=200):
    """The single-fprop workload (X[128][1024] ~ N(0,1), W[1024][1024] ~ N(0,0.02),
    seed 0) through the C ABI: fp8_quant_act(X), fp8_quant_weight(W) and the FPROP
    GEMM.  Latency-bound, so it is reported in microseconds: device time per layer
    call (events around `reps` calls back to back) and per GEMM alone, plus the host
    time to issue one layer call; then the same layer captured once in a CUDA graph
    and replayed `reps` times (no host work per kernel), with a check that the
    replayed output equals the eager one."""
    import torch
    import blockwise_fp8_linear_b200 as fb
    from blockwise_fp8_linear_b200 import synth
    L = fb.lib()
    T, Din, Dout = 128, 1024, 1024
    t = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
    X = t(synth.normal_bf16(T, Din, 1.0, seed=synth.seed_for(0, 0)))
    W = t(synth.normal_bf16(Dout, Din, 0.02, seed=synth.seed_for(0, 1)))
    qx = torch.empty(T, Din, dtype=torch.uint8, device=dev)
    sx = torch.empty(Din // 128, T, dtype=torch.float32, device=dev)
    qw = torch.empty(Dout, Din, dtype=torch.uint8, device=dev)
    sw = torch.empty(Dout // 128, Din // 128, dtype=torch.float32, device=dev)
    Y = torch.empty(T, Dout, dtype=torch.bfloat16, device=dev)
    st = torch.cuda.current_stream().cuda_stream

    def layer(s=st):
        rc = (L.fp8_quant_act(X.data_ptr(), T, Din, qx.data_ptr(), sx.data_ptr(), s)
              or L.fp8_quant_weight(W.data_ptr(), Dout, Din, qw.data_ptr(), sw.data_ptr(), None, s)
              or L.fp8_gemm_blockwise(0, qx.data_ptr(), sx.data_ptr(), qw.data_ptr(),
                                      sw.data_ptr(), Y.data_ptr(), T, Dout, Din, s))
        if rc:
            raise fb.Fp8bwError(rc, "single fprop")

    def gemm():
        rc = L.fp8_gemm_blockwise(0, qx.data_ptr(), sx.data_ptr(), qw.data_ptr(), sw.data_ptr(),
                                  Y.data_ptr(), T, Dout, Din, st)
        if rc:
            raise fb.Fp8bwError(rc, "single fprop gemm")

    out = {"workload": "single fprop linear: X[128x1024], W[1024x1024], Y = X W^T (bf16)",
           "gflop": round(2 * T * Din * Dout / 1e9, 4)}
    for name, fn in (("layer", layer), ("gemm", gemm)):
        for _ in range(10):
            fn()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        h0 = time.perf_counter()
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        h1 = time.perf_counter()
        torch.cuda.synchronize()
        out[f"{name}_us"] = round(1e3 * e0.elapsed_time(e1) / reps, 2)
        out[f"{name}_host_issue_us"] = round(1e6 * (h1 - h0) / reps, 2)

    # The layer captured once (warmed up on a side stream first, then captured) and
    # replayed: the three launches cost one graph launch on the host.
    layer()
    torch.cuda.synchronize()
    y_eager = Y.clone()
    try:
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            layer(side.cuda_stream)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="relaxed"):
            layer(torch.cuda.current_stream().cuda_stream)
        Y.zero_()
        for _ in range(10):
            g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        h0 = time.perf_counter()
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        h1 = time.perf_counter()
        torch.cuda.synchronize()
        out["layer_graph_us"] = round(1e3 * e0.elapsed_time(e1) / reps, 2)
        out["layer_graph_host_issue_us"] = round(1e6 * (h1 - h0) / reps, 2)
        out["graph_output_identical"] = bool(torch.equal(Y, y_eager))
        del g
    except Exception as exc:  # report, do not hide, a capture the runtime refused
        out["layer_graph_us"] = None
        out["graph_error"] = repr(exc)[:200]
    out["unit"] = "us"
    return out


def run_ours(args):
    import torch
    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    from blockwise_fp8_linear_b200 import build as fbuild
    fbuild.build()
    import blockwise_fp8_linear_b200 as fb

    host = make_inputs(rank)
    work = LayerWork(dev, host, separate=args.separate_quant)
    side = None if args.no_overlap else torch.cuda.Stream(device=dev)
    reducer = None
    if world > 1 and args.dp_grad == "reduce-scatter":
        from blockwise_fp8_linear_b200.dp import DpGradReducer
        reducer = DpGradReducer([(dout, din) for _, din, dout in LINEARS], world, dev)

    # warm-up
    for _ in range(args.warmup):
        work.step(side=side, reducer=reducer)
    torch.cuda.synchronize()
    if fb.fp8bw_last_device_error() != 0:
        raise RuntimeError("a bounded in-kernel wait ran out during warm-up")

    # kernel roofline: the same K steps on one stream, every GEMM launch bracketed by
    # events, so that each launch's time is its own (no overlap with another kernel)
    gemm_events, quant_events = [], []
    barrier(world)
    torch.cuda.synchronize()
    r0 = torch.cuda.Event(enable_timing=True)
    r1 = torch.cuda.Event(enable_timing=True)
    r0.record()
    for _ in range(args.steps):
        work.step(gemm_events, quant_events=quant_events)
    r1.record()
    torch.cuda.synchronize()
    serial_ms = r0.elapsed_time(r1)
    gemm_ms = sum(e0.elapsed_time(e1) for e0, e1, _ in gemm_events)
    gemm_flops = sum(f for _, _, f in gemm_events)
    quant_rows = quant_summary(quant_events)

    # timed region: K steps, device time by CUDA events on the launching stream
    with ClockSampler(dev.index) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        marks = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        t0.record()
        for i in range(args.steps):
            work.step(side=side, reducer=reducer)
            marks[i].record()  # end of step i on the main stream (it waits for the side one)
        t1.record()
        torch.cuda.synchronize()
        barrier(world)
    local_ms = t0.elapsed_time(t1)
    step_ms = [t0.elapsed_time(marks[0])] + [marks[i - 1].elapsed_time(marks[i])
                                             for i in range(1, args.steps)]
    elapsed_ms = max_over_ranks(local_ms, world)
    if fb.fp8bw_last_device_error() != 0:
        raise RuntimeError("a bounded in-kernel wait ran out in the timed region")
    clock_info = clocks.summary()

    ms_per_step = elapsed_ms / args.steps
    value = world * STEP_FLOPS / (ms_per_step * 1e-3) / 1e12
    pct = np.percentile(np.array(step_ms), [10, 50, 90])
    step_percentiles = {"p10": round(float(pct[0]), 4), "p50": round(float(pct[1]), 4),
                        "p90": round(float(pct[2]), 4), "unit": "ms",
                        "of": "per-step device time of the timed steps (rank 0)"}

    # sustained: the same step repeated for a few seconds, deep into the power cap
    sustained = None
    if args.sustain_s > 0:
        n_sus = max(args.steps, int(args.sustain_s * 1e3 / max(ms_per_step, 1e-3)))
        n_sus = int(max_over_ranks(float(n_sus), world))
        with ClockSampler(dev.index) as sclk:
            barrier(world)
            torch.cuda.synchronize()
            s0 = torch.cuda.Event(enable_timing=True)
            s1 = torch.cuda.Event(enable_timing=True)
            s0.record()
            for _ in range(n_sus):
                work.step(side=side, reducer=reducer)
            s1.record()
            torch.cuda.synchronize()
            barrier(world)
        sus_ms = max_over_ranks(s0.elapsed_time(s1), world)
        if fb.fp8bw_last_device_error() != 0:
            raise RuntimeError("a bounded in-kernel wait ran out in the sustained run")
        sustained = {"value": round(world * STEP_FLOPS / (sus_ms / n_sus * 1e-3) / 1e12, 3),
                     "unit": UNIT, "ms_per_step": round(sus_ms / n_sus, 4), "steps": n_sus,
                     "seconds": round(sus_ms / 1e3, 3), "clocks": sclk.summary()}

    # end to end through the public API: pinned host inputs -> device, step,
    # results -> pinned host, all inside the timed region
    e2e = None
    if not args.no_e2e:
        pin_in = [(torch.from_numpy(X.view(np.int16)).pin_memory(),
                   torch.from_numpy(W.view(np.int16)).pin_memory(),
                   torch.from_numpy(dY.view(np.int16)).pin_memory()) for X, W, dY in host]
        pin_out = [(torch.empty(d["Y"].shape, dtype=torch.int16).pin_memory(),
                    torch.empty(d["dX"].shape, dtype=torch.int16).pin_memory(),
                    torch.empty(d["dW"].shape, dtype=torch.int16).pin_memory()) for d in work.lin]

        # Pipelined per linear over three streams: uploads (h2d), compute (the current
        # stream, wgrad on `side`), downloads (d2h).  Events order every buffer's
        # writer after its previous reader: an upload after the previous step's
        # quantizers of that linear, the compute after its upload and after the
        # previous step's download of its outputs, a download after the compute.
        h2d, d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        n_lin = len(work.lin)
        mk = lambda: [torch.cuda.Event() for _ in range(n_lin)]
        ev = {"in_free": mk(), "up": mk(), "done_main": mk(), "done_side": mk(), "out_read": mk()}
        for k in ("in_free", "done_side", "out_read"):
            for e in ev[k]:
                e.record()

        class Hooks:
            def before(self, i):
                main = torch.cuda.current_stream()
                main.wait_event(ev["up"][i])
                main.wait_event(ev["out_read"][i])
                main.wait_event(ev["done_side"][i])

            def inputs_read(self, i):
                ev["in_free"][i].record()

            def after(self, i, main, side_s):
                ev["done_main"][i].record(main)
                ev["done_side"][i].record(side_s)
                d = work.lin[i]
                Y, dX, dW = pin_out[i]
                d2h.wait_event(ev["done_main"][i])
                d2h.wait_event(ev["done_side"][i])
                with torch.cuda.stream(d2h):
                    Y.copy_(d["Y"].view(torch.int16), non_blocking=True)
                    dX.copy_(d["dX"].view(torch.int16), non_blocking=True)
                    dW.copy_(d["dW"].view(torch.int16), non_blocking=True)
                ev["out_read"][i].record(d2h)

        hooks = Hooks()

        def e2e_step():
            for i, (d, (X, W, dY)) in enumerate(zip(work.lin, pin_in)):
                h2d.wait_event(ev["in_free"][i])
                with torch.cuda.stream(h2d):
                    d["X"].view(torch.int16).copy_(X, non_blocking=True)
                    d["W"].view(torch.int16).copy_(W, non_blocking=True)
                    d["dY"].view(torch.int16).copy_(dY, non_blocking=True)
                ev["up"][i].record(h2d)
            work.step(side=side, hooks=hooks)

        e2e_step()
        torch.cuda.synchronize()
        n_e2e = max(3, min(args.steps, 20))
        barrier(world)
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record()
        for _ in range(n_e2e):
            e2e_step()
        torch.cuda.current_stream().wait_stream(d2h)
        a1.record()
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(a0.elapsed_time(a1), world) / n_e2e
        e2e = {"value": round(world * STEP_FLOPS / (e2e_ms * 1e-3) / 1e12, 3), "unit": UNIT,
               "h2d_bytes_per_step": work.h2d_bytes, "d2h_bytes_per_step": work.d2h_bytes,
               "ms_per_step": round(e2e_ms, 4), "steps": n_e2e}

    peaks, peak_src = measured_peaks()
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    hbm_peak = float(peaks["hbm_gbs"])
    achieved = gemm_flops / (gemm_ms * 1e-3) / 1e12
    roofline = {
        "kernel": "fp8_gemm_kernel (fprop/dgrad/wgrad, all 12 GEMMs of the step)",
        "bound": "tensor", "achieved": round(achieved, 2),
        "peak": round(fp8_peak, 1), "unit": "TFLOP/s", "frac": round(achieved / fp8_peak, 4),
        "peak_source": f"{peak_src} cuBLAS bf16 burst x {FP8_OVER_BF16:g} (nominal FP8:BF16)",
        "nominal_peak": NOMINAL_FP8_TFLOPS,
        "frac_of_nominal": round(achieved / NOMINAL_FP8_TFLOPS, 4),
        "target": ">= 0.60 of dense FP8 peak, reported against both the measured peak "
                  "(frac) and the nominal 4.5 PFLOP/s (frac_of_nominal)",
        "traffic": recorded_traffic(),
        "traffic_unit": "bytes per GEMM launch (mean over the step's 12 GEMMs, ncu dram read+write)",
        "gemm_share_of_step": round(gemm_ms / serial_ms, 4),
        "measured_on": "a separate pass of the same steps on one stream (no kernel overlap)",
        "per_gemm": gemm_summary(gemm_events, work),
    }
    quant_roofline = {
        "bound": "hbm", "unit": "GB/s", "peak": hbm_peak,
        "peak_source": f"{peak_src} HBM copy bandwidth",
        "nominal_peak": NOMINAL_HBM_GBS,
        "target": ">= 0.75 of HBM bandwidth, reported against both the measured copy "
                  "bandwidth (frac) and the nominal 8 TB/s (frac_of_nominal)",
        "bytes_per_element": {"quant_act_dual": DUAL_BYTES, "quant_weight": WEIGHT_BYTES},
        "measured_on": "us / gbs / frac: each kind and shape launched back to back through the "
                       "C ABI, inputs and outputs rotating over copies larger than twice the "
                       "L2 (every launch reads HBM); in_step_us: the same launches inside the "
                       "one-stream pass, each bracketed by events (adds the launch gap the "
                       "brackets force)",
        "kernels": quant_kernel_rows(dev, quant_rows, hbm_peak, args.steps),
    }
    single = single_fprop_latency(dev) if not args.no_single else None

    # the same step with power-of-two (E8M0) scales applied by the block-scaled MMA
    # (the MXFP8 form of the recipe), for comparison; not the headline
    variant = None
    if not args.no_variant:
        work8 = LayerWork(dev, host, separate=args.separate_quant, scales="e8m0")
        for _ in range(args.warmup):
            work8.step(side=side)
        torch.cuda.synchronize()
        ev8 = []
        for _ in range(args.steps):
            work8.step(ev8)
        v0 = torch.cuda.Event(enable_timing=True)
        v1 = torch.cuda.Event(enable_timing=True)
        with ClockSampler(dev.index) as vclk:
            barrier(world)
            torch.cuda.synchronize()
            v0.record()
            for _ in range(args.steps):
                work8.step(side=side)
            v1.record()
            torch.cuda.synchronize()
            barrier(world)
        if fb.fp8bw_last_device_error() != 0:
            raise RuntimeError("a bounded in-kernel wait ran out in the E8M0 variant")
        v_ms = max_over_ranks(v0.elapsed_time(v1), world) / args.steps
        g8_ms = sum(e0.elapsed_time(e1) for e0, e1, _ in ev8)
        g8 = sum(f for _, _, f in ev8) / (g8_ms * 1e-3) / 1e12
        variant = {"scales": "e8m0 (power of two, scale blocks applied by tcgen05.mma block_scale)",
                   "value": round(world * STEP_FLOPS / (v_ms * 1e-3) / 1e12, 3), "unit": UNIT,
                   "ms_per_step": round(v_ms, 4), "gemm_tflops": round(g8, 2),
                   "gemm_frac": round(g8 / fp8_peak, 4),
                   "gemm_frac_of_nominal": round(g8 / NOMINAL_FP8_TFLOPS, 4),
                   "gemm_kernel": "fp8_gemm_mx_kernel", "clocks": vclk.summary()}
        del work8

    cpu = None
    if rank == 0 and not args.no_cpu:
        cpu = cpu_baseline(budget_s=args.cpu_budget, host=host)
    sweep = None
    if world == 1 and not args.no_sweep:
        # the micro-batch knee (28-layer step linear work at M = 4096 .. 32768)
        per_m, knee_line = run_sweep(args, emit=False, cpu_budget=min(args.cpu_budget, 5.0))
        sweep = {"knee_tokens": knee_line["knee_tokens"], "rule": knee_line["rule"],
                 "per_m": [{k: r[k] for k in ("tokens", "value", "ms_per_step", "gemm_tflops",
                                              "gemm_share_of_step", "clocks")} for r in per_m],
                 "unit": UNIT, "steps_per_m": args.sweep_steps, "layers": SWEEP_LAYERS,
                 "cpu_baseline": knee_line.get("cpu_baseline")}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3", "data": "synthetic (seeded splitmix64/Box-Muller BF16)",
            "config": config_dict(world, overlap=side is not None,
                                  dp_grad=reducer is not None), "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e, "gpu_launches": work.launches_per_step * args.steps,
            "step_ms_percentiles": step_percentiles,
            "micro_batch_sweep": sweep,
            "clocks": clock_info,
            "pct_of_fp8_peak": round(100 * value / world / fp8_peak, 2),
            "pct_of_nominal_fp8_peak": round(100 * value / world / NOMINAL_FP8_TFLOPS, 2),
            "quant_roofline": quant_roofline,
            "single_fprop": single,
            "sustained": sustained,
            "variant_e8m0": variant,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ----------------------------------------------------- oracle (CPU) timing

def oracle_sample_step(i, host, threads, tokens=TOKENS):
    """One bounded sample of the step on the CPU oracle: linear i % 4, GEMM mode
    (i // 4) % 3, one 128-row tile of the output, with the quantization of exactly
    the groups that tile reads; `tokens` of the host inputs are used.  Returns (GEMM
    flops done, seconds)."""
    import oracle
    li = i % len(LINEARS)
    mode = (i // len(LINEARS)) % 3
    name, din, dout = LINEARS[li]
    X, W, dY = host[li]
    X, dY = X[:tokens], dY[:tokens]
    r0 = 128 * ((i // 12) % (tokens // 128))
    t = time.perf_counter()
    if mode == oracle.FPROP:
        a, sa = oracle.quant_act(np.ascontiguousarray(X[r0:r0 + 128]))
        b, sb, _ = oracle.quant_weight(W)
        M, N, K = 128, dout, din
    elif mode == oracle.DGRAD:
        a, sa = oracle.quant_act(np.ascontiguousarray(dY[r0:r0 + 128]))
        b, sb, _ = oracle.quant_weight(W)
        M, N, K = 128, din, dout
    else:
        # output rows r0..r0+127 of dW (out-features): those columns of dY, all tokens
        a, sa = oracle.quant_act_t(np.ascontiguousarray(dY[:, r0 % dout:(r0 % dout) + 128]))
        b, sb = oracle.quant_act_t(np.ascontiguousarray(X))
        M, N, K = 128, din, tokens
    oracle.gemm(mode, a, sa, b, sb, M, N, K, nthreads=threads)
    return 2 * M * N * K, time.perf_counter() - t


def cpu_model():
    """The host CPU's model name (Linux /proc/cpuinfo), or the platform's processor string."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(budget_s=15.0, host=None, max_steps=None):
    import oracle
    threads = oracle.max_threads()
    if host is None:
        host = make_inputs(0)
    flops = 0
    secs = 0.0
    n = 0
    while secs < budget_s and (max_steps is None or n < max_steps):
        f, s = oracle_sample_step(n, host, threads)
        flops += f
        secs += s
        n += 1
    return {"value": round(flops / secs / 1e12, 6), "unit": UNIT, "cores": threads,
            "cpu_model": cpu_model(), "nproc": os.cpu_count(), "kind": "oracle",
            "sample": f"{n} samples, each one 128-row output tile of one of the 12 GEMMs of the "
                      f"step (rotating linear x mode) plus the oracle quantization of the groups "
                      f"it reads; FP64 GEMM, {threads} OpenMP threads, {secs:.1f} s"}


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    threads = oracle.max_threads()
    host = make_inputs(0)
    for i in range(args.warmup):
        oracle_sample_step(i, host, threads)
    flops = 0
    secs = 0.0
    for i in range(args.steps):
        f, s = oracle_sample_step(args.warmup + i, host, threads)
        flops += f
        secs += s
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(world),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": threads,
                         "cpu_model": cpu_model(), "nproc": os.cpu_count(), "kind": "oracle",
                         "sample": "each step: one 128-row output tile of one of the 12 GEMMs "
                                   "(rotating), with the quantization of the groups it reads"},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


KERNEL_CASES = ("gemm_fprop", "gemm_dgrad", "gemm_wgrad", "gemm_mx_fprop", "gemm_mx_wgrad",
                "quant_dual_e8m0", "quant_act", "quant_act_t",
                "quant_dual", "quant_weight")


def run_kernel_only(args):
    """Launch one kernel of the step (the GEMMs on one linear's shapes, --kernel-linear,
    QKV by default: M=8192, 2048 -> 4096; the quantizers on --quant-shape, by default
    the 8192x12288 gate/up gradient so inputs exceed L2) warmup+steps times back to back
    and print its mean device time.  For profilers."""
    import torch
    import blockwise_fp8_linear_b200 as fb
    from blockwise_fp8_linear_b200 import build as fbuild
    fbuild.build()
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(0)
    T = TOKENS
    _, din, dout = next(x for x in LINEARS if x[0] == args.kernel_linear)
    case = args.kernel_only

    def randn(r, c, std):
        return (torch.randn(r, c, device=dev, generator=g) * std).to(torch.bfloat16)

    if case.startswith("gemm_mx"):
        X, W, dY = randn(T, din, 1.0), randn(dout, din, 0.02), randn(T, dout, 1e-3)
        if case == "gemm_mx_fprop":
            a, sa = fb.fp8_quant_act_e8m0(X)
            b, sb, _ = fb.fp8_quant_weight_e8m0(W)
            launch = lambda: fb.fp8_gemm_blockwise_e8m0(fb.FPROP, a, sa, b, sb, T, dout, din)
        else:
            a, sa = fb.fp8_quant_act_t_e8m0(dY)
            b, sb = fb.fp8_quant_act_t_e8m0(X)
            launch = lambda: fb.fp8_gemm_blockwise_e8m0(fb.WGRAD, a, sa, b, sb, dout, din, T)
        work = ("TFLOP/s", 2 * T * din * dout / 1e12)
    elif case.startswith("gemm"):
        X, W, dY = randn(T, din, 1.0), randn(dout, din, 0.02), randn(T, dout, 1e-3)
        qw, sw, _ = fb.fp8_quant_weight(W)
        if case == "gemm_fprop":
            a, sa = fb.fp8_quant_act(X)
            launch = lambda: fb.fp8_gemm_blockwise(fb.FPROP, a, sa, qw, sw, T, dout, din)
            flops = 2 * T * din * dout
        elif case == "gemm_dgrad":
            a, sa = fb.fp8_quant_act(dY)
            launch = lambda: fb.fp8_gemm_blockwise(fb.DGRAD, a, sa, qw, sw, T, din, dout)
            flops = 2 * T * din * dout
        else:
            a, sa = fb.fp8_quant_act_t(dY)
            b, sb = fb.fp8_quant_act_t(X)
            launch = lambda: fb.fp8_gemm_blockwise(fb.WGRAD, a, sa, b, sb, dout, din, T)
            flops = 2 * T * din * dout
        work = ("TFLOP/s", flops / 1e12)
    else:
        R, C = (int(v) for v in args.quant_shape.split("x"))
        X = randn(R, C, 1.0)
        # outputs allocated once and the C ABI called directly, so that host work per
        # launch stays well below the kernel time even for the small shapes
        L = fb.lib()
        st = fb._stream(None)
        u8 = lambda r, c: torch.empty(r, c, dtype=torch.uint8, device=dev)
        f32 = lambda r, c: torch.empty(r, c, dtype=torch.float32, device=dev)
        q, qt = u8(R, C), u8(C, R)
        if case == "quant_dual_e8m0":
            s, sT = u8(R // 128, (C // 128) * 512), u8(C // 128, (R // 128) * 512)
        else:
            s, sT = f32(C // 128, R), f32(R // 128, C)
        p = lambda x: x.data_ptr()

        def run(fn, *a):
            rc = fn(*a)
            if rc:
                raise fb.Fp8bwError(rc, case)
        if case == "quant_act":
            launch = lambda: run(L.fp8_quant_act, p(X), R, C, p(q), p(s), st)
        elif case == "quant_act_t":
            launch = lambda: run(L.fp8_quant_act_t, p(X), R, C, p(qt), p(sT), st)
        elif case == "quant_dual":
            launch = lambda: run(L.fp8_quant_act_dual, p(X), R, C, p(q), p(s), p(qt), p(sT), st)
        elif case == "quant_dual_e8m0":
            launch = lambda: run(L.fp8_quant_act_dual_e8m0, p(X), R, C, p(q), p(s), p(qt), p(sT), st)
        else:
            sw = f32(R // 128, C // 128)
            launch = lambda: run(L.fp8_quant_weight, p(X), R, C, p(q), p(sw), None, st)
        per_elem = (4 + 8 / 128) if case.startswith("quant_dual") else (3 + 4 / 128)
        work = ("GB/s", R * C * per_elem / 1e9)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        launch()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        launch()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    print(json.dumps({"kernel_only": case, "linear": args.kernel_linear,
                      "quant_shape": args.quant_shape, "ms": round(ms, 5),
                      work[0]: round(work[1] / (ms * 1e-3), 2)}), flush=True)


# ------------------------------------------------- micro-batch knee sweep

SWEEP_TOKENS = (4096, 8192, 16384, 32768)   # micro-batch 1, 2, 4, 8 x sequence 4096
SWEEP_LAYERS = 28


def run_sweep(args, emit=True, cpu_budget=None):
    """Knee sweep of one 28-layer step's linear work: per layer the four linears of the
    block in fprop + dgrad + wgrad with all quantizers (24 launches), each layer with its
    own weights, at M = 4096 ... 32768 tokens.  Prints one JSON line per M and a
    summary line naming the knee: the smallest M whose doubling gains < 5% of T_lin.
    Inputs come from torch's seeded device generator (X ~ N(0,1) with 1% outlier
    channels x20, W ~ N(0,0.02), dY ~ N(0,1e-3)); activations are shared by the
    layers, weights are distinct per layer (2.8 GB of BF16).  With emit=False nothing is
    printed and the per-M lines and the knee line are returned (the default bench run
    carries them in its own line)."""
    import torch
    import blockwise_fp8_linear_b200 as fb
    from blockwise_fp8_linear_b200 import build as fbuild
    fbuild.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    L = fb.lib()
    g = torch.Generator(device=dev).manual_seed(4)

    def randn(r, c, std, outliers=False):
        x = torch.randn(r, c, device=dev, generator=g) * std
        if outliers:
            cols = torch.randperm(c, device=dev, generator=g)[: c // 100]
            x[:, cols] *= 20.0
        return x.to(torch.bfloat16)

    weights = [[randn(dout, din, 0.02) for _, din, dout in LINEARS] for _ in range(SWEEP_LAYERS)]
    qw = [torch.empty(dout, din, dtype=torch.uint8, device=dev) for _, din, dout in LINEARS]
    sw = [torch.empty(dout // 128, din // 128, dtype=torch.float32, device=dev) for _, din, dout in LINEARS]
    results = []
    for T in SWEEP_TOKENS:
        bufs = []
        for _, din, dout in LINEARS:
            u8 = lambda r, c: torch.empty(r, c, dtype=torch.uint8, device=dev)
            f32 = lambda r, c: torch.empty(r, c, dtype=torch.float32, device=dev)
            bufs.append({
                "X": randn(T, din, 1.0, outliers=True), "dY": randn(T, dout, 1e-3),
                "qx": u8(T, din), "sx": f32(din // 128, T), "qxt": u8(din, T), "sxt": f32(T // 128, din),
                "qdy": u8(T, dout), "sdy": f32(dout // 128, T), "qdyt": u8(dout, T), "sdyt": f32(T // 128, dout),
                "Y": torch.empty(T, dout, dtype=torch.bfloat16, device=dev),
                "dX": torch.empty(T, din, dtype=torch.bfloat16, device=dev),
                "dW": torch.empty(dout, din, dtype=torch.bfloat16, device=dev)})
        st = fb._stream(None)

        def chk(rc, what):
            if rc:
                raise fb.Fp8bwError(rc, what)

        def step(gemm_events=None):
            for layer in range(SWEEP_LAYERS):
                for i, (_, din, dout) in enumerate(LINEARS):
                    b, W = bufs[i], weights[layer][i]
                    p = lambda k: b[k].data_ptr()
                    chk(L.fp8_quant_act_dual(p("X"), T, din, p("qx"), p("sx"), p("qxt"), p("sxt"), st), "qd")
                    chk(L.fp8_quant_weight(W.data_ptr(), dout, din, qw[i].data_ptr(), sw[i].data_ptr(), None, st), "qw")
                    chk(L.fp8_quant_act_dual(p("dY"), T, dout, p("qdy"), p("sdy"), p("qdyt"), p("sdyt"), st), "qd")
                    for mode, a, sa, bb, sb, out, M, N, K in (
                            (fb.FPROP, p("qx"), p("sx"), qw[i].data_ptr(), sw[i].data_ptr(), p("Y"), T, dout, din),
                            (fb.DGRAD, p("qdy"), p("sdy"), qw[i].data_ptr(), sw[i].data_ptr(), p("dX"), T, din, dout),
                            (fb.WGRAD, p("qdyt"), p("sdyt"), p("qxt"), p("sxt"), p("dW"), dout, din, T)):
                        if gemm_events is not None:
                            e0 = torch.cuda.Event(enable_timing=True)
                            e0.record()
                        chk(L.fp8_gemm_blockwise(mode, a, sa, bb, sb, out, M, N, K, st), "gemm")
                        if gemm_events is not None:
                            e1 = torch.cuda.Event(enable_timing=True)
                            e1.record()
                            gemm_events.append((e0, e1))

        for _ in range(max(3, args.warmup)):
            step()
        torch.cuda.synchronize()
        if fb.fp8bw_last_device_error() != 0:
            raise RuntimeError("a bounded in-kernel wait ran out during the sweep warm-up")
        ev = []
        with ClockSampler(dev.index) as clocks:
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            t0.record()
            for _ in range(args.sweep_steps):
                step(ev)
            t1.record()
            torch.cuda.synchronize()
        if fb.fp8bw_last_device_error() != 0:
            raise RuntimeError("a bounded in-kernel wait ran out in the sweep")
        ms = t0.elapsed_time(t1) / args.sweep_steps
        gemm_ms = sum(a.elapsed_time(b) for a, b in ev) / args.sweep_steps
        flops = SWEEP_LAYERS * sum(3 * 2 * T * din * dout for _, din, dout in LINEARS)
        line = {"sweep": "micro-batch knee, 28-layer step linear work", "tokens": T,
                "layers": SWEEP_LAYERS, "value": round(flops / (ms * 1e-3) / 1e12, 2),
                "unit": UNIT, "ms_per_step": round(ms, 3), "step_tflop": round(flops / 1e12, 3),
                "gemm_tflops": round(flops / (gemm_ms * 1e-3) / 1e12, 2),
                "gemm_share_of_step": round(gemm_ms / ms, 4), "steps": args.sweep_steps,
                "launches_per_step": SWEEP_LAYERS * 24, "clocks": clocks.summary(),
                "data": "synthetic (torch seeded device generator)"}
        results.append(line)
        if emit:
            print(json.dumps(line), flush=True)
        del bufs
        torch.cuda.empty_cache()
    knee = None
    for a, b in zip(results, results[1:]):
        if b["value"] < 1.05 * a["value"]:
            knee = a["tokens"]
            break
    line = {"sweep": "knee", "knee_tokens": knee,
            "rule": "smallest M whose doubling gains < 5% of T_lin",
            "values": {r["tokens"]: r["value"] for r in results}}
    budget = args.cpu_budget if cpu_budget is None else cpu_budget
    if not args.no_cpu and budget > 0:
        # The CPU oracle on one layer at M = 4096 (a bounded sample of 128-row output
        # tiles of its 12 GEMMs, with the quantization each tile reads), extrapolated
        # linearly in FLOPs to each M's 28-layer step.
        import oracle
        threads = oracle.max_threads()
        host = make_inputs(0)
        flops, secs, n = 0, 0.0, 0
        while secs < budget:
            f, t = oracle_sample_step(n, host, threads, tokens=SWEEP_TOKENS[0])
            flops += f
            secs += t
            n += 1
        rate = flops / secs
        line["cpu_baseline"] = {
            "value": round(rate / 1e12, 6), "unit": UNIT, "kind": "oracle", "cores": threads,
            "cpu_model": cpu_model(), "nproc": os.cpu_count(),
            "sample": f"one layer at M={SWEEP_TOKENS[0]}: {n} samples, each one 128-row output "
                      f"tile of one of the 12 GEMMs plus the quantization it reads, {secs:.1f} s",
            "extrapolated_step_s": {
                r["tokens"]: round(SWEEP_LAYERS * sum(3 * 2 * r["tokens"] * din * dout
                                                      for _, din, dout in LINEARS) / rate, 1)
                for r in results},
            "extrapolation": "linear in FLOPs (stated as such; not measured at full size)"}
    if emit:
        print(json.dumps(line), flush=True)
    return results, line


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work")
    ap.add_argument("--separate-quant", action="store_true",
                    help="quantize X and dY with separate row-wise and token-wise passes "
                         "instead of the fused dual-output quantizer")
    ap.add_argument("--dp-grad", choices=["none", "reduce-scatter"], default="none",
                    help="with N > 1: none = independent replicas; reduce-scatter = sum each "
                         "linear's dW over the ranks (NCCL), overlapped with the next linear")
    ap.add_argument("--no-variant", action="store_true",
                    help="skip the power-of-two (E8M0) scale variant of the step")
    ap.add_argument("--sustain-s", type=float, default=2.5,
                    help="seconds of the same step repeated after the timed region, reported "
                         "as 'sustained' (0 = skip)")
    ap.add_argument("--no-single", action="store_true",
                    help="skip the single-fprop latency measurement")
    ap.add_argument("--no-overlap", action="store_true",
                    help="run every kernel on one stream (no dgrad/wgrad overlap)")
    ap.add_argument("--kernel-only", choices=KERNEL_CASES, default=None,
                    help="launch one kernel repeatedly (for profilers); no JSON metric line")
    ap.add_argument("--kernel-linear", choices=[n for n, _, _ in LINEARS], default="qkv",
                    help="with --kernel-only gemm_*: the linear whose GEMM shapes to launch")
    ap.add_argument("--quant-shape", default="8192x12288",
                    help="with --kernel-only quant_*: ROWSxCOLS of the BF16 input")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the micro-batch knee sweep that the default run carries")
    ap.add_argument("--sweep", action="store_true",
                    help="micro-batch knee sweep (28 layers, M = 4096..32768); one JSON line per M")
    ap.add_argument("--sweep-steps", type=int, default=3)
    args = ap.parse_args()
    if args.sweep:
        run_sweep(args)
        return
    if args.kernel_only:
        run_kernel_only(args)
        return
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
