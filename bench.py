#!/usr/bin/env python
"""Benchmark of the GPTQ layer solver on B200: Gparam/s and Hessian TFLOP/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload layer-1024x4096] [--no-cpu-baseline] [--no-e2e]

One step = one pass of the whole path over one layer: H = 2.X.X^T from the
calibration activations, preparation (damping, act-order, the Cholesky factor
U) and quantization (sweep, lazy trailing updates, packing), inputs resident in
HBM.  Each step is timed with CUDA events on the launching stream; L2 is
flushed (a 256 MiB write) between steps, outside the timed events.

With N > 1 (torchrun, one process per GPU) every rank quantizes its own,
independently seeded layer: layers are independent problems, so there is no
data-path collective and scaling is weak; the process group only carries the
barrier and the max-over-ranks of the timings.

The default line also carries the two decoder blocks (Llama-2-70B- and 7B-shaped:
seconds per block, per-input stage times, Hessian and kernel roofline fractions),
per-kernel roofline entries from the library's timing trace, and the tf32 and FP32
peaks measured in the same run.

`--impl reference` times the fp64 CPU oracle on rank 0 (the other ranks exit),
each step the whole layer with all of its tokens, nothing extrapolated.
"""
from __future__ import annotations

import argparse
import dataclasses
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

import synthetic as S  # noqa: E402

METRIC = "GPTQ layer quantize: weights/sec (Gparam/s) + Hessian TFLOP/s, % roofline, 1 B200"
UNIT = "Gparam/s"
DEFAULT_WORKLOAD = "layer-1024x4096"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------------- #
# helpers
# --------------------------------------------------------------------------- #
def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def rank_layer(layer: "S.Layer", rank: int) -> "S.Layer":
    """Each rank quantizes its own, independently seeded layer of the same shape."""
    import dataclasses
    return dataclasses.replace(layer, w=dataclasses.replace(layer.w, seed=layer.w.seed + rank),
                               x=dataclasses.replace(layer.x, seed=layer.x.seed + rank))


def max_over_ranks(ms: float, world: int, device=None) -> float:
    """The slowest rank's time (all ranks take this collective in the same order)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gparams_per_s(world: int, out: int, n: int, ms: float) -> float:
    """Whole-job throughput: every rank quantized one out x n layer in (at most) ms."""
    return world * out * n / (ms * 1e-3) / 1e9


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["_source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["_source"] = "fallback"
    return d


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons sampled during the timed
    region: NVML polled every 10 ms (reads only), else nvidia-smi every 200 ms."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.samples = []
        self.t = None
        self.stop_flag = threading.Event()
        self.nvml = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[self.gpu]) if vis and vis.split(",")[self.gpu].isdigit() else self.gpu
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_sm = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.nvml = pynvml
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
            return
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _poll(self):
        nv = self.nvml
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self.stop_flag.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                rs = get_reasons(self.h)
                self.samples.append((float(sm), pw, int(rs)))
            except Exception:
                pass
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.nvml is not None:
            self.stop_flag.set()
            self.t.join(timeout=5)
            sm = [x[0] for x in self.samples]
            reasons = sorted({nm for _, _, r in self.samples for nm, bit in self.REASONS.items() if r & bit})
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
            return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": float(self.max_sm),
                    "power_w_max": max((x[1] for x in self.samples), default=None), "samples": len(sm),
                    "source": "nvml, 10 ms", "reasons": reasons}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.t is not None:
            self.t.join(timeout=5)
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None, "samples": len(sm), "source": "nvidia-smi, 200 ms",
                "reasons": sorted(reasons)}


# --------------------------------------------------------------------------- #
# CPU oracle leg (bounded sample)
# --------------------------------------------------------------------------- #
def oracle_sample(layer: S.Layer, st: S.QuantSettings, tokens: int):
    """Run the oracle on the full layer with the first `tokens` calibration tokens.

    Returns (seconds extrapolated to the full token count, sample description).
    The Hessian's cost is linear in tokens; preparation and sweep do not depend on them.
    """
    from oracle import gptq_oracle as O  # the oracle is only ever run here, for the CPU baseline
    W = S.make_w(layer.w)
    x = S.make_x(layer.x, 0, tokens)
    t0 = time.perf_counter()
    H = O.hessian(x)
    t1 = time.perf_counter()
    prep = O.prepare(H, st.damp_percent, st.desc_act)
    sw, codes = O.quantize_layer(W, prep, st.bits, st.group_size, st.sym, st.block)
    O.pack(codes, st.bits)
    O.g_idx(prep.perm, st.group_size)
    t2 = time.perf_counter()
    scale = layer.x.tokens / tokens
    est = (t1 - t0) * scale + (t2 - t1)
    if tokens == layer.x.tokens:
        desc = (f"full layer {layer.w.out}x{layer.w.n} with all {tokens} tokens, every stage measured "
                f"(nothing extrapolated): {t2 - t0:.1f} s")
    else:
        desc = (f"full layer {layer.w.out}x{layer.w.n} (prepare, sweep, pack run in full); Hessian on the first "
                f"{tokens} of {layer.x.tokens} tokens, its time extrapolated x{scale:g}; measured {t2 - t0:.1f} s")
    return est, desc


def oracle_single_thread(workload: str = "layer-256x512"):
    """The oracle on the small layer, whole (all its tokens), with one BLAS thread.

    Returns {"value", "unit", "cores": 1, "seconds", "workload"}.
    """
    from threadpoolctl import threadpool_limits
    wl = S.workloads()[workload]
    layer, st = wl.layers[0], wl.settings[0]
    with threadpool_limits(limits=1):
        est, _ = oracle_sample(layer, st, layer.x.tokens)
    return {"value": layer.w.out * layer.w.n / est / 1e9, "unit": UNIT, "cores": 1, "seconds": est,
            "workload": workload}


# --------------------------------------------------------------------------- #
# reference arm: the oracle
# --------------------------------------------------------------------------- #
def run_reference(args):
    rank, _, world = env_rank()
    if rank != 0:
        return 0
    wl = S.workloads()[args.workload]
    layer, st = wl.layers[0], wl.settings[0]
    # every step is the whole layer with all of its calibration tokens: nothing is
    # extrapolated, so the line's ms_per_step is the oracle's measured time
    tokens = layer.x.tokens
    times = []
    desc = ""
    for i in range(args.warmup + args.steps):
        est, desc = oracle_sample(layer, st, tokens)
        if i >= args.warmup:
            times.append(est)
    t = statistics.mean(times)
    value = layer.w.out * layer.w.n / t / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(args.workload, layer, st),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": host_cores(), "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one hessian_pair_kernel launch
# on layer-1024x4096, from one ncu capture of this bench command, valid while the kernel's
# sources are the ones that were captured (their SHA-256 below); otherwise the traffic is null.
HESSIAN_TRAFFIC = {"n": 4096, "tokens": 65536, "bytes": 1008786688 + 26257920,
                   "sha256": {"post_weight_quantization_15_b200/csrc/hessian.cu": "4ea0a4d9c5f6d896",
                              "post_weight_quantization_15_b200/csrc/tc_common.cuh": "397409833b5bb824"}}


def hessian_traffic(n: int, tokens: int):
    import hashlib
    if n != HESSIAN_TRAFFIC["n"] or tokens != HESSIAN_TRAFFIC["tokens"]:
        return None
    root = os.path.dirname(os.path.abspath(__file__))
    for rel, digest in HESSIAN_TRAFFIC["sha256"].items():
        try:
            with open(os.path.join(root, rel), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest()[:16] != digest:
                    return None
        except OSError:
            return None
    return HESSIAN_TRAFFIC["bytes"]


def measure_peaks(G, torch, dev):
    """Denominators MEASURED_PEAKS.json does not hold: the dense tf32 tensor-core peak
    (torch.matmul on fp32 with TF32 allowed, 8192^3, best of 10 — the method of the
    measured bf16 peak) and the FP32 CUDA-core peak (the library's FMA probe, best of 5)."""
    out = {}
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = True
    try:
        a = torch.randn((8192, 8192), device=dev)
        b = torch.randn((8192, 8192), device=dev)
        best = float("inf")
        for _ in range(12):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch.matmul(a, b)
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        out["tf32_tflops"] = 2.0 * 8192 ** 3 / (best * 1e-3) / 1e12
        del a, b
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev
    blocks, iters = 148 * 8, 4096
    buf = torch.empty(blocks * 256, dtype=torch.float32, device=dev)
    best = float("inf")
    flop = 0.0
    for _ in range(6):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        flop = G.gptq.probe_fp32_peak(blocks, iters, buf)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    out["fp32_tflops"] = flop / (best * 1e-3) / 1e12
    out["how"] = ("tf32: torch.matmul fp32 8192^3 with TF32 allowed, best of 12; fp32: the library's FMA probe "
                  f"({blocks} x 256 threads, 8 chains), best of 6; CUDA events")
    return out


def kernel_rooflines(trace, peaks, measured, prepare_ms=None, n=None):
    """Per-kernel roofline entries from a traced pass (device time on each launch's stream)."""
    hbm = float(peaks["hbm_gbs"])
    tf32 = measured.get("tf32_tflops")
    fp32 = measured.get("fp32_tflops")
    bf16 = float(peaks["bf16_tflops"])
    res = {}
    for name, r in trace.items():
        if r["ms"] <= 0:
            continue
        rate = r["work"] / (r["ms"] * 1e-3)
        e = {"launches": r["launches"], "ms_total": r["ms"], "ms_per_launch": r["ms"] / r["launches"]}
        if name == "hessian_tc":
            e.update(bound="tensor", unit="TFLOP/s", achieved=rate / 1e12, peak=bf16, frac=rate / 1e12 / bf16,
                     peak_source=f"{peaks['_source']} bf16 burst", work="n(n+1)N flop")
        elif name in ("trailing_update", "prepare_gemm3") and tf32:
            e.update(bound="tensor", unit="TFLOP/s", achieved=3 * rate / 1e12, peak=tf32, frac=3 * rate / 1e12 / tf32,
                     useful_tflops=rate / 1e12, frac_useful=rate / 1e12 / tf32, peak_source="measured tf32 (in this run)",
                     work="3 x 2MNK flop (3xTF32: three tensor passes per product)")
        elif name == "potrf_inv" and fp32:
            e.update(bound="alu", unit="TFLOP/s", achieved=rate / 1e12, peak=fp32, frac=rate / 1e12 / fp32,
                     peak_source="measured fp32 FMA probe (in this run)",
                     work="per panel: the previous panel's two 128-deep products + Cholesky + inverse of the block")
        elif r["unit"] == "byte":
            e.update(bound="hbm", unit="GB/s", achieved=rate / 1e9, peak=hbm, frac=rate / 1e9 / hbm,
                     peak_source=f"{peaks['_source']} HBM copy", work="algorithmic bytes")
        res[name] = e
    if prepare_ms and n and tf32:
        useful = 2.0 / 3.0 * float(n) ** 3 / (prepare_ms * 1e-3) / 1e12
        res["prepare (stage)"] = {"bound": "tensor", "unit": "TFLOP/s", "achieved": 3 * useful, "peak": tf32,
                                  "frac": 3 * useful / tf32, "useful_tflops": useful, "frac_useful": useful / tf32,
                                  "ms": prepare_ms, "peak_source": "measured tf32 (in this run)",
                                  "work": "(2/3) n^3 flop (Cholesky n^3/3 + triangular inverse n^3/3), x3 for 3xTF32"}
    return res


# Decode shapes for the consumer of the stored format (out, in): the 70B block's gate/up
# and down, the 7B block's gate/up, 4-bit g128 with an act-order g_idx.
DECODE_SHAPES = ((28672, 8192), (8192, 28672), (11008, 4096))


def time_qmatvec(G, torch, dev, peaks, flush, iters=20):
    """gptq_qmatvec at decode shapes (1 and 16 activation rows): device time per call (CUDA
    events on this stream, L2 flushed before every call) against the HBM roofline on the
    bytes the call must move (packed weights, scales and zeros, g_idx, X in, Y out)."""
    res = []
    stream = torch.cuda.current_stream()
    for out, n in DECODE_SHAPES:
        gen = torch.Generator(device=dev)
        gen.manual_seed(out + n)
        G_ = n // 128
        q = G.QuantizedLayer(
            qweight=torch.randint(-2 ** 31, 2 ** 31 - 1, (n * 4 // 32, out), generator=gen, device=dev,
                                  dtype=torch.int64).to(torch.int32),
            scales=(torch.rand((G_, out), generator=gen, device=dev) * 0.01 + 1e-4).half(),
            zeros=torch.randint(0, 16, (G_, out), generator=gen, device=dev).half(),
            g_idx=(torch.randperm(n, generator=gen, device=dev) // 128).to(torch.int32),
            codes=None, err_sq=None, bits=4, group_size=128, sym=False)
        st = G.new_status(dev)
        qg, xperm = G.reorder_groups(q, st)       # once per layer: the columns sorted by group
        G.raise_on_status(st, "reorder")
        for layout, lay, xp in (("act-order, as stored", q, None), ("act-order, reordered once", qg, xperm)):
            for M in (1, 16):
                X = torch.randn((M, n), generator=gen, device=dev).half()
                Y = torch.empty((M, out), dtype=torch.float32, device=dev)
                ws = G.workspace(G.lib().gptq_qmatvec_workspace_size(M, n, out), dev)
                times = []
                for i in range(iters + 3):
                    flush.fill_(1.0)
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    G.qmatvec(lay, X, st, ws=ws, out=Y, xperm=xp)
                    e1.record(stream)
                    torch.cuda.synchronize()
                    if i >= 3:
                        times.append(e0.elapsed_time(e1))
                G.raise_on_status(st, "qmatvec bench")
                ms = statistics.median(times)
                nbytes = out * n * 4 / 8 + 4.0 * G_ * out + 4.0 * n + 2.0 * M * n + 4.0 * M * out + \
                    (4.0 * n if xp is not None else 0.0)
                gbs = nbytes / (ms * 1e-3) / 1e9
                res.append({"out": out, "in": n, "tokens": M, "bits": 4, "group_size": 128, "layout": layout,
                            "us_per_call": ms * 1e3, "bytes": nbytes, "achieved_gbs": gbs,
                            "frac": gbs / float(peaks["hbm_gbs"]),
                            "flop": 2.0 * M * out * n, "tflops": 2.0 * M * out * n / (ms * 1e-3) / 1e12})
    return {"kernel": "qmatvec (+ its k-split reduction)", "bound": "hbm", "peak": float(peaks["hbm_gbs"]),
            "unit": "GB/s", "peak_source": f"{peaks['_source']} HBM copy",
            "timing": f"CUDA events around each call, L2 flushed before each, median of {iters}",
            "shapes": res}


def time_pipeline(G, torch, dev, blocks=2, warmup=1):
    """The sequential pipeline (pipeline.quantize_mlp_blocks) over the MLP halves of
    Llama-2-7B-shaped blocks: d 4096, d_ff 11008, 65,536 tokens, 4-bit symmetric g128
    act-order; inputs drawn on the device.  Device time per block and per stage."""
    from post_weight_quantization_15_b200 import pipeline as PL
    wl = S.workloads()["llama2-7b-block"]
    st = wl.settings[0]
    by = {l.name: l for l in wl.layers}
    X0 = S.make_x_device(by["gate"].x, dev)
    X0 = X0.contiguous() if X0.stride(0) != X0.shape[1] else X0
    weights = []
    for b in range(blocks):
        weights.append(tuple(S.make_w_device(dataclasses.replace(by[nm].w, stream=by[nm].w.stream + 1000 * b), dev)
                             for nm in ("gate", "up", "down")))
    # whole passes as warm-up, three at least: the library captures its stages as CUDA
    # graphs at the second call with the same arguments, and the caching allocator may
    # hand a pass the addresses of the pass before the last one
    for _ in range(max(3, warmup)):
        PL.quantize_mlp_blocks(X0, weights, st.bits, st.group_size, st.sym, st.desc_act, st.damp_percent)
    res, _ = PL.quantize_mlp_blocks(X0, weights, st.bits, st.group_size, st.sym, st.desc_act, st.damp_percent)
    per = [r.ms for r in res]
    ms = statistics.mean(p["block"] for p in per)
    n_w = sum(int(w.numel()) for w in weights[0])
    return {"workload": "llama2-7b MLP blocks (gate, up, down), 65,536 tokens, each block calibrated on the "
                        "previous quantized block's output", "blocks": blocks,
            "ms_per_block": ms, "gparam_per_s": n_w / (ms * 1e-3) / 1e9, "per_block_stages_ms": per,
            "timing": "CUDA events on the calling stream around each stage"}


def config_dict(name, layer, st):
    return {"workload": name, "out": layer.w.out, "in": layer.w.n, "tokens": layer.x.tokens,
            "w_dtype": layer.w.dtype, "bits": st.bits, "group_size": st.group_size, "sym": st.sym,
            "desc_act": st.desc_act, "damp_percent": st.damp_percent, "block": st.block,
            "x": f"bf16 outlier/low-rank synthetic, rank {layer.x.rank}, {layer.x.outlier_frac:g} outliers "
                 f"x{layer.x.outlier_mult:g}",
            "l2": "flushed between steps (256 MiB write outside the per-step events)"}


# --------------------------------------------------------------------------- #
# our arm
# --------------------------------------------------------------------------- #
def run_ours(args):
    import torch
    import torch.distributed as dist

    import post_weight_quantization_15_b200 as G

    rank, local_rank, world = env_rank()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    wl = S.workloads()[args.workload]
    layer0, st = wl.layers[0], wl.settings[0]
    layer = rank_layer(layer0, rank)      # independent problem per rank
    out, n, N = layer.w.out, layer.w.n, layer.x.tokens

    W_np = S.make_w(layer.w)
    X_np = S.make_x(layer.x)
    W_host = torch.from_numpy(W_np).pin_memory()
    X_host = torch.from_numpy(X_np.view(np.int16)).pin_memory()
    W = W_host.to(dev)
    X = X_host.to(dev).view(torch.bfloat16)

    stream = torch.cuda.current_stream()
    status = G.new_status(dev)
    H = torch.empty((n, n), dtype=torch.float32, device=dev)
    hdiag = torch.empty(n, dtype=torch.float64, device=dev) if st.desc_act else None
    prep_ws = G.workspace(G.lib().gptq_prepare_workspace_size(n), dev)
    q_ws = G.workspace(G.quantize_workspace_size(out, n, st.block), dev)
    prep = G.Prepared(U=torch.empty((n, n), dtype=torch.float32, device=dev),
                      perm=torch.empty(n, dtype=torch.int32, device=dev),
                      dead=torch.empty(n, dtype=torch.uint8, device=dev), status=status, desc_act=st.desc_act)
    qout = G.alloc_quantized(out, n, st.bits, st.group_size, st.sym, dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]

    def step(e=None):
        if e is not None:
            e[0].record(stream)
        # H (and the act-order key) accumulate: clearing them is part of the step
        G.status_reset(status)
        H.zero_()
        if hdiag is not None:
            hdiag.zero_()
        if e is not None:
            e[4].record(stream)
        G.hessian_accumulate(H, X, hdiag, status)
        if e is not None:
            e[1].record(stream)
        G.prepare(H, st.damp_percent, st.desc_act, hdiag, status, ws=prep_ws, out=prep)
        if e is not None:
            e[2].record(stream)
        G.quantize_layer(W, prep, st.bits, st.group_size, st.sym, st.block, ws=q_ws, out=qout)
        if e is not None:
            e[3].record(stream)

    for _ in range(args.warmup):
        step()
        flush.fill_(1.0)
    torch.cuda.synchronize()
    G.raise_on_status(status, "warm-up")

    clocks = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    launches0 = G.kernel_launches()
    t_wall0 = time.perf_counter()
    for i in range(args.steps):
        step(ev[i])
        flush.fill_(1.0)
    torch.cuda.synchronize()
    t_wall1 = time.perf_counter()
    launches = G.kernel_launches() - launches0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    G.raise_on_status(status, "timed steps")

    # A second pass of the same steps with the library's timing trace on: events around
    # every kernel on the stream it runs on, for the per-kernel roofline entries (kept out
    # of the headline timing above, whose events bracket whole steps on this stream).
    G.trace_read()
    G.trace_enable(True)
    for i in range(args.steps):
        step()
        flush.fill_(1.0)
    torch.cuda.synchronize()
    G.trace_enable(False)
    trace = G.trace_read()
    G.raise_on_status(status, "traced steps")

    step_ms = [e[0].elapsed_time(e[3]) for e in ev]
    hess_ms = [e[4].elapsed_time(e[1]) for e in ev]        # the Hessian launch(es) alone
    clear_ms = [e[0].elapsed_time(e[4]) for e in ev]
    prep_ms = [e[1].elapsed_time(e[2]) for e in ev]
    quant_ms = [e[2].elapsed_time(e[3]) for e in ev]
    ms = max_over_ranks(statistics.mean(step_ms), world, dev)
    value = job_gparams_per_s(world, out, n, ms)
    # the same metric without the Hessian: prepare + ingest + sweep + trailing + pack (every rank
    # takes this collective, in the same order)
    solver_ms = max_over_ranks(statistics.mean(p + q for p, q in zip(prep_ms, quant_ms)), world, dev)
    solver_value = job_gparams_per_s(world, out, n, solver_ms)

    # dominant kernel: the Hessian tile product (one launch per step)
    peaks = load_peaks()
    h_flops = float(n) * (n + 1) * N
    h_s = statistics.mean(hess_ms) * 1e-3
    achieved = h_flops / h_s / 1e12
    peak = float(peaks["bf16_tflops"])
    roofline = {"kernel": "hessian (K1)", "bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": hessian_traffic(n, N),
                "traffic_unit": "DRAM bytes read + written per launch (ncu)",
                "peak_source": f"{peaks['_source']} bf16 burst",
                "work": f"n(n+1)N = {h_flops:.4g} flop per launch (upper triangle incl. diagonal)"}

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(G, torch, W_host, X_host, st, n, out, dev, args.steps, flush)
        e2e["ms_per_step"] = max_over_ranks(e2e["ms_per_step"], world, dev)
        e2e["value"] = job_gparams_per_s(world, out, n, e2e["ms_per_step"])

    measured = measure_peaks(G, torch, dev) if not args.no_peaks else {}
    kernels = kernel_rooflines(trace, peaks, measured, prepare_ms=statistics.mean(prep_ms), n=n)
    kernels["note"] = (f"device time of each kernel on the stream it runs on, from the library's timing trace over a "
                       f"second pass of the same {args.steps} steps (the K4 and prepare products run on library "
                       "streams beside other kernels, so their times include sharing the SMs)")

    decode = time_qmatvec(G, torch, dev, peaks, flush) if world == 1 and not args.no_decode else None
    pipeline = time_pipeline(G, torch, dev) if world == 1 and not args.no_pipeline else None

    blocks = None
    if world == 1 and not args.no_blocks:
        del X, H, prep_ws, q_ws, prep, qout
        torch.cuda.empty_cache()
        blocks = {}
        for name in ("llama2-70b-block", "llama2-7b-block"):
            blocks[name] = time_block(G, torch, name, dev, steps=2, warmup=1, peaks=peaks, measured=measured)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        est, desc = oracle_sample(layer, st, min(N, args.ref_tokens))
        cpu = {"value": out * n / est / 1e9, "unit": UNIT, "cores": host_cores(), "kind": "oracle", "sample": desc}
        try:
            cpu["single_thread"] = oracle_single_thread()
        except Exception as e:  # a side figure: never let it cost the bench line
            cpu["single_thread"] = {"unavailable": f"{type(e).__name__}: {e}"}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16->f32 (Hessian), f32 (solver)", "data": "synthetic",
        "config": config_dict(args.workload, layer0, st),
        "hessian_tflops": achieved,
        "solver_gparam_per_s": solver_value,
        "stages_ms": {"clear": statistics.mean(clear_ms), "hessian": statistics.mean(hess_ms),
                      "prepare": statistics.mean(prep_ms), "quantize": statistics.mean(quant_ms)},
        "wall_ms_per_step_incl_flush": (t_wall1 - t_wall0) * 1e3 / args.steps,
        "roofline": roofline,
        "kernel_rooflines": kernels,
        "peaks_measured_here": measured,
        "blocks": blocks,
        "decode_qmatvec": decode,
        "pipeline": pipeline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_e2e(G, torch, W_host, X_host, st, n, out, dev, steps, flush):
    """Gparam/s through gptq_quantize with host inputs (pinned): H2D of W and X, D2H of the stored result."""
    stream = torch.cuda.current_stream()
    times = []
    h2d = W_host.numel() * W_host.element_size() + X_host.numel() * X_host.element_size()
    d2h = 0
    res_host = None
    # four untimed passes: the first allocates the pinned result buffers, and the library
    # captures its stages as CUDA graphs at the second call with the same arguments; the
    # call allocates its buffers while the previous step's are alive, so two sets of
    # addresses alternate and each needs two calls
    for i in range(steps + 4):
        flush.fill_(1.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        # host tensors: the library copies X in token chunks behind the Hessian's tile products
        q, prep, H = G.gptq_quantize(W_host, X_host.view(torch.bfloat16), st.bits, st.group_size, st.sym,
                                     st.desc_act, st.damp_percent, st.block, check=False)
        if res_host is None:
            res_host = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                        for t in (q.qweight, q.scales, q.zeros, q.g_idx)]
            d2h = sum(t.numel() * t.element_size() for t in res_host)
        for h, t in zip(res_host, (q.qweight, q.scales, q.zeros, q.g_idx)):
            h.copy_(t, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        G.raise_on_status(prep.status, "e2e")
        if i > 3:
            times.append(e0.elapsed_time(e1))
    ms = statistics.mean(times)
    return {"value": out * n / (ms * 1e-3) / 1e9, "unit": UNIT, "ms_per_step": ms, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h}


# --------------------------------------------------------------------------- #
# one whole decoder block
# --------------------------------------------------------------------------- #
# The inputs of a decoder block's linear layers: q, k and v read the same activations,
# o reads the attention output, gate and up the same MLP input, down the MLP's inner
# activations; H and U are formed once per input.
BLOCK_INPUTS = (("q", "k", "v"), ("o",), ("gate", "up"), ("down",))


def time_block(G, torch, name, dev, steps, warmup, peaks, measured):
    """One decoder block on one GPU: H and U once per input, then the layers of that input.

    Inputs are drawn on the device (synthetic.make_x_device / make_w_device: the same
    recipe as the parity tests' inputs, torch's generator).  Timed with CUDA events on
    this stream per input stage; a traced pass after the timed passes gives the
    per-kernel device times.  Returns a dict for the bench line.
    """
    wl = S.workloads()[name]
    st = wl.settings[0]
    by = {l.name: l for l in wl.layers}
    groups = [[by[nm] for nm in g if nm in by] for g in BLOCK_INPUTS]
    groups = [g for g in groups if g]
    xs = {}
    work = []     # (n, X, [W...], tokens, names) per input
    for g in groups:
        xspec = g[0].x
        if xspec.stream not in xs:
            xs[xspec.stream] = S.make_x_device(xspec, dev)
        Ws = [S.make_w_device(l.w, dev) for l in g]
        work.append((xspec.n, xs[xspec.stream], Ws, xspec.tokens, [l.name for l in g]))
    status = G.new_status(dev)
    stream = torch.cuda.current_stream()
    bufs = []
    for n, X, Ws, N, names in work:
        H = torch.empty((n, n), dtype=torch.float32, device=dev)
        hd = torch.empty(n, dtype=torch.float64, device=dev) if st.desc_act else None
        ws = G.workspace(G.lib().gptq_prepare_workspace_size(n), dev)
        prep = G.Prepared(U=torch.empty((n, n), dtype=torch.float32, device=dev),
                          perm=torch.empty(n, dtype=torch.int32, device=dev),
                          dead=torch.empty(n, dtype=torch.uint8, device=dev), status=status, desc_act=st.desc_act)
        rows = sum(int(W.shape[0]) for W in Ws)      # the layers of one input, stacked in one call
        qws = G.workspace(G.quantize_workspace_size(rows, n, st.block), dev)
        outs = G.alloc_quantized(rows, n, st.bits, st.group_size, st.sym, dev)
        bufs.append((H, hd, ws, prep, qws, outs))

    def once(ev=None):
        G.status_reset(status)
        for gi, ((n, X, Ws, N, names), (H, hd, ws, prep, qws, outs)) in enumerate(zip(work, bufs)):
            if ev is not None:
                ev[gi][4].record(stream)
            H.zero_()
            if hd is not None:
                hd.zero_()
            if ev is not None:
                ev[gi][0].record(stream)
            G.hessian_accumulate(H, X, hd, status)
            if ev is not None:
                ev[gi][1].record(stream)
            G.prepare(H, st.damp_percent, st.desc_act, hd, status, ws=ws, out=prep)
            if ev is not None:
                ev[gi][2].record(stream)
            G.quantize_layers(Ws, prep, st.bits, st.group_size, st.sym, st.block, ws=qws, out=outs)
            if ev is not None:
                ev[gi][3].record(stream)

    # two warm-up passes at least: the library captures a stage as a CUDA graph the second
    # time it sees the same arguments, so the timed passes replay graphs
    for _ in range(max(2, warmup)):
        once()
    torch.cuda.synchronize()
    G.raise_on_status(status, "block warm-up")
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in work] for _ in range(steps)]
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    for i in range(steps):
        once(evs[i])
    torch.cuda.synchronize()
    clk = clocks.stop()
    G.raise_on_status(status, "block")
    G.trace_read()
    G.trace_enable(True)
    once()
    torch.cuda.synchronize()
    G.trace_enable(False)
    trace = G.trace_read()
    # for comparison: the same layers quantized one call per layer (same U, same outputs' sizes)
    separate = []
    for (n, X, Ws, N, names), (H, hd, ws, prep, qws, outs) in zip(work, bufs):
        if len(Ws) == 1:
            separate.append(None)
            continue
        qs = [G.alloc_quantized(int(W.shape[0]), n, st.bits, st.group_size, st.sym, dev) for W in Ws]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for W, q in zip(Ws, qs):
            G.quantize_layer(W, prep, st.bits, st.group_size, st.sym, st.block, ws=qws, out=q)
        e1.record(stream)
        torch.cuda.synchronize()
        separate.append(e0.elapsed_time(e1))
        del qs
    G.raise_on_status(status, "block, separate calls")
    per_input = []
    hess_flop, hess_s = 0.0, 0.0
    for gi, (n, X, Ws, N, names) in enumerate(work):
        h = statistics.mean(evs[i][gi][0].elapsed_time(evs[i][gi][1]) for i in range(steps))
        pr = statistics.mean(evs[i][gi][1].elapsed_time(evs[i][gi][2]) for i in range(steps))
        qu = statistics.mean(evs[i][gi][2].elapsed_time(evs[i][gi][3]) for i in range(steps))
        per_input.append({"layers": names, "in": n, "out": [int(W.shape[0]) for W in Ws], "tokens": N,
                          "hessian_ms": h, "prepare_ms": pr, "quantize_ms": qu,
                          "quantize_ms_one_call_per_layer": separate[gi],
                          "hessian_tflops": float(n) * (n + 1) * N / (h * 1e-3) / 1e12})
        hess_flop += float(n) * (n + 1) * N
        hess_s += h * 1e-3
    block_ms = statistics.mean(evs[i][0][4].elapsed_time(evs[i][-1][3]) for i in range(steps))   # clears included
    weights = sum(int(W.numel()) for _, _, Ws, _, _ in work for W in Ws)
    achieved = hess_flop / hess_s / 1e12
    kr = kernel_rooflines(trace, peaks, measured)
    res = {
        "seconds_per_block": block_ms * 1e-3, "gparam_per_s": weights / (block_ms * 1e-3) / 1e9,
        "weights": weights, "steps": steps, "warmup": warmup,
        "config": {"workload": name, "bits": st.bits, "group_size": st.group_size, "sym": st.sym,
                   "desc_act": st.desc_act, "damp_percent": st.damp_percent,
                   "inputs": "H and U once per input: q/k/v, o, gate/up, down; the layers of one input "
                             "quantized in one call (gptq_quantize_layers)",
                   "data": "synthetic, drawn on the device (same recipe as the tests' inputs)"},
        "per_input": per_input,
        "hessian_roofline": {"bound": "tensor", "unit": "TFLOP/s", "achieved": achieved,
                             "peak": float(peaks["bf16_tflops"]), "frac": achieved / float(peaks["bf16_tflops"]),
                             "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained",
                                                                             peaks["bf16_tflops"])),
                             "peak_source": f"{peaks['_source']} bf16 burst (and sustained)"},
        "kernel_rooflines": kr,
        "clocks": clk,
    }
    del work, bufs, xs
    torch.cuda.empty_cache()
    return res


def run_block(args):
    """Time every layer of a decoder block on one GPU; prints its own JSON line."""
    import torch

    import post_weight_quantization_15_b200 as G

    if not torch.cuda.is_available():
        raise SystemExit("bench.py --block needs a CUDA device")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    measured = measure_peaks(G, torch, dev)
    r = time_block(G, torch, args.block, dev, max(1, min(args.steps, 3)), max(1, min(args.warmup, 2)), peaks,
                   measured)
    line = {"metric": f"GPTQ decoder block ({args.block}): seconds per block, 1 B200",
            "value": r["seconds_per_block"], "unit": "s", "higher_is_better": False, "n_gpus": 1,
            "data": "synthetic", **r, "peaks_measured_here": measured}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(S.workloads().keys()))
    ap.add_argument("--ref-tokens", type=int, default=8192,
                    help="token sample of the CPU oracle legs (its Hessian time is scaled to the full count)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--block", default=None, choices=["llama2-7b-block", "llama2-70b-block"],
                    help="time every layer of a decoder block instead (its own JSON line)")
    ap.add_argument("--no-blocks", action="store_true",
                    help="leave the two decoder blocks out of the default line")
    ap.add_argument("--no-decode", action="store_true", help="leave the decode-shape qmatvec leg out")
    ap.add_argument("--no-pipeline", action="store_true", help="leave the sequential-pipeline leg out")
    ap.add_argument("--no-peaks", action="store_true", help="do not measure the tf32 / fp32 peaks here")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.block:
        return run_block(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
