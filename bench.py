#!/usr/bin/env python3
"""Benchmark of the fused tile-rANS decode + GEMM on one B200 per rank.

Headline workload (the largest layer of the pages' workloads that fits one
GPU): a 53248 x 16384 fp8 e4m3 weight matrix shaped like a Llama-405B
projection (w ~ N(0, 0.02), per-row absmax scale amax/448 stored fp32),
coded as one rANS stream of 8-bit symbols per 128 x 128 tile (one 12-bit
codebook per layer, 32 lanes; by default the wide-state stream format,
--state-bits 32 for 32-bit lane states), multiplied by X (16 x 16384 bf16,
N(0, 1)).  One step is one ans_gemm call (decode inside the GEMM, fp32 Y).
The compressed layer (~0.7 GB, two copies alternating) is far larger than
the 126 MB L2, so every step reads its weights from HBM.

A secondary entry times the bf16 4096 x 4096 split-stream layer at M = 16
(exponent coded per 128 x 64 tile, raw sign/mantissa byte), twelve rotating
copies in CUDA graphs of consecutive calls.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle on
the same workload instead.  Under torchrun every rank runs its own replica
(no data-path collective: the layers are independent); the time is the max
over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "fp8_405b"
M_HEAD = 16
HEAD_COPIES = 2
SECOND = "bf16_4096"
SECOND_COPIES = 12
METRIC = ("fused decode-GEMM effective weight GB/s (405B-shaped fp8 e4m3 layer "
          "53248x16384, M=16)")
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
# nominal storage bytes per weight of the decompressed layer
NOMINAL = {0: 0.5, 1: 2.0, 2: 1.0, 3: 0.5, 4: 1.0, 5: 0.5, 6: 0.5}
# sources of the kernel the bench times at M = 16 (the local schedule); the
# committed DRAM-traffic summary is only used while they are unchanged
KERNEL_SOURCES = ["rans_decode_gemm_b200/csrc/cuda/gemm_local.cu",
                  "rans_decode_gemm_b200/csrc/cuda/kernels.h",
                  "rans_decode_gemm_b200/csrc/cuda/gemm_common.cuh",
                  "rans_decode_gemm_b200/csrc/cuda/rans_core.cuh",
                  "rans_decode_gemm_b200/csrc/cuda/ptx.cuh",
                  "rans_decode_gemm_b200/csrc/cuda/launch.h"]
TRAFFIC_PROFILE = "profiles/fused_gemm_local_fp8_405b_m16.json"


def workload_name(name, state_bits, M):
    fmt = ("64-bit lane states, 32-bit words, one renormalisation test per symbol pair"
           if state_bits == 64 else "32-bit lane states, 16-bit words") + \
        ", final states flushed in whole bytes"
    if name == "fp8_405b":
        return ("405B-shaped fp8 e4m3 53248x16384, w~N(0,0.02) / (row amax/448), fp32 row "
                "scales, 8-bit symbols, 128x128 tiles, 32 lanes, 12-bit freqs, "
                f"{fmt}; X {M}x16384 bf16 N(0,1); seed 4")
    return ("bf16 split-stream 4096x4096 N(0,0.02), 128x64 tiles, 32 lanes, 12-bit freqs, "
            f"{fmt}; X {M}x4096 bf16 N(0,1); seed 1")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="every workload of the pages at full size, one JSON line per point "
                         "(instead of the benchmark line)")
    ap.add_argument("--sweep-configs", default="", help="comma-separated subset for --sweep")
    ap.add_argument("--sweep-ms", default="", help="comma-separated token counts for --sweep "
                                                   "(default: each workload's own)")
    ap.add_argument("--state-bits", type=int, default=64, choices=[32, 64],
                    help="stream format: 64 = wide lane states (32-bit words, one "
                         "renormalisation test per symbol pair), 32 = 32-bit states")
    ap.add_argument("--nibble-symbols", default="pairs", choices=["pairs", "element"],
                    help="--sweep: code int4 and fp4 weights one symbol per packed byte "
                         "(two K elements) or one per element")
    ap.add_argument("--rows", type=int, default=0,
                    help="profiling: the headline layer (or, with --sweep, every matrix) cut "
                         "to its first ROWS rows (a multiple of the tile height); 0 = whole")
    ap.add_argument("--quick", action="store_true",
                    help="only the headline timing: no context sweep, secondary entry or "
                         "CPU baseline (profiling runs)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            return json.load(fh), "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """dram read+write bytes per launch of the headline kernel from the
    committed ncu summary, if it was taken on the current kernel source."""
    path = os.path.join(ROOT, TRAFFIC_PROFILE)
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        d = json.load(fh)
    if d.get("kernel_source_sha") != kernel_source_hash():
        return None
    return d.get("dram_bytes_per_launch")


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class ClockSampler:
    """nvidia-smi clock / throttle sampling (20 ms period, host timestamps),
    started before the warm-up; the samples that fall inside the timed window
    are reported separately from those of the whole loaded window."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.window = None

    def start(self, wait_s: float = 3.0):
        """Starts the sampler and returns once its first sample is written."""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            return
        t_end = time.time() + wait_s
        while time.time() < t_end:
            if os.path.getsize(self.file.name) > 0:
                break
            time.sleep(0.01)

    def mark(self, t0: float, t1: float):
        """Host-time bounds of the timed region."""
        self.window = (t0, t1)

    @staticmethod
    def _ts(s: str):
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(s, fmt).timestamp()
            except ValueError:
                pass
        return None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        rows = []
        with open(self.file.name) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 10:
                    rows.append(parts)
        os.unlink(self.file.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None

        timed = []
        if self.window is not None:
            a, b = self.window
            for r in rows:
                t = self._ts(r[0])
                if t is not None and a - 0.02 <= t <= b + 0.02:
                    timed.append(r)
        use = timed if timed else rows
        sm = [v for v in (num(r[2]) for r in use) if v is not None]
        smax = [v for v in (num(r[3]) for r in rows) if v is not None]
        reasons = sorted({n for r in use for n, v in zip(self.REASONS, r[6:10])
                          if v.lower() == "active"})
        under_load = sorted(sm)[len(sm) // 2:] if sm else []
        return {"sm_mhz": statistics.median(under_load) if under_load else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(use), "samples_in_timed_region": len(timed),
                "samples_total": len(rows), "period_ms": 20,
                "window": "timed region" if timed else
                          "warm-up and timed region (no sample fell inside the timed region)"}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args is not None and world > 1 and args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    return world, rank, local


def max_over_ranks(pg, values, device):
    """Every rank's times -> the max over ranks of each, on every rank.  All
    ranks call it at the same point with the same number of values."""
    if pg is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return [float(v) for v in t.cpu().tolist()]


def replica_gbs(world, bytes_per_step, ms_per_step):
    """Whole-job throughput of `world` independent replicas, each moving
    `bytes_per_step` per step, timed by the slowest rank at `ms_per_step`."""
    return world * bytes_per_step / (ms_per_step * 1e-3) / 1e9


def percentiles(vals):
    v = sorted(vals)
    if not v:
        return None

    def q(p):
        return v[min(len(v) - 1, max(0, int(round(p * (len(v) - 1)))))]
    return {"p10": round(q(0.10), 6), "p50": round(q(0.50), 6), "p90": round(q(0.90), 6),
            "n": len(v)}


def build_layers(torch, ans, WL, name, device, state_bits, copies, rows=0):
    """Offline path through the library (GPU histogram -> codebook -> host
    encode), then `copies` device copies of the compressed layer (its first
    `rows` rows when rows > 0)."""
    cfg = WL.CONFIGS[name]
    d = WL.make_weights(cfg, 0, N=rows if rows else None)
    lay = ans.make_layout(cfg.dtype, d["N"], d["K"], cfg.tile_n, cfg.tile_k, state_bits)
    w = d["w"]
    dw = torch.from_numpy(w.view(np.int16) if w.dtype == np.uint16 else w).to(device)
    A = ans.ALPHABET[cfg.dtype]
    hist = torch.zeros(A, dtype=torch.int64, device=device)
    ans.ans_histogram(dw, lay, hist)
    hist_h = hist.cpu().numpy().astype(np.uint64)
    t0 = time.perf_counter()
    cb = ans.ans_build_codebook(hist_h, A, 12)
    stream, offsets, raw = ans.ans_encode_tiles(w, lay, cb)
    encode_s = time.perf_counter() - t0
    layers = [ans.CompressedLayer(lay, cb, stream, offsets, raw, device) for _ in range(copies)]
    sc = None
    if d["scales"] is not None:
        s = np.ascontiguousarray(d["scales"])
        sc = torch.from_numpy(s.view(np.int16) if s.dtype == np.uint16 else s).to(device)
    return cfg, d, lay, layers, hist_h, encode_s, dw, sc


def algo_bytes(layer, cfg, M, N, K):
    """Bytes one ans_gemm call must move at the least: the compressed layer,
    the scales, X in and Y out."""
    sbytes = 0
    if cfg.scale_kind in (1, 3):
        sbytes = 2 * N * (K // cfg.group_k if cfg.scale_kind == 3 else 1)
    elif cfg.scale_kind == 2:
        sbytes = 4 * N
    return layer.compressed_bytes + sbytes + 2 * M * K + 4 * M * N


def time_ours(args):
    import torch
    from rans_decode_gemm_b200 import ans
    from rans_decode_gemm_b200 import workloads as WL

    world, rank, local = dist_setup(args)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=device)
        pg = dist
    cfg, d, lay, layers, hist, encode_s, dw, sc = build_layers(
        torch, ans, WL, WORKLOAD, device, args.state_bits, HEAD_COPIES, args.rows)
    N, K, M = lay.N, lay.K, M_HEAD
    X_h = WL.make_x(cfg, M, K)
    X = torch.from_numpy(X_h.view(np.int16)).to(device)
    Y = torch.empty(M, N, dtype=torch.float32, device=device)
    ws_bytes = ans.ans_gemm_workspace(lay, M, cfg.scale_kind)
    ws = torch.zeros(max(ws_bytes, 256), dtype=torch.uint8, device=device)
    st = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.Stream(device=device)
    torch.cuda.set_stream(stream)

    def step(i):
        ans.ans_gemm(X, M, layers[i % HEAD_COPIES].tiles, cfg.scale_kind, sc, cfg.group_k, Y, ws,
                     ws.numel(), st, stream)

    def barrier():
        torch.cuda.synchronize()
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()

    # Each call is about a millisecond of GPU work, so plain stream launches
    # keep the GPU busy; an event before every call gives the per-call
    # spread, the first and last events bracket the timed region.
    sampler = ClockSampler(local)
    sampler.start()
    for i in range(args.warmup):
        step(i)
    barrier()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    h0 = time.time()
    ev[0].record(stream)
    for i in range(args.steps):
        step(i)
        ev[i + 1].record(stream)
    barrier()
    h1 = time.time()
    sampler.mark(h0, h1)
    clocks = sampler.stop()
    total_ms = ev[0].elapsed_time(ev[-1])
    per_call = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    kern_ms = total_ms / args.steps
    status = int(st.item())
    total_ms, = max_over_ranks(pg, [total_ms], device)

    # e2e through the same C ABI with host buffers: pinned X in, Y out per step
    Xp = torch.from_numpy(X_h.view(np.int16)).pin_memory()
    Yp = torch.empty(M, N, dtype=torch.float32).pin_memory()
    Xd = torch.empty_like(X)

    def e2e_step(i):
        Xd.copy_(Xp, non_blocking=True)
        ans.ans_gemm(Xd, M, layers[i % HEAD_COPIES].tiles, cfg.scale_kind, sc, cfg.group_k, Y,
                     ws, ws.numel(), st, stream)
        Yp.copy_(Y, non_blocking=True)

    for i in range(min(args.warmup, 20)):
        e2e_step(i)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    n_e2e = max(1, min(args.steps, 200))
    e0.record(stream)
    for i in range(n_e2e):
        e2e_step(i)
    e1.record(stream)
    barrier()
    e2e_ms, = max_over_ranks(pg, [e0.elapsed_time(e1) / n_e2e], device)

    extra = {}
    if rank == 0 and not args.quick:
        extra = context_numbers(torch, ans, WL, cfg, d, lay, layers, dw, sc, device, stream)
        del dw
        torch.cuda.empty_cache()
        extra["secondary"] = secondary_entry(torch, ans, WL, args, device, stream)

    result = None
    if rank == 0:
        peaks, peaks_src = load_peaks()
        weight_bytes = N * K * NOMINAL[cfg.dtype]  # nominal storage of the decompressed weights
        layer = layers[0]
        ab = algo_bytes(layer, cfg, M, N, K)
        # the local schedule (M <= 32 tokens per 128-row half) is one kernel
        launches_per_step = 1
        ms_per_step = total_ms / args.steps
        value = replica_gbs(world, weight_bytes, ms_per_step)
        achieved = ab / (kern_ms * 1e-3) / 1e9
        peak = float(peaks["hbm_gbs"])
        H = ans.ans_entropy(hist)
        bpw = 8.0 * layer.compressed_bytes / (N * K)
        result = {
            "metric": METRIC,
            "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {"workload": workload_name(WORKLOAD, args.state_bits, M) +
                                   (f" (first {N} rows only)" if args.rows else ""),
                       "state_bits": args.state_bits,
                       "M": M, "N": N, "K": K, "global_batch": M * world,
                       "parallelism": f"replicas x{world}",
                       "l2": f"inputs larger than L2: {HEAD_COPIES} alternating copies of the "
                             f"compressed layer ({layer.compressed_bytes / 1e6:.0f} MB each)"},
            "per_call_ms": percentiles(per_call),
            "bits_per_weight": round(bpw, 4),
            "entropy_bits": round(H, 4), "gap_bits": round(bpw - H, 4),
            "status": status,
            "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                         "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "traffic": profiled_traffic(), "peak_source": peaks_src,
                         "algorithmic_bytes_per_launch": ab,
                         "kernel_ms_per_launch": round(kern_ms, 6),
                         "timing": "CUDA events on the launch stream around each ans_gemm "
                                   "call (one kernel launch per call)"},
            "e2e": {"value": round(replica_gbs(world, weight_bytes, e2e_ms), 2), "unit": "GB/s",
                    "h2d_bytes_per_step": 2 * M * K, "d2h_bytes_per_step": 4 * M * N},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "offline": {"host_encode_s": round(encode_s, 3)},
        }
        result.update(extra)
        if "decode_tiles_Tsym_per_s" in extra:
            # the second ceiling: the rate at which the fused kernel decodes
            # symbols against the standalone decode kernel on the same layer
            fused_rate = N * K / (kern_ms * 1e-3) / 1e12
            ceil = extra["decode_tiles_Tsym_per_s"]
            result["decode_ceiling"] = {
                "unit": "T symbols/s", "fused": round(fused_rate, 4),
                "standalone_decode": ceil, "frac": round(fused_rate / ceil, 4),
                "note": "ans_gemm symbol rate / ans_decode_tiles symbol rate, same layer, same run"}
        if not (args.no_cpu_baseline or args.quick):
            result["cpu_baseline"] = cpu_baseline(cfg, d, lay, layer, X_h)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    return result


def timed_events(torch, stream, fn, iters, warm):
    """Average µs per call of fn(i) over `iters` calls after `warm` untimed
    ones (CUDA events on `stream`)."""
    for i in range(warm):
        fn(i)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(iters):
        fn(i)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters * 1e3


def context_numbers(torch, ans, WL, cfg, d, lay, layers, dw, sc, device, stream):
    """Single-GPU context on the headline layer: ans_gemm at the workload's
    token counts, the same kernel on uncompressed weights, cuBLAS on dense
    bf16 weights, ans_decode_tiles and the two-pass baselines (decode to HBM,
    then the uncompressed kernel or cuBLAS)."""
    N, K = lay.N, lay.K
    st = torch.zeros(1, dtype=torch.int32, device=device)
    peaks, _ = load_peaks()
    nc = len(layers)
    Wb = dequant_bf16(torch, cfg, d, device)
    dec = torch.empty(dw.numel() * dw.element_size(), dtype=torch.uint8, device=device)
    t_d = timed_events(torch, stream, lambda i: ans.ans_decode_tiles(layers[i % nc].tiles, dec, st),
                       10, 2)
    out = {"sweep": []}
    for M in cfg.Ms:
        X = torch.from_numpy(WL.make_x(cfg, M, K).view(np.int16)).to(device)
        Y = torch.empty(M, N, dtype=torch.float32, device=device)
        Yu = torch.empty(M, N, dtype=torch.float32, device=device)
        nb = ans.ans_gemm_workspace(lay, M, cfg.scale_kind)
        ws = torch.zeros(max(nb, 256), dtype=torch.uint8, device=device)
        it = max(3, min(50, int(40000 / (M + 100))))
        t_f = timed_events(torch, stream, lambda i: ans.ans_gemm(
            X, M, layers[i % nc].tiles, cfg.scale_kind, sc, cfg.group_k, Y, ws, ws.numel(), st),
            it, 2)
        t_u = timed_events(torch, stream, lambda i: ans.ans_gemm_uncompressed(
            X, M, dw, lay, cfg.scale_kind, sc, cfg.group_k, Yu, ws, ws.numel(), st), it, 2)
        same = bool(torch.equal(Y, Yu))
        Xb = X.view(torch.bfloat16)
        t_c = timed_events(torch, stream, lambda i: torch.matmul(Xb, Wb.t()), it, 2)
        ab = algo_bytes(layers[0], cfg, M, N, K)
        flops = 2.0 * M * N * K
        out["sweep"].append({
            "M": M, "ans_gemm_us": round(t_f, 2),
            "effective_weight_GBps": round(N * K * NOMINAL[cfg.dtype] / (t_f * 1e-6) / 1e9, 1),
            "hbm_frac": round(ab / (t_f * 1e-6) / 1e9 / float(peaks["hbm_gbs"]), 4),
            "tensor_frac": round(flops / (t_f * 1e-6) / 1e12 / float(peaks["bf16_tflops"]), 5),
            "uncompressed_us": round(t_u, 2), "bit_identical_to_uncompressed": same,
            "cublas_bf16_us": round(t_c, 2), "decode_tiles_us": round(t_d, 2),
            "two_pass_us": round(t_d + t_u, 2), "two_pass_cublas_us": round(t_d + t_c, 2),
            "speedup_vs_two_pass": round((t_d + t_u) / t_f, 3),
            "speedup_vs_two_pass_cublas": round((t_d + t_c) / t_f, 3),
            "status": int(st.item())})
        del X, Y, Yu, ws
    out["decode_tiles_Tsym_per_s"] = round(N * K / (t_d * 1e-6) / 1e12, 4)
    del Wb, dec
    return out


def secondary_entry(torch, ans, WL, args, device, stream):
    """The bf16 4096 x 4096 split-stream layer at M = 16: twelve rotating
    copies, CUDA graphs of twelve consecutive calls, events per replay."""
    cfg, d, lay, layers, hist, encode_s, dw, sc = build_layers(
        torch, ans, WL, SECOND, device, args.state_bits, SECOND_COPIES)
    N, K, M = lay.N, lay.K, 16
    X = torch.from_numpy(WL.make_x(cfg, M, K).view(np.int16)).to(device)
    Y = torch.empty(M, N, dtype=torch.float32, device=device)
    nb = ans.ans_gemm_workspace(lay, M, 0)
    ws = torch.zeros(max(nb, 256), dtype=torch.uint8, device=device)
    st = torch.zeros(1, dtype=torch.int32, device=device)

    def step(i):
        ans.ans_gemm(X, M, layers[i % SECOND_COPIES].tiles, 0, None, 0, Y, ws, ws.numel(), st,
                     stream)
    for i in range(SECOND_COPIES):
        step(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(SECOND_COPIES):
            step(i)
    reps = 60
    for _ in range(5):
        g.replay()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    ev[0].record(stream)
    for r in range(reps):
        g.replay()
        ev[r + 1].record(stream)
    torch.cuda.synchronize()
    per = [ev[r].elapsed_time(ev[r + 1]) / SECOND_COPIES for r in range(reps)]
    ms = ev[0].elapsed_time(ev[-1]) / (reps * SECOND_COPIES)
    del g
    peaks, _ = load_peaks()
    ab = algo_bytes(layers[0], cfg, M, N, K)
    return {"workload": workload_name(SECOND, args.state_bits, M),
            "value": round(N * K * 2 / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "ms_per_call": round(ms, 6), "per_call_ms": percentiles(per),
            "bits_per_weight": round(8.0 * layers[0].compressed_bytes / (N * K), 4),
            "entropy_bits_split_bound": round(ans.ans_entropy(hist) + 8, 4),
            "roofline": {"bound": "hbm", "achieved": round(ab / (ms * 1e-3) / 1e9, 2),
                         "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                         "frac": round(ab / (ms * 1e-3) / 1e9 / float(peaks["hbm_gbs"]), 4),
                         "algorithmic_bytes_per_launch": ab},
            "status": int(st.item()),
            "timing": f"CUDA graphs of {SECOND_COPIES} consecutive calls over rotating copies"}


def dequant_bf16(torch, cfg, d, device):
    """Dense bf16 copy of the dequantised weights (for the cuBLAS reference)."""
    N, K = d["N"], d["K"]
    if cfg.dtype == 1:  # bf16 bits
        return torch.from_numpy(d["w"].view(np.int16)).to(device).view(torch.bfloat16).view(N, K)
    if cfg.dtype == 0:  # packed int4 nibbles, element k even in the low nibble
        b = torch.from_numpy(d["w"]).to(device)
        nib = torch.stack([b & 0xF, b >> 4], dim=1).view(N, K).to(torch.int16)
        q = torch.where(nib >= 8, nib - 16, nib).to(torch.float32)
        s = torch.from_numpy(d["scales"].view(np.int16)).to(device).view(torch.bfloat16).float()
        if s.dim() == 1:
            return (q * s[:, None]).to(torch.bfloat16)
        return (q * s.repeat_interleave(K // s.shape[1], dim=1)).to(torch.bfloat16)
    if cfg.dtype == 5:  # e2m1 codes (packed like int4), fp32 row scales
        b = torch.from_numpy(d["w"]).to(device)
        c = torch.stack([b & 0xF, b >> 4], dim=1).view(N, K).long()
        grid = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], device=device)
        v = grid[c & 7] * torch.where((c & 8) != 0, -1.0, 1.0)
        s = torch.from_numpy(d["scales"]).to(device)
        return (v * s[:, None]).to(torch.bfloat16)
    if cfg.dtype == 4:  # int8 codes, fp32 row scales
        q = torch.from_numpy(d["w"].view(np.int8)).to(device).view(N, K).float()
        s = torch.from_numpy(d["scales"]).to(device)
        return (q * s[:, None]).to(torch.bfloat16)
    out = torch.empty(N, K, dtype=torch.bfloat16, device=device)
    codes = torch.from_numpy(d["w"]).to(device).view(torch.float8_e4m3fn).view(N, K)
    s = torch.from_numpy(d["scales"]).to(device)
    for r0 in range(0, N, 4096):  # in row chunks: the fp32 temporary stays small
        out[r0:r0 + 4096] = (codes[r0:r0 + 4096].float() * s[r0:r0 + 4096, None]).to(torch.bfloat16)
    return out


def whole16_row(args, torch, ans, name, mname, w, N, K, cfg, split_bpw, split_bound, split_dec_us,
                st, timed_graph):
    """bf16 coded as whole 16-bit symbols against the split stream on the same
    layer: bits/weight, the entropy bound, and the standalone decode time."""
    hist = ans.ans_histogram16_host(w)
    freq = ans.ans_build_codebook16(hist, 16)
    lay = ans.make_layout(ans.BF16_WHOLE, N, K, cfg.tile_n, cfg.tile_k, args.state_bits)
    stream, offsets = ans.ans_encode_tiles16(w, lay, freq, 16)
    table = ans.ans_decode_table16(freq, 16)
    d_stream = torch.from_numpy(np.concatenate([stream, np.zeros(16, np.uint8)])).cuda()
    d_off = torch.from_numpy(offsets.view(np.int64)).cuda()
    d_table = torch.from_numpy(table).cuda()
    out = torch.empty(N * K, dtype=torch.int16, device="cuda")
    call = [lambda: ans.ans_decode_tiles16(lay, d_table, d_stream, stream.size, d_off, out, st)]
    t = timed_graph(call, 3)
    t = timed_graph(call, max(3, min(200, int(20000 / max(t, 1.0)))))
    exact = bool(np.array_equal(out.cpu().numpy().view(np.uint16), w))
    bpw = 8.0 * (stream.size + 8 * offsets.size) / (N * K)
    return {"workload": name, "matrix": mname, "N": N, "K": K, "coding": "bf16 whole 16-bit symbols",
            "state_bits": args.state_bits, "prob_bits": 16, "present_symbols": int((freq > 0).sum()),
            "bits_per_weight": round(bpw, 4), "entropy_bound_bits": round(ans.ans_entropy(hist), 4),
            "gap_bits": round(bpw - ans.ans_entropy(hist), 4), "decode_tiles16_us": round(t, 2),
            "decode_Tsym_per_s": round(N * K / (t * 1e-6) / 1e12, 4), "bit_exact": exact,
            "split_bits_per_weight": round(split_bpw, 4), "split_entropy_bound_bits": round(split_bound, 4),
            "split_decode_tiles_us": round(split_dec_us, 2), "status": int(st.item())}


def sweep(args):
    """Every workload of the pages at full size on one GPU: bits/weight against
    the entropy bound, ans_gemm at each M of the workload, the same kernel on
    uncompressed weights, ans_decode_tiles, cuBLAS on dense bf16 weights, the
    two-pass baselines (decode to HBM, then ans_gemm_uncompressed on the decoded
    weights, or cuBLAS on bf16 weights), and roofline fractions.  Weights stream from HBM (enough rotating copies
    to exceed L2).  One JSON line per point."""
    import torch
    from rans_decode_gemm_b200 import ans
    from rans_decode_gemm_b200 import workloads as WL
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    peaks, peaks_src = load_peaks()
    st = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.Stream(device=device)
    torch.cuda.set_stream(stream)

    def timed_graph(calls, reps):
        """Average µs per call of `calls` (a list of closures), captured as one
        CUDA graph and replayed `reps` times after one warm replay."""
        for c in calls:
            c()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for c in calls:
                c()
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        del g
        return a.elapsed_time(b) * 1e3 / (reps * len(calls))

    only = set(args.sweep_configs.split(",")) if args.sweep_configs else None
    ms_only = [int(m) for m in args.sweep_ms.split(",")] if args.sweep_ms else None
    for name, cfg in WL.CONFIGS.items():
        if only and name not in only:
            continue
        for mi, (mname, mN, mK) in enumerate(cfg.matrices):
            d = WL.make_weights(cfg, mi, N=args.rows if args.rows else None)
            N, K = d["N"], d["K"]
            pairs = cfg.dtype in (WL.INT4, WL.FP4_E2M1) and args.nibble_symbols == "pairs"
            coded = ({WL.INT4: WL.INT4_PAIRS, WL.FP4_E2M1: WL.FP4_PAIRS}[cfg.dtype] if pairs
                     else cfg.dtype)
            lay = ans.make_layout(coded, N, K, cfg.tile_n, cfg.tile_k, args.state_bits)
            dw = torch.from_numpy(d["w"].view(np.int16) if d["w"].dtype == np.uint16 else d["w"]).to(device)
            A = ans.ALPHABET[coded]
            hist = torch.zeros(A, dtype=torch.int64, device=device)
            ans.ans_histogram(dw, lay, hist)
            hist_h = hist.cpu().numpy().astype(np.uint64)
            t0 = time.perf_counter()
            cb = ans.ans_build_codebook(hist_h, A, 12)
            stream_h, offsets_h, raw_h = ans.ans_encode_tiles(d["w"], lay, cb)
            encode_s = time.perf_counter() - t0
            comp = int(stream_h.size + 8 * offsets_h.size + (raw_h.size if raw_h is not None else 0))
            copies = int(max(1, min(12, -(-256e6 // comp))))
            layers = [ans.CompressedLayer(lay, cb, stream_h, offsets_h, raw_h, device) for _ in range(copies)]
            H = ans.ans_entropy(hist_h)
            # per weight: + the raw byte (bf16); a pair symbol carries two weights
            bound = H + 8.0 if cfg.dtype == 1 else (H / 2 if pairs else H)
            bpw = 8.0 * layers[0].compressed_bytes / (N * K)
            sc = None
            if d["scales"] is not None:
                s = np.ascontiguousarray(d["scales"])
                sc = torch.from_numpy(s.view(np.int16) if s.dtype == np.uint16 else s).to(device)
            Wb = dequant_bf16(torch, cfg, d, device)
            wcopies = max(1, min(copies, int(-(-256e6 // (N * K * 2)))))
            Wbs = [Wb] + [Wb.clone() for _ in range(wcopies - 1)]
            dec = torch.empty(N * K * (2 if cfg.dtype == 1 else 1) // (2 if cfg.dtype in (0, 5) else 1),
                              dtype=torch.uint8, device=device)
            rep_for = lambda us_est: max(3, min(200, int(20000 / max(us_est, 1.0))))
            t_dec = timed_graph([lambda l=l: ans.ans_decode_tiles(l.tiles, dec, st) for l in layers], 3)
            t_dec = timed_graph([lambda l=l: ans.ans_decode_tiles(l.tiles, dec, st) for l in layers],
                                rep_for(t_dec * copies))
            if cfg.dtype == WL.BF16_SPLIT:
                print(json.dumps(whole16_row(args, torch, ans, name, mname, d["w"], N, K, cfg, bpw,
                                             bound, t_dec, st, timed_graph)), flush=True)
            for M in (ms_only or cfg.Ms):
                X = torch.from_numpy(WL.make_x(cfg, M, K).view(np.int16)).to(device)
                Y = torch.empty(M, N, dtype=torch.float32, device=device)
                Yu = torch.empty(M, N, dtype=torch.float32, device=device)
                nb = ans.ans_gemm_workspace(lay, M, cfg.scale_kind)
                ws = torch.zeros(max(nb, 256), dtype=torch.uint8, device=device)
                fused = [lambda l=l: ans.ans_gemm(X, M, l.tiles, cfg.scale_kind, sc, cfg.group_k, Y, ws, nb, st)
                         for l in layers]
                plain = [lambda: ans.ans_gemm_uncompressed(X, M, dw, lay, cfg.scale_kind, sc, cfg.group_k,
                                                           Yu, ws, nb, st)]
                t_f = timed_graph(fused, 2)
                t_f = timed_graph(fused, rep_for(t_f * copies))
                t_u = timed_graph(plain, 2)
                t_u = timed_graph(plain, rep_for(t_u))
                same = bool(torch.equal(Y, Yu))
                Xb = X.view(torch.bfloat16)
                cub = [lambda w=w: torch.matmul(Xb, w.t()) for w in Wbs]
                t_c = timed_graph(cub, 2)
                t_c = timed_graph(cub, rep_for(t_c * len(cub)))
                ab = algo_bytes(layers[0], cfg, M, N, K)
                rec = {"workload": name, "matrix": mname, "N": N, "K": K, "M": M,
                       "state_bits": args.state_bits,
                       **({"nibble_symbols": args.nibble_symbols}
                          if cfg.dtype in (WL.INT4, WL.FP4_E2M1) else {}),
                       "tile": f"{lay.tile_n}x{lay.tile_k}", "bits_per_weight": round(bpw, 4),
                       "entropy_bound_bits": round(bound, 4), "gap_bits": round(bpw - bound, 4),
                       "encode_s": round(encode_s, 2), "copies": copies,
                       "ans_gemm_us": round(t_f, 2),
                       "effective_weight_GBps": round(N * K * NOMINAL[cfg.dtype] / (t_f * 1e-6) / 1e9, 1),
                       "hbm_frac": round(ab / (t_f * 1e-6) / 1e9 / float(peaks["hbm_gbs"]), 4),
                       "tensor_frac": round(2.0 * M * N * K / (t_f * 1e-6) / 1e12 / float(peaks["bf16_tflops"]), 4),
                       "uncompressed_us": round(t_u, 2), "bit_identical_to_uncompressed": same,
                       "decode_tiles_us": round(t_dec, 2),
                       "decode_Tsym_per_s": round(N * K / (t_dec * 1e-6) / 1e12, 4),
                       "two_pass_us": round(t_dec + t_u, 2),
                       "speedup_vs_two_pass": round((t_dec + t_u) / t_f, 3),
                       "cublas_bf16_us": round(t_c, 2),
                       # decode to HBM, then cuBLAS on dense bf16 weights (for int4 /
                       # fp8 this GEMM reads 2 B per weight: no cuBLAS kernel takes
                       # those codes with a bf16 X)
                       "two_pass_cublas_us": round(t_dec + t_c, 2),
                       "speedup_vs_two_pass_cublas": round((t_dec + t_c) / t_f, 3),
                       "status": int(st.item()),
                       "peak_source": peaks_src}
                print(json.dumps(rec), flush=True)
                del X, Y, Yu, ws
            del layers, Wbs, Wb, dec, dw
            torch.cuda.empty_cache()
    if not only or "llama8b_mlp" in only:
        sweep_batched(args, torch, ans, WL, device, stream, st, timed_graph)


def sweep_batched(args, torch, ans, WL, device, stream, st, timed_graph):
    """The Llama MLP's gate and up projections (same layout, same X): two
    ans_gemm calls against one ans_gemm_batched call; then the whole MLP
    (gate, up and the 4096 x 14336 down projection, mixed shapes): three calls
    against one batched launch.  Weights from HBM."""
    cfg = WL.CONFIGS["llama8b_mlp"]
    mats = []
    for mi in (0, 1, 2):
        d = WL.make_weights(cfg, mi)
        lay = ans.make_layout(cfg.dtype, d["N"], d["K"], cfg.tile_n, cfg.tile_k, args.state_bits)
        l0 = ans.CompressedLayer.from_weights(d["w"], lay, device=device)
        copies = [l0] + [ans.CompressedLayer(lay, l0.codebook, l0.h_stream, l0.h_offsets, l0.h_raw,
                                             device) for _ in range(3)]
        mats.append((lay, copies))
    lay = mats[0][0]
    for M in (1, 8, 16, 32):
        X = torch.from_numpy(WL.make_x(cfg, M, lay.K).view(np.int16)).to(device)
        Ys = [torch.empty(M, lay.N, dtype=torch.float32, device=device) for _ in range(2)]
        nb1 = ans.ans_gemm_workspace(lay, M, 0)
        ws1 = torch.zeros(max(nb1, 256), dtype=torch.uint8, device=device)
        jobs = [[(X, mats[j][1][c].tiles, None, Ys[j]) for j in range(2)] for c in range(4)]
        nb2 = ans.ans_gemm_batched_workspace(jobs[0], M, 0)
        ws2 = torch.zeros(max(nb2, 256), dtype=torch.uint8, device=device)
        two = [lambda c=c, j=j: ans.ans_gemm(X, M, mats[j][1][c].tiles, 0, None, 0, Ys[j], ws1, nb1, st)
               for c in range(4) for j in range(2)]
        one = [lambda c=c: ans.ans_gemm_batched(jobs[c], M, 0, 0, ws2, nb2, st) for c in range(4)]
        t2 = timed_graph(two, 20) * 2   # per pair of layers
        t1 = timed_graph(one, 20)
        rec = {"workload": "llama8b_mlp", "matrix": "gate+up", "N": 2 * lay.N, "K": lay.K, "M": M,
               "state_bits": args.state_bits, "two_ans_gemm_us": round(t2, 2),
               "ans_gemm_batched_us": round(t1, 2), "speedup": round(t2 / t1, 3),
               "effective_weight_GBps": round(2 * lay.N * lay.K * 2 / (t1 * 1e-6) / 1e9, 1),
               "status": int(st.item())}
        print(json.dumps(rec), flush=True)
    # the whole MLP in one launch: gate and up read X (M x 4096), down reads an
    # activation of M x 14336 (synthetic here)
    lay_d = mats[2][0]
    n_w = sum(m[0].N * m[0].K for m in mats)
    for M in (1, 16):
        X = torch.from_numpy(WL.make_x(cfg, M, lay.K).view(np.int16)).to(device)
        Hx = torch.from_numpy(WL.make_x(cfg, M, lay_d.K).view(np.int16)).to(device)
        Ys = [torch.empty(M, m[0].N, dtype=torch.float32, device=device) for m in mats]
        ins = [X, X, Hx]
        wss = []
        for j in range(3):
            nb = ans.ans_gemm_workspace(mats[j][0], M, 0)
            wss.append((torch.zeros(max(nb, 256), dtype=torch.uint8, device=device), nb))
        jobs = [[(ins[j], mats[j][1][c].tiles, None, Ys[j]) for j in range(3)] for c in range(4)]
        nb3 = ans.ans_gemm_batched_workspace(jobs[0], M, 0)
        ws3 = torch.zeros(max(nb3, 256), dtype=torch.uint8, device=device)
        three = [lambda c=c, j=j: ans.ans_gemm(ins[j], M, mats[j][1][c].tiles, 0, None, 0, Ys[j],
                                               wss[j][0], wss[j][1], st)
                 for c in range(4) for j in range(3)]
        one = [lambda c=c: ans.ans_gemm_batched(jobs[c], M, 0, 0, ws3, nb3, st) for c in range(4)]
        t3 = timed_graph(three, 20) * 3   # per MLP
        t1 = timed_graph(one, 20)
        rec = {"workload": "llama8b_mlp", "matrix": "gate+up+down", "weights": n_w, "M": M,
               "state_bits": args.state_bits, "three_ans_gemm_us": round(t3, 2),
               "ans_gemm_batched_us": round(t1, 2), "speedup": round(t3 / t1, 3),
               "effective_weight_GBps": round(n_w * 2 / (t1 * 1e-6) / 1e9, 1),
               "status": int(st.item())}
        print(json.dumps(rec), flush=True)


def oracle_rows_rate(O, cfg, d, lay, layer, X_h, budget_s, threads, max_rb=None):
    """Oracle decode of whole W row blocks plus the fp64 GEMM of their rows,
    until `budget_s` of CPU time is spent; returns (weights, seconds, blocks)."""
    N, K, M = lay.N, lay.K, X_h.shape[0]
    n_kt = K // lay.tile_k
    freq = layer.codebook.freq_array()
    rb_total = N // lay.tile_n
    if max_rb is not None:
        rb_total = min(rb_total, max_rb)
    if cfg.dtype == 1:
        out = np.zeros(N * K, np.uint16)
    else:
        out = np.zeros(int(N * K * NOMINAL[cfg.dtype]), np.uint8)
    done_rb, t_spent = 0, 0.0
    while done_rb < rb_total and t_spent < budget_s:
        t0 = time.perf_counter()
        st, _ = O.decode(cfg.dtype, layer.h_stream, layer.h_offsets, layer.h_raw, N, K,
                         lay.tile_n, lay.tile_k, freq, tile_begin=done_rb * n_kt,
                         tile_end=(done_rb + 1) * n_kt, out=out, threads=threads,
                         state_bits=lay.state_bits or 32)
        rows = np.arange(done_rb * lay.tile_n, (done_rb + 1) * lay.tile_n, dtype=np.uint32)
        O.gemm(cfg.dtype, X_h, M, K, out, N, cfg.scale_kind, d["scales"], cfg.group_k,
               rows=rows, threads=threads)
        t_spent += time.perf_counter() - t0
        done_rb += 1
    return done_rb * lay.tile_n * K, t_spent, done_rb


def cpu_baseline(cfg, d, lay, layer, X_h, budget_s=15.0, budget_1core_s=8.0):
    """The CPU oracle, as it stands, on the host cores (all of them, then one):
    decode of a sample of whole W row blocks plus the fp64 GEMM on their rows,
    scaled to the metric (effective weight GB/s)."""
    from oracle import oracle as O
    O.build()
    cores = os.cpu_count() or 1
    w_all, t_all, rb_all = oracle_rows_rate(O, cfg, d, lay, layer, X_h, budget_s, cores)
    w_one, t_one, rb_one = oracle_rows_rate(O, cfg, d, lay, layer, X_h, budget_1core_s, 1)
    M, K = X_h.shape
    nb = NOMINAL[cfg.dtype]
    return {"value": round(w_all * nb / t_all / 1e9, 4), "unit": "GB/s", "cores": cores,
            "kind": "oracle", "cpu_model": cpu_model(),
            "sample": f"{rb_all} of {lay.N // lay.tile_n} row blocks of {lay.tile_n} rows: "
                      f"oracle decode of their {rb_all * (K // lay.tile_k)} tiles + fp64 GEMM of "
                      f"their rows with X {M}x{K}, {cores} threads",
            "one_core": {"value": round(w_one * nb / t_one / 1e9, 4), "unit": "GB/s", "cores": 1,
                         "sample": f"{rb_one} row blocks, 1 thread"}}


def time_reference(args):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return None
    from oracle import oracle as O
    from rans_decode_gemm_b200 import workloads as WL
    O.build()
    cfg = WL.CONFIGS[WORKLOAD]
    d = WL.make_weights(cfg, 0)
    N, K, M = d["N"], d["K"], M_HEAD
    counts = O.histogram(cfg.dtype, d["w"], N * K)
    _, freq = O.normalize(counts)
    # the oracle codes only the row blocks the timed steps decode
    n_kt = K // cfg.tile_k
    rb_total = N // cfg.tile_n
    n_rb = min(rb_total, max(1, args.warmup + args.steps))
    rows_w = d["w"][:n_rb * cfg.tile_n * K]
    st, stream, offsets, raw = O.encode(cfg.dtype, rows_w, n_rb * cfg.tile_n, K, cfg.tile_n,
                                        cfg.tile_k, freq, state_bits=args.state_bits)
    X_h = WL.make_x(cfg, M, K)
    cores = os.cpu_count() or 1
    out = np.zeros(n_rb * cfg.tile_n * K, np.uint8)
    Nr = n_rb * cfg.tile_n

    def one(rb):
        O.decode(cfg.dtype, stream, offsets, raw, Nr, K, cfg.tile_n, cfg.tile_k, freq,
                 tile_begin=rb * n_kt, tile_end=(rb + 1) * n_kt, out=out, threads=cores,
                 state_bits=args.state_bits)
        rows = np.arange(rb * cfg.tile_n, (rb + 1) * cfg.tile_n, dtype=np.uint32)
        O.gemm(cfg.dtype, X_h, M, K, out, Nr, cfg.scale_kind, d["scales"][:Nr], cfg.group_k,
               rows=rows, threads=cores)

    for i in range(args.warmup):
        one(i % n_rb)
    t0 = time.perf_counter()
    for i in range(args.steps):
        one((args.warmup + i) % n_rb)
    dt = time.perf_counter() - t0
    per_rb_s = dt / max(1, args.steps)
    value = cfg.tile_n * K * NOMINAL[cfg.dtype] / per_rb_s / 1e9
    sample = (f"each step: oracle decode of one {cfg.tile_n}-row block ({n_kt} tiles) + fp64 "
              f"GEMM of its rows with X {M}x{K}, {cores} threads")
    return {"impl": "reference", "metric": METRIC,
            "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(per_rb_s * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": workload_name(WORKLOAD, args.state_bits, M),
                       "state_bits": args.state_bits, "M": M, "N": N, "K": K,
                       "global_batch": M * world, "parallelism": f"replicas x{world}",
                       "l2": "host memory (CPU oracle)"},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                             "kind": "oracle", "sample": sample, "cpu_model": cpu_model()},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    if args.sweep:
        sweep(args)
        return
    if args.impl == "reference":
        res = time_reference(args)
    else:
        res = time_ours(args)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
