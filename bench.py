"""Benchmark of the rotated low-bit linear layer on B200.

One step = one full layer call on one batch of synthetic tokens: the
rotate + quantise prologue with the low-rank down product, then the tcgen05
W4A4 GEMM with group-64 dequant, rank-32 branch and sigmoid gate epilogue
(the grouped Q|K|V|gate projection, M=4096 tokens, K=3072, N=4*3072).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --sweep small-m|stack|prologue|ffdown|kv4|nvfp4|qknorm|attn|svdquant|peaks
                                                            (one JSON line per case)

Sweeps: small-m (K = N = 3072 layer at 1..1024 tokens, W4A4 row / group-64 and
NVFP4, HBM roofline; --m-list and --formats restrict it), stack (the 28-block
stack of 224 linears), prologue (the activation prologues at the layer shapes,
HBM roofline), ffdown (the W8A8 ff.down layer with its gated residual), kv4
(the INT4 KV-cache codec, HBM roofline), nvfp4 (the NVFP4 variant at the
Q|K|V|gate shape against the FP4 dense peak), qknorm (Q/K RMSNorm + RoPE, HBM
roofline), attn (the INT8 attention and its operand preparation), svdquant
(the offline SVDQuant fit), peaks (measured INT8 / FP8 library GEMM ceilings).

Under torchrun each rank runs its own replica on its own batch (tokens are
independent; no collective on the data path), scaling is weak and the value
is the whole-job throughput over the slowest rank.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

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

WORKLOAD = "w4a4_qkvg"
METRIC = "W4A4 rotated linear TOPS & tokens/s at M=4096, % of B200 INT8 tensor peak"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def workload_desc(cfg):
    return (f"{WORKLOAD}: grouped Q|K|V|gate W4A4 projection, M={cfg['M']} tokens, K={cfg['K']}, "
            f"N={cfg['N']}, group-64 scales, rank-{cfg['rank']} bf16 low-rank branch, sigmoid on columns "
            f"[{cfg['gate_cols'][0]},{cfg['gate_cols'][1]})")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- CPU oracle leg
def oracle_sample(t, cfg, wq_qw_sw, rows):
    """The oracle's per-token path on `rows` (weights already quantised, as on the GPU side)."""
    from oracle import rbd_oracle as O
    qw, sw = wq_qw_sw
    x = t["x"][rows]
    qx, sx = O.rot_quant(x, 4, 256, 64)
    y = O.dequant(qx, sx, qw, sw, 64)
    ld = O.lowrank_down(x, t["l1"])
    return O.epilogue(y, None, ld, t["l2"], 1, cfg["gate_cols"])


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(t, cfg, target_s=10.0):
    """The oracle timed on a bounded sample of token rows sized to about `target_s` seconds."""
    from oracle import rbd_oracle as O
    wq, sw = O.quantize_weights(t["w"], 4, 256, 64)
    prep = (O.unpack_int4(wq), sw)
    t0 = time.perf_counter()
    oracle_sample(t, cfg, prep, np.arange(64))                  # warm, and size the sample
    per_row = (time.perf_counter() - t0) / 64
    rows_n = int(min(cfg["M"], max(64, round(target_s / per_row / 64) * 64)))
    rows = np.arange(rows_n)
    t0 = time.perf_counter()
    oracle_sample(t, cfg, prep, rows)
    dt = time.perf_counter() - t0
    tops = 2.0 * rows_n * cfg["N"] * cfg["K"] / dt / 1e12
    return {"value": tops, "unit": "TOPS", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{rows_n} of {cfg['M']} token rows of the same layer (per-token path: rotate, quantise, "
                      f"group-64 dequant GEMM, low-rank branch, sigmoid; weights quantised beforehand), "
                      f"{dt:.2f} s", "tokens_per_s": rows_n / dt, "seconds": dt}


def run_reference(args, cfg, t):
    """--impl reference: the CPU oracle, as it stands, on bounded samples of the workload."""
    from oracle import rbd_oracle as O
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wq, sw = O.quantize_weights(t["w"], 4, 256, 64)
    prep = (O.unpack_int4(wq), sw)
    rows_n = 256
    rows = np.arange(rows_n)
    for _ in range(args.warmup):
        oracle_sample(t, cfg, prep, rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample(t, cfg, prep, rows)
    dt = (time.perf_counter() - t0) / args.steps
    tops = 2.0 * rows_n * cfg["N"] * cfg["K"] / dt / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": tops, "unit": "TOPS", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(cfg), "sample_rows_per_step": rows_n},
            "cpu_baseline": {"value": tops, "unit": "TOPS", "cores": blas_threads(), "kind": "oracle",
                             "sample": f"{rows_n} token rows per step of the {cfg['M']}-token layer"},
            "e2e": {"value": tops, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "tokens_per_s": rows_n / dt}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- multi-rank host logic
def max_over_ranks(x: float, device=None) -> float:
    """The slowest rank's value: every rank calls this with its own number."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, steps: int, units_per_step: float, t_max: float) -> float:
    """Units all ranks processed divided by the slowest rank's time (weak scaling)."""
    return world * steps * units_per_step / t_max


# ----------------------------------------------------------------------------- GPU leg
def run_ours(args, cfg, t):
    import torch
    import torch.distributed as dist

    import rotated_bit_dit_b200 as R
    from rotated_bit_dit_b200 import _binding as B

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    R.load()

    def up(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    M, K, N, r = cfg["M"], cfg["K"], cfg["N"], cfg["rank"]
    layer = R.RotatedLowBitLinear(up(t["w"]), bits=4, scale_group=64, l1=up(t["l1"]), l2=up(t["l2"]),
                                  gate_mode=1, gate_cols=cfg["gate_cols"])
    x = up(t["x"])
    out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    codes, sx, ld = layer.buffers(M, dev)
    epi = B.make_epilogue(None, ld, layer.l2t, 1, cfg["gate_cols"])
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)   # > 126 MB L2

    def step(ev=None):
        if ev:
            ev[0].record()
        B.rbd_lowrank_fused(x, codes, sx, layer.l1t, ld, 4, 256, 64, code_format=layer.code_format)
        if ev:
            ev[1].record()
        B.rbd_w4a4_linear(codes, sx, layer.wq, layer.sw, out, 64, epi, code_format=layer.code_format)
        if ev:
            ev[2].record()

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    assert R.rbd_check() == 0
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.zero_()
            step(evs[i])
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    status = R.rbd_check()
    if status != 0:
        raise RuntimeError(f"device status {status}")
    pro = [e[0].elapsed_time(e[1]) for e in evs]
    gemm = [e[1].elapsed_time(e[2]) for e in evs]
    tot = [e[0].elapsed_time(e[2]) for e in evs]
    t_rank = sum(tot) / 1e3           # seconds over K steps, this rank
    t_max = max_over_ranks(t_rank, dev)
    ops_step = 2.0 * M * N * K
    value = whole_job_rate(world, args.steps, ops_step, t_max) / 1e12
    tokens_s = whole_job_rate(world, args.steps, M, t_max)

    # ---- end to end through the public layer call with host buffers: forward_host streams
    # 1024-token slices through two CUDA streams so the copies overlap the kernels
    xh = torch.from_numpy(np.ascontiguousarray(t["x"]).view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for _ in range(2):
        layer.forward_host(xh, yh)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        e2e_ev[i][0].record()
        layer.forward_host(xh, yh)
        e2e_ev[i][1].record()
    torch.cuda.synchronize()
    e2e_t = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in e2e_ev) / 1e3, dev)
    e2e_value = whole_job_rate(world, args.steps, ops_step, e2e_t) / 1e12
    # the end-to-end bound: the pinned-memory copy rates of this machine, one direction at a time
    # (a step needs X in and Y out; with the copies overlapped the slower direction bounds it)
    def copy_rate(dst, src):
        for _ in range(2):
            dst.copy_(src, non_blocking=True)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(5):
            dst.copy_(src, non_blocking=True)
        b.record()
        torch.cuda.synchronize()
        return 5 * src.numel() * src.element_size() / (a.elapsed_time(b) / 1e3) / 1e9
    yd_probe = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    xd_probe = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    d2h_gbs = copy_rate(yh, yd_probe)
    h2d_gbs = copy_rate(xd_probe, xh)
    del yd_probe, xd_probe
    e2e_bound_s = max(yh.numel() * 2 / (d2h_gbs * 1e9), xh.numel() * 2 / (h2d_gbs * 1e9), t_rank / args.steps)

    if rank == 0:
        peaks, src = load_peaks()
        int8_peak, int8_src = int8_peak_tops(peaks, src)
        gemm_s = statistics.mean(gemm) / 1e3
        pro_s = statistics.mean(pro) / 1e3
        achieved = ops_step / gemm_s / 1e12
        pro_bytes = M * K * 2 + M * K + M * (K // 64) * 4 + K * r * 2 + M * r * 2
        traffic = _profile_traffic()
        line = {
            "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": t_max / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": workload_desc(cfg), "M": M, "K": K, "N": N, "rank": r, "scale_group": 64,
                       "bits": 4, "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "flushed (256 MB write) before every timed step"},
            "tokens_per_s": tokens_s,
            "pct_int8_peak": 100.0 * value / world / int8_peak,
            "kernels_ms": {"rot_quant_lowrank": statistics.mean(pro), "w4a4_gemm": statistics.mean(gemm)},
            "roofline": {"bound": "tensor", "kernel": "lowbit_gemm_kernel<W4,G64,LR>", "achieved": achieved,
                         "peak": int8_peak, "unit": "TOPS", "frac": achieved / int8_peak,
                         "peak_source": int8_src, "frac_of_datasheet_4500": achieved / 4500.0,
                         "traffic": traffic,
                         "algorithmic": "2*M*N*K int ops per launch"},
            "prologue_roofline": {"bound": "hbm", "achieved": pro_bytes / pro_s / 1e9, "peak": peaks["hbm_gbs"],
                                  "unit": "GB/s", "frac": pro_bytes / pro_s / 1e9 / peaks["hbm_gbs"],
                                  "algorithmic_bytes": pro_bytes},
            "e2e": {"value": e2e_value, "unit": "TOPS", "h2d_bytes_per_step": int(xh.numel() * 2),
                    "d2h_bytes_per_step": int(yh.numel() * 2),
                    "call": "RotatedLowBitLinear.forward_host: pinned host X in, Y out, 1024-token slices on "
                            "two streams (copies overlap the kernels)",
                    "bound": {"d2h_gbs": d2h_gbs, "h2d_gbs": h2d_gbs,
                              "value": ops_step / e2e_bound_s / 1e12,
                              "frac": e2e_value / world / (ops_step / e2e_bound_s / 1e12),
                              "what": "slowest of: Y device->host at the measured pinned copy rate, X "
                                      "host->device likewise, the device step; all perfectly overlapped"}},
            "gpu_launches": 2 * args.steps,   # fused prologue + GEMM per step
            "clocks": clk.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(t, cfg)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


GEMM_SOURCES = [os.path.join(ROOT, "rotated_bit_dit_b200", "csrc", f)
                for f in ("rbd_gemm.cu", "rbd_common.cuh", "rbd_internal.cuh")]
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "lowbit_gemm_w4a4_qkvg.json")


def gemm_source_hash():
    """First 16 hex digits of the sha256 over the sources the GEMM kernel is built from."""
    import hashlib
    h = hashlib.sha256()
    for p in GEMM_SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# ----------------------------------------------------------------------------- tensor ceilings
PEAKS_FILE = os.path.join(ROOT, "profiles", "peaks.json")


def run_peaks(args):
    """Dense tensor-core ceilings of library GEMMs on this GPU, for the roofline denominators:
    INT8 (torch._int_mm, int32 out) and FP8 E4M3 (torch._scaled_mm, bf16 out) at 8192^3, each the
    best of 10 single calls (burst) and the mean over a 4 s back-to-back loop (sustained), with
    the SM clocks sampled during the loops.  Prints one JSON line (kept as profiles/peaks.json)."""
    import torch
    dev = torch.device("cuda", 0)
    n = 8192
    ops = 2.0 * n ** 3
    out = {"what": "dense GEMM ceilings, 8192^3, CUDA events", "gpu": torch.cuda.get_device_name(dev),
           "torch": torch.__version__}

    def measure(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(10):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            best = min(best, a.elapsed_time(b) / 1e3)
        with ClockSampler(0) as clk:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            calls = max(8, int(4.0 / best))
            a.record()
            for _ in range(calls):
                fn()
            b.record()
            b.synchronize()
        sus = a.elapsed_time(b) / 1e3 / calls
        return {"burst_tops": ops / best / 1e12, "sustained_tops": ops / sus / 1e12, "clocks": clk.summary()}

    g = torch.Generator(device=dev).manual_seed(0)
    a8 = torch.randint(-128, 128, (n, n), dtype=torch.int8, device=dev, generator=g)
    b8 = torch.randint(-128, 128, (n, n), dtype=torch.int8, device=dev, generator=g).t()
    try:
        out["int8"] = measure(lambda: torch._int_mm(a8, b8))
        out["int8"]["call"] = "torch._int_mm int8 x int8 -> int32"
    except RuntimeError as e:
        out["int8"] = {"unavailable": str(e).splitlines()[0]}
    del a8, b8
    af = torch.randn((n, n), device=dev, generator=g).to(torch.float8_e4m3fn)
    bf = torch.randn((n, n), device=dev, generator=g).to(torch.float8_e4m3fn).t()
    one = torch.ones((), dtype=torch.float32, device=dev)
    try:
        out["fp8_e4m3"] = measure(lambda: torch._scaled_mm(af, bf, one, one, out_dtype=torch.bfloat16))
        out["fp8_e4m3"]["call"] = "torch._scaled_mm e4m3 x e4m3 -> bf16, tensor scales"
    except RuntimeError as e:
        out["fp8_e4m3"] = {"unavailable": str(e).splitlines()[0]}
    print(json.dumps(out), flush=True)


def load_tensor_peaks():
    """Measured INT8 / FP8 dense ceilings (profiles/peaks.json) or None when not measured."""
    if not os.path.exists(PEAKS_FILE):
        return None
    with open(PEAKS_FILE) as f:
        return json.load(f)


def int8_peak_tops(peaks, src, sustained=False):
    """INT8 dense roofline peak: the measured library INT8 ceiling when profiles/peaks.json holds
    one (burst for a kernel timed alone, sustained for one timed inside a long run), else the
    bf16 peak of MEASURED_PEAKS.json times the nominal 2x ratio."""
    tp = load_tensor_peaks()
    key = "sustained_tops" if sustained else "burst_tops"
    if tp and key in tp.get("int8", {}):
        return tp["int8"][key], f"measured INT8 GEMM ceiling (torch._int_mm 8192^3, {key[:-5]}), profiles/peaks.json"
    bf = peaks["bf16_tflops_sustained" if sustained and "bf16_tflops_sustained" in peaks else "bf16_tflops"]
    return 2.0 * bf, f"{src} bf16 dense {bf} TFLOP/s x 2 (nominal INT8:BF16 ratio)"


# ----------------------------------------------------------------------------- small-M sweep
def run_small_m_sweep(args):
    """K = N = 3072 layer at small token counts (HBM-bound): W4A4 rotated per-row and the NVFP4
    variant.  Each timed call is a full layer (prologue + GEMM); 128 calls on 128 distinct weight
    copies (several times L2) are captured in one CUDA graph, so weights stream from HBM and launch
    gaps do not count.  One JSON line per (format, M)."""
    import torch

    import rotated_bit_dit_b200 as R
    from rotated_bit_dit_b200 import _binding as B
    from rotated_bit_dit_b200 import inputs as I

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    R.load()
    K = N = 3072
    copies = 128
    peaks, src = load_peaks()
    wb = I.gaussian_bf16(1, (N, K), 0.02)
    w = torch.from_numpy(np.ascontiguousarray(wb).view(np.int16)).view(torch.bfloat16).to(dev)
    # W4A4 per-row weights, then NVFP4 weights, each replicated into `copies` distinct buffers
    wq4 = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    sw4 = torch.empty((N,), dtype=torch.float32, device=dev)
    B.rbd_pack_weights_int4(w, wq4, sw4, 256, 0)
    wq4s = [wq4.clone() for _ in range(copies)]
    sw4s = [sw4.clone() for _ in range(copies)]
    wqf = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    wbf = torch.empty((B.rbd_nvfp4_scale_bytes(N, K),), dtype=torch.uint8, device=dev)
    wgf = torch.empty((1,), dtype=torch.float32, device=dev)
    work = torch.empty((1,), dtype=torch.int32, device=dev)
    B.rbd_nvfp4_quant(w, wqf, wbf, wgf, work, 256)
    wqfs = [wqf.clone() for _ in range(copies)]
    wbfs = [wbf.clone() for _ in range(copies)]
    torch.cuda.synchronize()
    # group-64 weights (the Q|K|V|gate layer's scale layout) for the E4M3-code path
    wq4g = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    sw4g = torch.empty((N, K // 64), dtype=torch.float32, device=dev)
    B.rbd_pack_weights_int4(w, wq4g, sw4g, 256, 64)
    wq4gs = [wq4g.clone() for _ in range(copies)]
    sw4gs = [sw4g.clone() for _ in range(copies)]
    torch.cuda.synchronize()

    def graph_time(fn):
        """Median device time per call of a CUDA graph of `copies` calls fn(i)."""
        for i in range(3):
            fn(i)
        torch.cuda.synchronize()
        assert R.rbd_check() == 0
        stream = torch.cuda.Stream(device=dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for i in range(copies):
                    fn(i)
        for _ in range(max(args.warmup, 3)):
            g.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(args.steps):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) / 1e3 / copies)
        assert R.rbd_check() == 0
        del g
        return statistics.median(ts)

    fmts = args.formats.split(",") if args.formats else ["w4a4", "w4a4_g64", "nvfp4"]
    mlist = [int(v) for v in args.m_list.split(",")] if args.m_list else [1, 16, 64, 256, 1024]
    for fmt in fmts:
        for M in mlist:
            xb = I.gaussian_bf16(2 + M, (M, K), 1.0, 0.005, 30.0)
            x = torch.from_numpy(np.ascontiguousarray(xb).view(np.int16)).view(torch.bfloat16).to(dev)
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            if fmt in ("w4a4", "w4a4_g64"):
                g64 = fmt == "w4a4_g64"
                sg = 64 if g64 else 0
                cf = B.CODES_E4M3 if g64 else B.CODES_INT8
                codes = torch.empty((M, K), dtype=torch.int8, device=dev)
                sx = torch.empty((M, K // 64) if g64 else (M,), dtype=torch.float32, device=dev)
                wl, sl = (wq4gs, sw4gs) if g64 else (wq4s, sw4s)

                def prologue(i):
                    B.rbd_rot_quant_act(x, codes, sx, 4, 256, sg, code_format=cf)

                def gemm(i):
                    B.rbd_w4a4_linear(codes, sx, wl[i], sl[i], y, sg, None, code_format=cf)
                wbytes = N * K // 2 + N * 4 * (K // 64 if g64 else 1)
                gbytes = wbytes + M * (K + 4 * (K // 64 if g64 else 1) + 2 * N)   # GEMM alone
                abytes = M * (2 * K + K + 4 * (K // 64 if g64 else 1) + 2 * N)
            else:
                xq = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
                xbs = torch.empty((B.rbd_nvfp4_scale_bytes(M, K),), dtype=torch.uint8, device=dev)
                xgs = torch.empty((1,), dtype=torch.float32, device=dev)

                def prologue(i):
                    B.rbd_nvfp4_quant(x, xq, xbs, xgs, work, 256)

                def gemm(i):
                    B.rbd_nvfp4_linear(xq, xbs, xgs, wqfs[i], wbfs[i], wgf, y, None)
                wbytes = N * K // 2 + N * K // 16
                gbytes = wbytes + M * (K // 2 + K // 16 + 2 * N)
                abytes = M * (2 * K + 2 * K + K // 2 + K // 16 + 2 * N)   # X read twice (two passes)

            def layer(i):
                prologue(i)
                gemm(i)
            t = graph_time(layer)
            tg = graph_time(gemm)
            tp = graph_time(prologue)
            gbs = (wbytes + abytes) / t / 1e9
            print(json.dumps({
                "sweep": "small-m", "format": fmt, "M": M, "K": K, "N": N, "us_per_layer": t * 1e6,
                "tokens_per_s": M / t, "tops": 2.0 * M * N * K / t / 1e12, "hbm_gbs": gbs,
                "hbm_frac": gbs / peaks["hbm_gbs"], "peak_source": f"{src} copy {peaks['hbm_gbs']} GB/s",
                "algorithmic_bytes": wbytes + abytes,
                "gemm_us": tg * 1e6, "gemm_hbm_frac": gbytes / tg / 1e9 / peaks["hbm_gbs"],
                "prologue_us": tp * 1e6,
                "timing": f"median of {args.steps} replays of a graph of {copies} calls on distinct weight "
                          "copies (layer = prologue + GEMM; GEMM and prologue also timed alone)"}),
                flush=True)


# ----------------------------------------------------------------------------- ff.down layer
def run_ffdown_sweep(args):
    """The W8A8 ff.down layer (cfg2: M = 4096, K = 12288, N = 3072, per-row INT8, group-256
    rotation, gated residual): the rotate/quantise prologue and the GEMM (with the gated-residual
    epilogue) timed apart and together, each after a 256 MB L2 flush, CUDA events on the stream.
    The GEMM against the measured INT8 ceiling; the prologue against HBM."""
    import torch

    import rotated_bit_dit_b200 as R
    from rotated_bit_dit_b200 import _binding as B
    from rotated_bit_dit_b200 import inputs as I

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    R.load()
    cfg = I.CONFIGS["w8a8_ffdown"]
    t = I.make_layer_inputs(cfg, seed=0)
    M, K, N = cfg["M"], cfg["K"], cfg["N"]
    up = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    x, w, res, gate = up(t["x"]), up(t["w"]), up(t["residual"]), up(t["gate"])
    w8 = torch.empty((N, K), dtype=torch.int8, device=dev)
    sw = torch.empty((N,), dtype=torch.float32, device=dev)
    B.rbd_pack_weights_int8(w, w8, sw, 256, 0)
    codes = torch.empty((M, K), dtype=torch.int8, device=dev)
    sx = torch.empty((M,), dtype=torch.float32, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    epi = B.Epilogue(gate_mode=2, gate=gate.data_ptr(), residual=res.data_ptr(), ldr=N)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    peaks, src = load_peaks()
    int8_peak, int8_src = int8_peak_tops(peaks, src)
    pro = lambda: B.rbd_rot_quant_act(x, codes, sx, 8, 256, 0)
    gemm = lambda: B.rbd_w8a8_linear(codes, sx, w8, sw, y, 0, epi)

    def layer():
        pro()
        gemm()

    def timed(fn):
        for _ in range(max(args.warmup, 3)):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        assert R.rbd_check() == 0
        ts = []
        for _ in range(args.steps):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) / 1e3)
        assert R.rbd_check() == 0
        return statistics.median(ts)

    with ClockSampler(dev.index) as clk:
        tp, tg, tl = timed(pro), timed(gemm), timed(layer)
    ops = 2.0 * M * N * K
    pro_bytes = M * K * 2 + M * K + M * 4
    print(json.dumps({
        "sweep": "ffdown", "M": M, "K": K, "N": N, "prologue_us": tp * 1e6, "gemm_us": tg * 1e6,
        "layer_us": tl * 1e6, "gemm_tops": ops / tg / 1e12, "gemm_frac_int8": ops / tg / 1e12 / int8_peak,
        "layer_tops": ops / tl / 1e12, "prologue_hbm_frac": pro_bytes / tp / 1e9 / peaks["hbm_gbs"],
        "int8_peak_source": int8_src, "clocks": clk.summary(),
        "timing": f"median of {args.steps} calls each, every call after a 256 MB L2 flush"}), flush=True)


# ----------------------------------------------------------------------------- prologue sweep
def run_prologue_sweep(args):
    """The memory-bound activation prologues at the layer shapes: rotate/quantise, the normalising
    prologue (RMSNorm + modulation ahead of it) and the single-pass low-rank prologue.  Each timed
    call follows a 256 MB L2 flush; CUDA events on the launching stream.  One JSON line per case,
    achieved HBM bandwidth from the algorithmic bytes (read X once, write codes and scales)."""
    import torch

    import rotated_bit_dit_b200 as R
    from rotated_bit_dit_b200 import _binding as B
    from rotated_bit_dit_b200 import inputs as I

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    R.load()
    peaks, src = load_peaks()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def up(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    shapes = (("w4a4_qkvg input", 4096, 3072, 4, 64), ("w8a8_ffdown input", 4096, 12288, 8, 0),
              ("stack mlp input", 16384, 3072, 4, 0))
    for name, M, K, bits, sg in shapes:
        x = up(I.gaussian_bf16(3, (M, K), 1.0, 0.005, 30.0))
        gamma = up(I.f32_to_bf16_bits(1.0 + 0.1 * np.random.default_rng(4).standard_normal(K).astype(np.float32)))
        shift, scale = up(I.gaussian_bf16(5, (K,), 0.5)), up(I.gaussian_bf16(6, (K,), 0.3))
        codes = torch.empty((M, K), dtype=torch.int8, device=dev)
        sx = torch.empty((M, K // 64) if sg else (M,), dtype=torch.float32, device=dev)
        r = 32
        l1t = up(I.gaussian_bf16(7, (r, K), 0.01))
        ld = torch.empty((M, r), dtype=torch.bfloat16, device=dev)
        base = M * K * 2 + M * K + (M * (K // 64) if sg else M) * 4
        cf = B.CODES_E4M3 if (bits == 4 and sg == 64) else B.CODES_INT8   # as the layer stores them
        cases = [("rot_quant", lambda: B.rbd_rot_quant_act(x, codes, sx, bits, 256, sg, code_format=cf), base),
                 ("norm_rot_quant", lambda: B.rbd_norm_rot_quant_act(x, codes, sx, gamma, shift, scale, 1e-6,
                                                                     bits, 256, sg, code_format=cf),
                  base + 3 * K * 2)]
        if sg == 64:
            cases.append(("rot_quant_lowrank", lambda: B.rbd_lowrank_fused(x, codes, sx, l1t, ld, bits, 256, sg,
                                                                           code_format=cf),
                          base + M * r * 2 + r * K * 2))
        for cname, fn, nbytes in cases:
            for _ in range(max(args.warmup, 3)):
                flush.zero_()
                fn()
            torch.cuda.synchronize()
            assert R.rbd_check() == 0
            ts = []
            for _ in range(args.steps):
                flush.zero_()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record()
                fn()
                b.record()
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b) / 1e3)
            assert R.rbd_check() == 0
            t = statistics.median(ts)
            gbs = nbytes / t / 1e9
            print(json.dumps({
                "sweep": "prologue", "call": cname, "shape": name, "M": M, "K": K, "bits": bits,
                "scale_group": sg, "us": t * 1e6, "hbm_gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"],
                "peak_source": f"{src} copy {peaks['hbm_gbs']} GB/s", "algorithmic_bytes": nbytes,
                "timing": f"median of {args.steps} calls, each after a 256 MB L2 flush"}), flush=True)


# ----------------------------------------------------------------------------- KV-cache codec
def run_kv4_sweep(args):
    """INT4 KV-cache codec at 16384 tokens x 40 heads x 128 channels (a 168 MB bf16 slice, beyond L2):
    encode (slice write) and decode (slice read) for 3, 6 and 12 groups per head.  Each timed call
    follows a 256 MB L2 flush; bytes = bf16 slice + codes + scales."""
    import torch

    import rotated_bit_dit_b200 as R
    from rotated_bit_dit_b200 import _binding as B
    from rotated_bit_dit_b200 import inputs as I

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    R.load()
    peaks, src = load_peaks()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    T, H = 16384, 40
    x = torch.from_numpy(np.ascontiguousarray(I.gaussian_bf16(9, (T, H * 128), 1.0, 0.01, 20.0)).view(np.int16))
    x = x.view(torch.bfloat16).to(dev)
    y = torch.empty_like(x)
    for n in (1, 2, 4):
        codes = torch.empty((T, H, 64), dtype=torch.uint8, device=dev)
        scales = torch.empty((T, H, 3 * n), dtype=torch.float32, device=dev)
        nbytes = T * H * (256 + 64 + 12 * n)
        for op, fn in (("encode", lambda: B.rbd_kv4_encode(x, codes, scales, n)),
                       ("decode", lambda: B.rbd_kv4_decode(codes, scales, y, n))):
            for _ in range(max(args.warmup, 3)):
                flush.zero_()
                fn()
            torch.cuda.synchronize()
            assert R.rbd_check() == 0
            ts = []
            for _ in range(args.steps):
                flush.zero_()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record()
                fn()
                b.record()
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b) / 1e3)
            assert R.rbd_check() == 0
            t = statistics.median(ts)
            gbs = nbytes / t / 1e9
            print(json.dumps({
                "sweep": "kv4", "op": op, "tokens": T, "heads": H, "groups_per_head": 3 * n, "us": t * 1e6,
                "hbm_gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"], "peak_source": f"{src} copy {peaks['hbm_gbs']} GB/s",
                "algorithmic_bytes": nbytes, "timing": f"median of {args.steps} calls, each after a 256 MB L2 flush"}),
                flush=True)


# ----------------------------------------------------------------------------- Q/K RMSNorm + RoPE
def run_qknorm_sweep(args):
    """Q/K RMSNorm + RoPE at 16384 tokens x 24 heads x 128 channels (a 2048 x 2048 image's latent
    with the 3072-wide model): a contiguous Q [T, 3072], and Q turned in place inside the fused
    Q|K|V|gate GEMM output [T, 12288].  The rotary tables are built once, outside the timed calls.
    Each timed call follows a 256 MB L2 flush; bytes = heads read + written, cos / sin tables, gamma."""
    import torch

    import rotated_bit_dit_b200 as R
    from rotated_bit_dit_b200 import _binding as B
    from rotated_bit_dit_b200 import inputs as I

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    R.load()
    peaks, src = load_peaks()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    T, H = 16384, 24
    pos = torch.from_numpy(I.video_positions(1, 128, 128)).to(dev)
    cos = torch.empty((T, 64), dtype=torch.float32, device=dev)
    sin = torch.empty((T, 64), dtype=torch.float32, device=dev)
    B.rbd_rope_tables(pos, cos, sin)
    gamma = torch.from_numpy(I.f32_to_bf16_bits((1.0 + 0.1 * I.normal(12, 128)).astype(np.float32)).view(np.int16))
    gamma = gamma.view(torch.bfloat16).to(dev)
    q = torch.from_numpy(np.ascontiguousarray(I.gaussian_bf16(10, (T, H * 128), 1.0, 0.01, 20.0)).view(np.int16))
    q = q.view(torch.bfloat16).to(dev)
    fused = torch.zeros((T, 4 * H * 128), dtype=torch.bfloat16, device=dev)   # Q | K | V | gate
    fused[:, :H * 128] = q
    qo = torch.empty_like(q)
    nbytes = T * H * 512 + T * 512 + 256
    for case, fn in (("contiguous", lambda: B.rbd_qk_norm_rope(q, cos, sin, qo, gamma, 1e-6)),
                     ("in place, fused GEMM output", lambda: B.rbd_qk_norm_rope(fused[:, :H * 128], cos, sin,
                                                                                 fused[:, :H * 128], gamma, 1e-6))):
        for _ in range(max(args.warmup, 3)):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        assert R.rbd_check() == 0
        ts = []
        for _ in range(args.steps):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) / 1e3)
        assert R.rbd_check() == 0
        t = statistics.median(ts)
        gbs = nbytes / t / 1e9
        print(json.dumps({
            "sweep": "qknorm", "case": case, "tokens": T, "heads": H, "us": t * 1e6,
            "hbm_gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"], "peak_source": f"{src} copy {peaks['hbm_gbs']} GB/s",
            "algorithmic_bytes": nbytes, "timing": f"median of {args.steps} calls, each after a 256 MB L2 flush"}),
            flush=True)


# ----------------------------------------------------------------------------- INT8 attention
def run_attn_sweep(args):
    """INT8 attention (SageAttention v1 scheme) at 16384 tokens x 24 heads x 128 channels (a 2048 x 2048
    image's latent with the 3072-wide model), self-attention on Q and K after the library's Q/K
    RMSNorm + RoPE step (as attention receives them in the block): the preparation call (key smoothing,
    INT8 codes and scales, fp16 V^T) and the attention call timed separately.  Work = Q.K^T
    2 T^2 128 INT8 ops + P.V 2 T^2 128 fp16 FLOPs per head; the tensor floor is the INT8 part at the
    measured INT8 ceiling plus the fp16 part at the measured bf16 dense peak (the same rate)."""
    import torch

    import rotated_bit_dit_b200 as R
    from rotated_bit_dit_b200 import _binding as B
    from rotated_bit_dit_b200 import inputs as I

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    R.load()
    peaks, src = load_peaks()
    int8_peak, int8_src = int8_peak_tops(peaks, src)
    T, H = 16384, 24

    def up(seed):
        a = I.gaussian_bf16(seed, (T, H * 128), 1.0, 0.02, 20.0)
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    q, k, v = up(20), up(21), up(22)
    # Q and K as attention receives them: after the Q/K RMSNorm + RoPE step (one 128 x 128 frame)
    pos = torch.from_numpy(I.video_positions(1, 128, 128)).to(dev)
    cos = torch.empty((T, 64), dtype=torch.float32, device=dev)
    sin = torch.empty((T, 64), dtype=torch.float32, device=dev)
    B.rbd_rope_tables(pos, cos, sin)
    B.rbd_qk_norm_rope(q, cos, sin, q, None, 1e-6)
    B.rbd_qk_norm_rope(k, cos, sin, k, None, 1e-6)
    qc, sq, kc, sk, vt = R.attention_operands(q, k, v, H)
    work = torch.empty((B.rbd_attn_workspace_bytes(T, H),), dtype=torch.uint8, device=dev)
    o = torch.empty((T, H * 128), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    ops_qk = 2.0 * T * T * 128 * H
    floor_s = ops_qk / (int8_peak * 1e12) + ops_qk / (peaks["bf16_tflops"] * 1e12)
    prep_bytes = T * H * 128 * 2 * 3 + 2 * T * H * 128 + 2 * T * H * 4 + T * H * 128 * 2
    for case, fn in (("prepare", lambda: B.rbd_attn_quant(q, k, v, H, qc, sq, kc, sk, vt, work)),
                     ("attention", lambda: B.rbd_attn_int8(qc, sq, kc, sk, vt, o))):
        for _ in range(max(args.warmup, 3)):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        assert R.rbd_check() == 0
        ts = []
        for _ in range(args.steps):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) / 1e3)
        assert R.rbd_check() == 0
        t = statistics.median(ts)
        line = {"sweep": "attn", "case": case, "tokens": T, "heads": H, "us": t * 1e6,
                "timing": f"median of {args.steps} calls, each after a 256 MB L2 flush"}
        if case == "attention":
            line.update({"tops": 2 * ops_qk / t / 1e12, "tensor_floor_us": floor_s * 1e6,
                         "frac_of_tensor_floor": floor_s / t,
                         "peaks": f"INT8 {int8_peak:.0f} TOPS ({int8_src}); fp16 = {src} bf16 dense "
                                  f"{peaks['bf16_tflops']} TFLOP/s"})
        else:
            gbs = prep_bytes / t / 1e9
            line.update({"hbm_gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes": prep_bytes})
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- offline SVDQuant fit
def run_svdquant_sweep(args):
    """The offline SVDQuant fit (rbd_svdquant_fit) of the Q|K|V|gate weight (N = 12288, K = 3072),
    INT4 group-64, rank 32, oversampling 8, three iterates; wall time of the synchronous call (the
    fit is offline: float64 products on the device, QR / SVD on the host)."""
    import torch

    import rotated_bit_dit_b200 as R
    from rotated_bit_dit_b200 import inputs as I

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    R.load()
    N, K, rank, iters = 12288, 3072, 32, 3
    w = torch.from_numpy(np.ascontiguousarray(I.gaussian_bf16(30, (N, K), 0.02)).view(np.int16))
    w = w.view(torch.bfloat16).to(dev)
    om = np.random.default_rng(31).standard_normal((iters, K, rank + 8))
    R.rbd_svdquant_fit(w, rank, om[:1], 4, 256, 64)        # warm-up (one iterate)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    out = R.rbd_svdquant_fit(w, rank, om, 4, 256, 64)
    dt = time.perf_counter() - t0
    assert R.rbd_check() == 0
    print(json.dumps({"sweep": "svdquant", "N": N, "K": K, "rank": rank, "oversample": 8, "iters": iters,
                      "seconds": dt, "errs": out["errs"].tolist(), "best": out["best"],
                      "timing": "wall time of one synchronous call after a one-iterate warm-up"}), flush=True)


# ----------------------------------------------------------------------------- NVFP4 at the layer shape
def run_nvfp4_sweep(args):
    """The NVFP4 variant at the grouped Q|K|V|gate shape (K = 3072, N = 12288, rank-32 branch, sigmoid
    gate) and 1024 / 4096 tokens, compute-bound: the FP4 GEMM against the FP4 dense peak (measured
    bf16 x 4, the nominal FP4:BF16 ratio), plus the whole layer (two-pass quantiser + GEMM).  Each
    timed call follows a 256 MB L2 flush."""
    import torch

    import rotated_bit_dit_b200 as R
    from rotated_bit_dit_b200 import _binding as B
    from rotated_bit_dit_b200 import inputs as I

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    R.load()
    peaks, src = load_peaks()
    fp4_peak = 4.0 * peaks["bf16_tflops"]
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def up(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    K, N, r = 3072, 12288, 32
    w = up(I.gaussian_bf16(1, (N, K), 0.02))
    wq = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    wbs = torch.empty((B.rbd_nvfp4_scale_bytes(N, K),), dtype=torch.uint8, device=dev)
    wgs = torch.empty((1,), dtype=torch.float32, device=dev)
    work = torch.empty((1,), dtype=torch.int32, device=dev)
    B.rbd_nvfp4_quant(w, wq, wbs, wgs, work, 256)
    l1t = up(I.gaussian_bf16(2, (r, K), 0.01))
    l2t = up(I.gaussian_bf16(3, (N, r), 0.01))
    for M in (1024, 4096):
        x = up(I.gaussian_bf16(4, (M, K), 1.0, 0.005, 30.0))
        xq = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
        xbs = torch.empty((B.rbd_nvfp4_scale_bytes(M, K),), dtype=torch.uint8, device=dev)
        xgs = torch.empty((1,), dtype=torch.float32, device=dev)
        ld = torch.empty((M, r), dtype=torch.bfloat16, device=dev)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        epi = B.make_epilogue(None, ld, l2t, 1, (3 * 3072, 4 * 3072))

        def prologue():
            B.rbd_nvfp4_quant(x, xq, xbs, xgs, work, 256)
            B.rbd_lowrank_down(x, l1t, ld)

        def gemm():
            B.rbd_nvfp4_linear(xq, xbs, xgs, wq, wbs, wgs, y, epi)

        prologue()
        gemm()
        torch.cuda.synchronize()
        assert R.rbd_check() == 0
        tg, tl = [], []
        for i in range(max(args.warmup, 3) + args.steps):
            flush.zero_()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            ev[0].record()
            prologue()
            ev[1].record()
            gemm()
            ev[2].record()
            torch.cuda.synchronize()
            if i >= max(args.warmup, 3):
                tg.append(ev[1].elapsed_time(ev[2]) / 1e3)
                tl.append(ev[0].elapsed_time(ev[2]) / 1e3)
        assert R.rbd_check() == 0
        g, lay = statistics.median(tg), statistics.median(tl)
        ops = 2.0 * M * N * K
        print(json.dumps({
            "sweep": "nvfp4", "M": M, "K": K, "N": N, "rank": r, "gemm_us": g * 1e6, "layer_us": lay * 1e6,
            "gemm_tflops": ops / g / 1e12, "layer_tflops": ops / lay / 1e12,
            "frac_fp4_peak": ops / g / 1e12 / fp4_peak,
            "peak_source": f"{src} bf16 dense {peaks['bf16_tflops']} TFLOP/s x 4 (nominal FP4:BF16 ratio)",
            "timing": f"median of {args.steps} calls, each after a 256 MB L2 flush"}), flush=True)


# ----------------------------------------------------------------------------- 28-block stack
STACK_LAYERS = (("wq", 3072, 3072), ("wk", 3072, 3072), ("wv", 3072, 3072), ("gate", 3072, 3072),
                ("wo", 3072, 3072), ("mlp.gate", 3072, 12288), ("mlp.up", 3072, 12288), ("mlp.down", 12288, 3072))


def stack_layer_is_int8(block: int, name: str) -> bool:
    """The 96 protected INT8 layers: every wk and wv, wo of blocks 0-26, mlp.down of blocks 15-27."""
    return name in ("wk", "wv") or (name == "wo" and block <= 26) or (name == "mlp.down" and block >= 15)


def run_stack(args):
    """Timing of the full 28-block linear stack at M = 16384 tokens: 224 rotated low-bit linears
    (128 W4A4 per-row, 96 W8A8), each with its own weights and its own rotate/quantise prologue.
    Inputs are synthetic (N(0,1) with 0.5% outlier channels x30), not chained through the blocks."""
    import torch

    import rotated_bit_dit_b200 as R
    from rotated_bit_dit_b200 import _binding as B
    from rotated_bit_dit_b200 import inputs as I

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    R.load()
    M, blocks = 16384, 28
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    xs = {}
    for k in (3072, 12288):
        xb = I.gaussian_bf16(k, (M, k), 1.0, 0.005, 30.0)
        xs[k] = torch.from_numpy(np.ascontiguousarray(xb).view(np.int16)).view(torch.bfloat16).to(dev)
    codes = torch.empty((M, 12288), dtype=torch.int8, device=dev)
    sx = torch.empty((M,), dtype=torch.float32, device=dev)
    y = torch.empty((M, 12288), dtype=torch.bfloat16, device=dev)
    layers, ops, n8 = [], 0.0, 0
    for b in range(blocks):
        for name, K, N in STACK_LAYERS:
            w = (torch.randn((N, K), generator=gen, device=dev) * 0.02).to(torch.bfloat16)
            int8 = stack_layer_is_int8(b, name)
            wq = torch.empty((N, K) if int8 else (N, K // 2), dtype=torch.int8 if int8 else torch.uint8, device=dev)
            sw = torch.empty((N,), dtype=torch.float32, device=dev)
            (B.rbd_pack_weights_int8 if int8 else B.rbd_pack_weights_int4)(w, wq, sw, 256, 0)
            del w
            layers.append((int8, K, N, wq, sw))
            ops += 2.0 * M * N * K
            n8 += int8
    torch.cuda.synchronize()

    def stack():
        for int8, K, N, wq, sw in layers:
            c = codes.view(-1)[:M * K].view(M, K)          # contiguous [M, K]
            out = y.view(-1)[:M * N].view(M, N)
            B.rbd_rot_quant_act(xs[K], c, sx, 8 if int8 else 4, 256, 0)
            (B.rbd_w8a8_linear if int8 else B.rbd_w4a4_linear)(c, sx, wq, sw, out, 0, None)

    for _ in range(max(args.warmup, 1)):
        stack()
    torch.cuda.synchronize()
    assert R.rbd_check() == 0
    ts = []
    with ClockSampler(dev.index) as clk:
        for _ in range(args.steps):
            a = torch.cuda.Event(enable_timing=True)
            e = torch.cuda.Event(enable_timing=True)
            a.record()
            stack()
            e.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(e) / 1e3)
    assert R.rbd_check() == 0
    t = statistics.median(ts)
    peaks, src = load_peaks()
    print(json.dumps({
        "sweep": "stack", "blocks": blocks, "linears": len(layers), "int8_linears": n8, "M": M,
        "ms_per_stack": t * 1e3, "tokens_per_s": M / t, "tops": ops / t / 1e12,
        "pct_int8_peak": 100.0 * ops / t / 1e12 / int8_peak_tops(peaks, src, sustained=True)[0],
        "int8_peak_source": int8_peak_tops(peaks, src, sustained=True)[1], "total_top": ops / 1e12,
        "timing": f"median of {args.steps} stacks after {max(args.warmup, 1)} warm-up stacks",
        "clocks": clk.summary()}), flush=True)


def _profile_traffic():
    """DRAM bytes per GEMM launch from the committed ncu record (a small JSON beside the
    summary).  The record carries the hash of the GEMM source it was captured from; a record
    of an older kernel gives no figure (null)."""
    if not os.path.exists(TRAFFIC_RECORD):
        return None
    with open(TRAFFIC_RECORD) as f:
        rec = json.load(f)
    if rec.get("source_sha256_16") != gemm_source_hash():
        return None
    v = rec.get("dram_bytes_per_launch")
    return int(v) if isinstance(v, (int, float)) else None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--print-gemm-hash", action="store_true", help="print the GEMM source hash and exit")
    ap.add_argument("--m-list", default=None,
                    help="small-m sweep: comma-separated token counts (default 1,16,64,256,1024)")
    ap.add_argument("--formats", default=None,
                    help="small-m sweep: comma-separated subset of w4a4,w4a4_g64,nvfp4")
    ap.add_argument("--sweep", choices=["small-m", "stack", "prologue", "kv4", "nvfp4", "qknorm", "peaks", "attn", "svdquant", "ffdown"], default=None,
                    help="instead of the headline line, print the small-token-count sweep (one line per case)")
    args = ap.parse_args()
    if args.print_gemm_hash:
        print(gemm_source_hash())
        return
    if args.sweep == "svdquant":
        run_svdquant_sweep(args)
        return
    if args.sweep == "attn":
        run_attn_sweep(args)
        return
    if args.sweep == "peaks":
        run_peaks(args)
        return
    if args.sweep == "small-m":
        run_small_m_sweep(args)
        return
    if args.sweep == "stack":
        run_stack(args)
        return
    if args.sweep == "prologue":
        run_prologue_sweep(args)
        return
    if args.sweep == "ffdown":
        run_ffdown_sweep(args)
        return
    if args.sweep == "kv4":
        run_kv4_sweep(args)
        return
    if args.sweep == "nvfp4":
        run_nvfp4_sweep(args)
        return
    if args.sweep == "qknorm":
        run_qknorm_sweep(args)
        return
    if args.impl == "reference" and int(os.environ.get("RANK", "0")) != 0:
        return                      # the oracle arm runs on rank 0 only; other ranks do no work
    from rotated_bit_dit_b200 import inputs as I
    cfg = I.CONFIGS[WORKLOAD]
    t = I.make_layer_inputs(cfg, seed=0)
    if args.impl == "reference":
        run_reference(args, cfg, t)
    else:
        run_ours(args, cfg, t)


if __name__ == "__main__":
    main()
