#!/usr/bin/env python
"""Benchmark of the OrbitQuant quantized linear layer forward on B200.

One step is one pass of the hot path over one batch of synthetic tokens:
rotate + quantize (norm, permutation gather, block Walsh-Hadamard, Lloyd-Max
codes) followed by the codebook contraction with the s*r epilogue.  The
weights are prepared once beforehand (offline in the method).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  Multi-GPU runs (torchrun) shard tokens: every
rank processes its own batch of the workload with replicated weights (weak
scaling, no collective on the data path).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized-linear tokens/s at d=3072; RPBH+quant HBM GB/s; GEMM % TC peak"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_FLUSH_BYTES = 256 << 20
# batches of up to this many tokens take the GEMV kernel (the library's routing)
GEMV_MAX_T = 24


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="dit_image")
    ap.add_argument("--tokens", type=int, default=0, help="override the workload's token count (profiling)")
    ap.add_argument("--layer", default="", help="layer of the workload by name (default: its first)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--route", choices=["levels", "staged", "levels_wdec", "codes"], default="levels",
                    help="hot-path route of the timed step (the others are reported beside it)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--sweep", action="store_true",
                    help="the stress workload's sweep (every token count x every layer): one JSON line per point")
    ap.add_argument("--sweep-small", default="1,8,16,24",
                    help="batch sizes of the batch-1 / GEMV end added to the sweep (comma list, empty for none)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "bf16_tflops_sustained": None, "source": "fallback"}


def measured_traffic(key: str):
    """Per-launch DRAM bytes (read + write) of a kernel from the ncu capture
    recorded in profiles/traffic.json, or None when there is none or the
    kernel's sources changed since it was taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)["kernels"].get(key)
    if rec is None:
        return None
    m = hashlib.sha256()
    for name in rec["sources"]:
        with open(os.path.join(ROOT, "quantized_linear_token_b200", "csrc", name), "rb") as f:
            m.update(f.read())
    if m.hexdigest() != rec["sources_sha256"]:
        return None
    return rec["dram_read_bytes"] + rec["dram_write_bytes"]


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.lines = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            v = [t.strip() for t in ln.split(",")]
            if len(v) < 9:
                continue
            try:
                sm.append(float(v[1]))
                smax.append(float(v[2]))
                power.append(float(v[3]))
            except ValueError:
                continue
            for n, flag in zip(names, v[5:9]):
                if flag.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None, "reasons": sorted(reasons), "samples": len(sm)}


class NvmlClockSampler:
    """SM clock, power and throttle reasons polled through NVML about every
    half millisecond, with host timestamps, so that the summary covers the
    timed region itself (a few milliseconds here, shorter than nvidia-smi's
    sampling period).  stop(t0, t1) summarises the samples taken between the
    host times t0 and t1 (perf_counter), or, if the region held none, the
    samples closest to it."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, gpu_uuid: str, period_s: float = 0.0005):
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        self.h = pynvml.nvmlDeviceGetHandleByUUID(gpu_uuid)
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        self.reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        self.period = period_s
        self.samples = []
        self.stop_flag = threading.Event()
        self.thread = None
        # one reading of each query now, so that a query this driver lacks
        # fails here (and the caller falls back) rather than in the thread
        pynvml.nvmlDeviceGetClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        self.reasons_fn(self.h)
        pynvml.nvmlDeviceGetPowerUsage(self.h)

    def _poll(self):
        nv = self.nv
        try:
            while not self.stop_flag.is_set():
                t = time.perf_counter()
                sm = float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                mask = int(self.reasons_fn(self.h))
                power = float(nv.nvmlDeviceGetPowerUsage(self.h)) / 1000.0
                self.samples.append((t, sm, mask, power))
                self.stop_flag.wait(self.period)
        except Exception:        # sampling ends; what was gathered is kept
            return

    def start(self):
        self.thread = threading.Thread(target=self._poll, daemon=True)
        self.thread.start()

    def stop(self, t0: float, t1: float):
        self.stop_flag.set()
        if self.thread is not None:
            self.thread.join(timeout=2.0)
        inside = [x for x in self.samples if t0 <= x[0] <= t1]
        window = "timed region"
        if not inside and self.samples:
            mid = 0.5 * (t0 + t1)
            inside = sorted(self.samples, key=lambda x: abs(x[0] - mid))[:3]
            window = "the samples nearest the timed region"
        reasons = sorted({n for _, _, m, _ in inside for n, bit in self.REASONS if m & bit})
        return {"sm_mhz": statistics.median([x[1] for x in inside]) if inside else None,
                "sm_max_mhz": self.max_mhz,
                "power_w_max": max(x[3] for x in inside) if inside else None,
                "reasons": reasons, "samples": len(inside), "source": f"NVML, {window}"}


def start_clock_sampler(uuid: str):
    """NVML sampling of the timed region if NVML answers, else nvidia-smi."""
    try:
        c = NvmlClockSampler(uuid)
        c.start()
        return c
    except Exception:
        c = ClockSampler(uuid)
        c.start()
        time.sleep(0.3)
        return c


def stop_clock_sampler(c, t0: float, t1: float):
    if isinstance(c, NvmlClockSampler):
        return c.stop(t0, t1)
    return c.stop()


# ------------------------------------------------------------------ oracle timing (host)
def oracle_cpu_rate_single_thread(wl, lay, seconds: float):
    """oracle_cpu_rate with numpy's thread pools limited to one thread."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        rate, el, done, _ = oracle_cpu_rate(wl, lay, seconds)
    return rate, el, done


def oracle_cpu_rate(wl, lay, seconds: float, chunk: int = 32):
    """Tokens/s of the fp64 oracle (as it stands) on this host's cores, on a
    bounded sample of the workload: chunks of `chunk` tokens, until `seconds`
    of work have run.  Weight rows are prepared by the oracle beforehand
    (offline in the method, not timed)."""
    import numpy as np
    from threadpoolctl import threadpool_info

    import oracle as O
    from quantized_linear_token_b200 import workloads as W

    d = lay.d_in
    h = O.hadamard_block_size(d)
    perm = O.rpbh_permutation(d, W.ROTATION_SEED)
    cb_a, cb_w = O.lloyd_max(d, lay.a_bits), O.lloyd_max(d, lay.w_bits)
    Wm = W.weights(wl, lay).astype(np.float64)
    wc, r, _ = O.weight_prepare(Wm, perm, h, cb_w)
    x = W.activations(wl, d, tokens=min(wl.tokens, 1024))
    x64 = O.bf16_bits_to_f64(x) if x.dtype == np.uint16 else x.astype(np.float64)
    done, t0 = 0, time.perf_counter()
    while True:
        i0 = (done % x64.shape[0])
        xs = x64[i0:i0 + chunk]
        codes, s, _ = O.rotate_quantize(xs, perm, h, cb_a)
        O.linear_from_codes(codes, s, wc, r, cb_a.levels, cb_w.levels)
        done += xs.shape[0]
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    threads = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    return done / el, el, done, threads


# ------------------------------------------------------------------ multi-rank helpers
def rank_batch(wl, d: int, tokens: int, rank: int):
    """This rank's own batch: weak scaling gives every rank `tokens` tokens of
    the workload's recipe, drawn from the rank's own seeded stream."""
    from quantized_linear_token_b200 import workloads as W
    return W.activations(wl, d, tokens=tokens, stream=rank)


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank number over all ranks (a no-op on one process)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, tokens_per_rank: int, steps: int, max_total_ms: float) -> float:
    """Tokens per second of the whole job: all ranks' tokens over the slowest
    rank's timed total."""
    return world * tokens_per_rank * steps / (max_total_ms * 1e-3)


# ------------------------------------------------------------------ our arm
def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    from quantized_linear_token_b200 import binding as B
    from quantized_linear_token_b200 import build as Bld
    from quantized_linear_token_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0:
        Bld.build()
    if world > 1:
        dist.barrier()
    B.load_library()

    wl = W.WORKLOADS[args.workload]
    if wl.x_dtype != "bf16":
        raise SystemExit(f"bench.py times bf16-activation workloads; {args.workload} ({wl.x_dtype} activations) "
                         "is a parity case of the tests")
    lay = next(l for l in wl.layers if l.name == args.layer) if args.layer else wl.layers[0]
    T, d, dout = (args.tokens or wl.tokens), lay.d_in, lay.d_out
    x_np = rank_batch(wl, d, T, rank)
    Wm = W.weights(wl, lay)
    x = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).to(dev)
    layer = B.oq_layer_create(d, dout, W.ROTATION_SEED, lay.a_bits, lay.w_bits)
    Wc, r = B.oq_weight_prepare(layer, torch.from_numpy(Wm).to(dev))
    codes = torch.empty((T, layer.a_words_per_row), dtype=torch.int32, device=dev)
    s = torch.empty((T,), dtype=torch.float32, device=dev)
    y = torch.empty((T, dout), dtype=torch.float32, device=dev)
    ws = torch.empty((B.oq_linear_fused_workspace_size(layer, T),), dtype=torch.uint8, device=dev)
    flush = torch.empty((L2_FLUSH_BYTES,), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    a16 = torch.empty((T, d), dtype=torch.float16, device=dev)
    w16 = torch.empty((dout, d), dtype=torch.float16, device=dev)

    # the routes of the hot path (all give the same y):
    #   levels:      the stages of oq_linear_fused at this batch size.  The
    #                activation codes leave K1 as fp16 levels; from W16_MIN_T
    #                tokens on the weight codes are decoded once into fp16
    #                levels and both operands reach the MMAs by TMA
    #                (oq_weight_levels + oq_linear_decoded), below it the
    #                contraction decodes the weight codes (oq_linear_levels).
    #   levels_wdec: oq_rotate_quantize_levels -> oq_linear_levels at any size
    #   codes:       oq_rotate_quantize -> oq_linear (packed codes between them)
    decoded = T >= B.W16_MIN_T and dout % 256 == 0
    ws_fd = torch.empty((max(B.oq_linear_fused_decoded_workspace_size(layer, T), 1),), dtype=torch.uint8,
                        device=dev)
    # the fused call's large-batch route runs one kernel for rotate-quantize
    # and the contraction where the block size is 1024 or 512 with at most 12
    # warps per token row (bf16 x, no Rademacher signs)
    h_blk = d & -d
    fused_kernel = decoded and dout <= d and ((h_blk == 1024 and d // h_blk <= 8) or
                                                (h_blk == 512 and d // h_blk <= 12))
    stages = {
        # the stages of oq_linear_fused at this batch size: the weight decode,
        # then the fused kernel where it runs, else rotate-quantize and the
        # contraction in turn
        "levels": ([("wlevels", lambda: B.oq_weight_levels(layer, Wc, w16)),
                    ("fused", lambda: B.oq_linear_fused_decoded(layer, x, w16, r, y, ws_fd))] if fused_kernel else
                   [("wlevels", lambda: B.oq_weight_levels(layer, Wc, w16)),
                    ("rq", lambda: B.oq_rotate_quantize_levels(layer, x, a16, s)),
                    ("gemm", lambda: B.oq_linear_decoded(layer, a16, s, w16, r, y))] if decoded else
                   [("rq", lambda: B.oq_rotate_quantize_levels(layer, x, a16, s)),
                    ("gemm", lambda: B.oq_linear_levels(layer, a16, s, Wc, r, y))]),
        # the same route with rotate-quantize and the contraction as two kernels
        "staged": [("rq", lambda: B.oq_rotate_quantize_levels(layer, x, a16, s))]
        + ([("wlevels", lambda: B.oq_weight_levels(layer, Wc, w16)),
            ("gemm", lambda: B.oq_linear_decoded(layer, a16, s, w16, r, y))] if decoded else
           [("gemm", lambda: B.oq_linear_levels(layer, a16, s, Wc, r, y))]),
        "levels_wdec": [("rq", lambda: B.oq_rotate_quantize_levels(layer, x, a16, s)),
                        ("gemm", lambda: B.oq_linear_levels(layer, a16, s, Wc, r, y))],
        "codes": [("rq", lambda: B.oq_rotate_quantize(layer, x, codes, s)),
                  ("gemm", lambda: B.oq_linear(layer, codes, s, Wc, r, y))],
    }

    def timed(route, K, warmup, sample_clocks=False):
        st = stages[route]
        for _ in range(warmup):
            flush.zero_()
            for _, fn in st:
                fn()
        torch.cuda.synchronize()
        B.oq_poll_error(layer)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(st) + 1)] for _ in range(K)]
        clocks = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid)) \
            if (rank == 0 and sample_clocks) else None
        if clocks:
            clocks.start()
            time.sleep(0.3)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        wall0 = time.perf_counter()
        for i in range(K):
            flush.zero_()                              # L2 flushed, outside the events
            ev[i][0].record(stream)
            for j, (_, fn) in enumerate(st):
                fn()
                ev[i][j + 1].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        wall = time.perf_counter() - wall0
        clk = clocks.stop() if clocks else None
        per = {name: [ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(K)] for j, (name, _) in enumerate(st)}
        B.oq_poll_error(layer)
        return per, wall, clk

    K = args.steps
    route = args.route
    others = [o for o in ("levels", "staged", "levels_wdec", "codes") if o != route]
    # the step: one oq_linear_fused call (the whole hot path, x -> y; from
    # W16_MIN_T tokens on it also decodes the weight levels once)
    for _ in range(args.warmup):
        flush.zero_()
        B.oq_linear_fused(layer, x, Wc, r, y, ws)
    torch.cuda.synchronize()
    B.oq_poll_error(layer)
    evf = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    clocks = start_clock_sampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid)) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for i in range(K):
        flush.zero_()                                  # L2 flushed, outside the events
        evf[i][0].record(stream)
        B.oq_linear_fused(layer, x, Wc, r, y, ws)
        evf[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    wall1 = time.perf_counter()
    wall = wall1 - wall0
    clk = stop_clock_sampler(clocks, wall0, wall1) if clocks else None
    B.oq_poll_error(layer)
    t_fused = [evf[i][0].elapsed_time(evf[i][1]) for i in range(K)]
    total_ms = max_over_ranks(sum(t_fused), dev)

    # the same path as its separate stage calls, one event per kernel: the
    # per-kernel times of the rooflines
    per, _, _ = timed(route, K, args.warmup)
    stage_ms = max_over_ranks(sum(sum(v) for v in per.values()), dev)
    other_per = {o: timed(o, K, max(3, args.warmup // 2))[0] for o in others}
    other_ms = {o: max_over_ranks(sum(sum(v) for v in other_per[o].values()), dev) for o in others}

    # end to end through the public API with host buffers: the host-buffer
    # fused call copies pinned x in, computes and copies y out to pinned host
    # memory, overlapped chunk by chunk; all of it inside the events
    x_host = x.cpu().pin_memory()
    y_host = torch.empty((T, dout), dtype=torch.float32).pin_memory()
    ws_host = torch.empty((max(B.oq_linear_fused_host_workspace_size(layer, B.OQ_DTYPE_BF16, T), 1),),
                          dtype=torch.uint8, device=dev)
    eve = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    for i in range(max(2, args.warmup // 2)):
        B.oq_linear_fused_host(layer, x_host, Wc, r, y_host, ws_host)
    torch.cuda.synchronize()
    for i in range(K):
        eve[i][0].record(stream)
        B.oq_linear_fused_host(layer, x_host, Wc, r, y_host, ws_host)
        eve[i][1].record(stream)
    torch.cuda.synchronize()
    t_e2e = [eve[i][0].elapsed_time(eve[i][1]) for i in range(K)]
    e2e_ms = max_over_ranks(sum(t_e2e), dev)
    B.oq_poll_error(layer)

    # the same step and the same end-to-end call with bf16 y (half the output
    # bytes: the epilogue's write and the copy out)
    y_b = torch.empty((T, dout), dtype=torch.bfloat16, device=dev)
    y_host_b = torch.empty((T, dout), dtype=torch.bfloat16).pin_memory()
    evb = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    for _ in range(max(2, args.warmup // 2)):
        flush.zero_()
        B.oq_linear_fused(layer, x, Wc, r, y_b, ws)
        B.oq_linear_fused_host(layer, x_host, Wc, r, y_host_b, ws_host)
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()
        evb[i][0].record(stream)
        B.oq_linear_fused(layer, x, Wc, r, y_b, ws)
        evb[i][1].record(stream)
    for i in range(K):
        evb[i][2].record(stream)
        B.oq_linear_fused_host(layer, x_host, Wc, r, y_host_b, ws_host)
        evb[i][3].record(stream)
    torch.cuda.synchronize()
    B.oq_poll_error(layer)
    bf16_ms = max_over_ranks(sum(evb[i][0].elapsed_time(evb[i][1]) for i in range(K)), dev)
    bf16_e2e_ms = max_over_ranks(sum(evb[i][2].elapsed_time(evb[i][3]) for i in range(K)), dev)

    peaks = load_peaks()
    flops = 2.0 * T * d * dout

    def rq_bytes_per_launch(rt):
        # the bytes this route's kernel moves: bf16 x read + its A operand
        # written (fp16 levels, or packed codes) + norms
        return T * (2 * d + (2 * d if rt != "codes" else d * lay.a_bits / 8) + 4)

    # the method's algorithmic bytes of rotate + quantize, whatever the route
    # writes: bf16 x read, packed codes and the norm written
    rq_alg_bytes = T * (2 * d + d * lay.a_bits / 8 + 4)

    def contraction_key(pr):
        return "fused" if "fused" in pr else "gemm"

    # the stand-alone rotate-quantize kernel: in this route, or else in the
    # staged form of it (the fused kernel runs rotate-quantize inside the
    # contraction, so it has no time of its own)
    rq_src = per if "rq" in per else other_per.get("staged", other_per.get("levels_wdec"))
    rq_route = route if "rq" in per else "staged"
    wl_bytes = dout * d * (lay.w_bits / 8 + 2)     # weight codes read + fp16 levels written
    ckey = contraction_key(per)
    mm_ms = statistics.mean(per[ckey])
    rq_ms = statistics.mean(rq_src["rq"])
    rq_bytes = rq_bytes_per_launch(rq_route)
    gemm_tf = flops / (mm_ms * 1e-3) / 1e12
    rq_gbs = rq_bytes / (rq_ms * 1e-3) / 1e9
    gemm_desc = {
        "fused": ("fused layer kernel: producer warps rotate-quantize the tokens (norm, gather, block FWHT on "
                  "the CUDA cores, Lloyd-Max codes as fp16 levels) for the tcgen05 CTA-pair contraction of the "
                  "decoded weights, fp32 TMEM accumulate", "fused"),
        "decoded": ("codebook GEMM on fp16 levels of both operands, both by TMA "
                    "(tcgen05 CTA pair, fp32 TMEM accumulate)", "gemm_decoded"),
        "levels_wdec": ("codebook GEMM, fp16 A operand by TMA, weight codes decoded to fp16 in shared memory "
                        "(tcgen05 CTA pair, fp32 TMEM accumulate)", "gemm_levels"),
        "codes": ("codebook GEMM, both operands' codes decoded to fp16 in shared memory "
                  "(tcgen05 CTA pair, fp32 TMEM accumulate)", None),
    }
    gkey = ("fused" if ckey == "fused" else "decoded" if (decoded and route in ("levels", "staged")) else
            "codes" if route == "codes" else "levels_wdec")
    rq_desc = {
        "levels": "rotate + quantize (norm, gather, block FWHT, Lloyd-Max codes) writing the codes' fp16 levels",
        "codes": "rotate + quantize (norm, gather, block FWHT, Lloyd-Max codes, pack)",
    }
    steps_desc = {
        "levels": ("oq_weight_levels + oq_linear_fused_decoded (the fused kernel)" if fused_kernel
                   else "oq_weight_levels + oq_rotate_quantize_levels + oq_linear_decoded" if decoded else
                   "oq_rotate_quantize_levels + oq_linear_levels")
        + " (the stages of oq_linear_fused at this batch size; weights prepared once, offline)",
        "staged": ("oq_rotate_quantize_levels + oq_weight_levels + oq_linear_decoded" if decoded else
                   "oq_rotate_quantize_levels + oq_linear_levels")
        + " (the same route, rotate-quantize and the contraction as separate kernels)",
        "levels_wdec": "oq_rotate_quantize_levels + oq_linear_levels (weight codes decoded inside the contraction)",
        "codes": "oq_rotate_quantize + oq_linear (weights prepared once, offline)",
    }

    def route_summary(o):
        pr = other_per[o]
        c = contraction_key(pr)
        row = {"route": o, "step": steps_desc[o], "value": whole_job_rate(world, T, K, other_ms[o]), "unit": UNIT,
               "ms_per_step": other_ms[o] / K, "contraction": c,
               "gemm_tflops": flops / (statistics.mean(pr[c]) * 1e-3) / 1e12, "gemm_ms": statistics.mean(pr[c])}
        if "rq" in pr:
            row.update({"rq_gbs": rq_alg_bytes / (statistics.mean(pr["rq"]) * 1e-3) / 1e9,
                        "rq_route_gbs": rq_bytes_per_launch(o) / (statistics.mean(pr["rq"]) * 1e-3) / 1e9,
                        "rq_ms": statistics.mean(pr["rq"])})
        return row

    full_size = T == wl.tokens
    launches_per_step = (2 if fused_kernel else 3) if decoded else 2
    out = {
        "metric": METRIC,
        "value": whole_job_rate(world, T, K, total_ms),
        "unit": UNIT,
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": total_ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16",
        "data": "synthetic",
        "config": {
            **workload_config(args, wl, lay, T, world),
            "l2": "flushed (256 MiB write) before every step, outside the timed events",
            "step": "one oq_linear_fused call (x -> y: " + steps_desc["levels"].split(" (")[0] + ")",
        },
        "roofline": {
            "kernel": gemm_desc[gkey][0],
            "bound": "tensor", "achieved": gemm_tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": gemm_tf / peaks["bf16_tflops"],
            "traffic": measured_traffic(gemm_desc[gkey][1]) if (gemm_desc[gkey][1] and full_size) else None,
            "peak_source": f"{peaks['source']} bf16 dense burst (fp16 has the same tensor rate)",
            "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum per launch, profiles/traffic.json",
            "flops_per_launch": flops, "ms_per_launch": mm_ms,
        },
        "roofline_rotate_quantize": {
            "kernel": rq_desc["codes" if rq_route == "codes" else "levels"]
            + ("" if rq_route == route else " (the stand-alone kernel of the staged route)"),
            "bound": "hbm", "achieved": rq_alg_bytes / (rq_ms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": rq_alg_bytes / (rq_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "bytes_per_launch": rq_alg_bytes,
            "bytes_rule": "algorithmic: 2 d (bf16 x) + d a_bits / 8 (packed codes) + 4 (norm) per token",
            "traffic": measured_traffic("rq_levels" if rq_route != "codes" else "rq_codes") if full_size else None,
            "peak_source": f"{peaks['source']} HBM copy bandwidth",
            "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum per launch, profiles/traffic.json",
            "ms_per_launch": rq_ms,
            "route_bytes_per_launch": rq_bytes, "route_achieved": rq_gbs, "route_frac": rq_gbs / peaks["hbm_gbs"],
            "route_bytes_rule": ("the bytes this route's kernel moves: its A operand is written as fp16 levels, "
                                 "2 d bytes per token" if rq_route != "codes" else "same as algorithmic"),
        },
        **({"roofline_weight_levels": {
            "kernel": "weight codes -> fp16 levels (once per call)",
            "bound": "hbm", "achieved": wl_bytes / (statistics.mean(per["wlevels"]) * 1e-3) / 1e9,
            "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": wl_bytes / (statistics.mean(per["wlevels"]) * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "traffic": measured_traffic("weight_levels") if full_size else None,
            "bytes_per_launch": wl_bytes, "ms_per_launch": statistics.mean(per["wlevels"]),
        }} if "wlevels" in per else {}),
        "stages": {"value": whole_job_rate(world, T, K, stage_ms), "unit": UNIT, "ms_per_step": stage_ms / K,
                   "step": steps_desc[route] + "; separate calls on one stream, one event per kernel"},
        "other_routes": [route_summary(o) for o in others],
        "e2e": {"value": whole_job_rate(world, T, K, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": int(x.numel() * x.element_size()),
                "d2h_bytes_per_step": int(y.numel() * y.element_size()),
                "path": "oq_linear_fused_host: pinned host x -> device, fused call, y -> pinned host, overlapped in chunks of 1024 tokens"},
        "bf16_y": {"value": whole_job_rate(world, T, K, bf16_ms), "unit": UNIT, "ms_per_step": bf16_ms / K,
                   "step": "one oq_linear_fused call writing bf16 y",
                   "e2e": {"value": whole_job_rate(world, T, K, bf16_e2e_ms), "unit": UNIT,
                           "h2d_bytes_per_step": int(x.numel() * x.element_size()),
                           "d2h_bytes_per_step": int(y_b.numel() * y_b.element_size()),
                           "path": "oq_linear_fused_host with bf16 y_host"}},
        "gpu_launches": launches_per_step * K,
        "wall_s_timed_region": wall,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, el, done, threads = oracle_cpu_rate(wl, lay, args.cpu_seconds)
        rate1, el1, done1 = oracle_cpu_rate_single_thread(wl, lay, max(1.0, args.cpu_seconds / 4))
        out["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
                               "sample": f"{done} tokens of {args.workload} in chunks of 32 "
                                         f"({el:.1f} s): oracle rotate_quantize + linear_from_codes, "
                                         f"fp64 numpy; weight rows prepared beforehand",
                               "single_thread": {"value": rate1, "unit": UNIT, "cores": 1,
                                                 "sample": f"{done1} tokens ({el1:.1f} s), numpy limited to "
                                                           f"one thread"}}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


# ------------------------------------------------------------------ reference arm
def workload_config(args, wl, lay, T, world):
    """The config keys both arms report for one workload and layer."""
    return {
        "workload": f"{args.workload}: {wl.title}", "layer": lay.name,
        "tokens_per_gpu": T, "d_in": lay.d_in, "d_out": lay.d_out, "a_bits": lay.a_bits, "w_bits": lay.w_bits,
        "h": lay.d_in & -lay.d_in, "x_dtype": wl.x_dtype, "y_dtype": "fp32",
        "parallelism": f"token-sharded x{world}, weights replicated",
    }


def run_reference(args):
    """The oracle timed on the host cores, on this arm's workload/metric."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from quantized_linear_token_b200 import workloads as W
    wl = W.WORKLOADS[args.workload]
    lay = next(l for l in wl.layers if l.name == args.layer) if args.layer else wl.layers[0]
    per_step = max(1.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_cpu_rate(wl, lay, min(per_step, 2.0))
    rates, total_tok, total_s, threads = [], 0, 0.0, 1
    for _ in range(args.steps):
        rate, el, done, threads = oracle_cpu_rate(wl, lay, per_step)
        rates.append(rate)
        total_tok += done
        total_s += el
    value = total_tok / total_s
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {**workload_config(args, wl, lay, args.tokens or wl.tokens, args.gpus),
                   "step": "the oracle (fp64 numpy): rotate_quantize + linear_from_codes on a bounded "
                           "sample of the workload's tokens, weight rows prepared beforehand"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{total_tok} tokens, {args.steps} steps of ~{per_step:.1f} s, chunks of 32"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def run_sweep(args):
    """The stress sweep on one GPU: 13824 -> 5120 at every token count of the
    workload and every layer (W2A4, W3A3, W4A4, W4A8).  Per point: the step
    (one oq_linear_fused call, L2 flushed before each), then the same path as
    stage calls with an event after each kernel for the rooflines.  One JSON
    line per point."""
    import numpy as np
    import torch

    from quantized_linear_token_b200 import binding as B
    from quantized_linear_token_b200 import build as Bld
    from quantized_linear_token_b200 import workloads as W

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    Bld.build()
    B.load_library()
    peaks = load_peaks()
    wl = W.WORKLOADS["stress"]
    small = [int(v) for v in args.sweep_small.split(",") if v.strip()]
    sweep = tuple(sorted(set(small) | set(wl.token_sweep)))
    d = wl.layers[0].d_in
    # the recipe does not depend on the batch size, so every smaller batch is
    # the first rows of the largest one
    x_all = torch.from_numpy(W.activations(wl, d, tokens=max(sweep)).view(np.int16)).view(torch.bfloat16).to(dev)
    flush = torch.empty((L2_FLUSH_BYTES,), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    K, warm = args.steps, max(3, args.warmup)
    for lay in wl.layers:
        dout = lay.d_out
        layer = B.oq_layer_create(d, dout, W.ROTATION_SEED, lay.a_bits, lay.w_bits)
        Wc, r = B.oq_weight_prepare(layer, torch.from_numpy(W.weights(wl, lay)).to(dev))
        for T in sweep:
            x = x_all[:T]
            y = torch.empty((T, dout), dtype=torch.float32, device=dev)
            ws = torch.empty((B.oq_linear_fused_workspace_size(layer, T),), dtype=torch.uint8, device=dev)
            a16 = torch.empty((T, d), dtype=torch.float16, device=dev)
            s = torch.empty((T,), dtype=torch.float32, device=dev)
            decoded = T >= B.W16_MIN_T
            w16 = torch.empty((dout, d), dtype=torch.float16, device=dev) if decoded else None
            stages = [("rq", lambda: B.oq_rotate_quantize_levels(layer, x, a16, s))]
            if decoded:
                stages += [("wlevels", lambda: B.oq_weight_levels(layer, Wc, w16)),
                           ("gemm", lambda: B.oq_linear_decoded(layer, a16, s, w16, r, y))]
            else:
                stages += [("gemm", lambda: B.oq_linear_levels(layer, a16, s, Wc, r, y))]
            runs = {"step": [("step", lambda: B.oq_linear_fused(layer, x, Wc, r, y, ws))], "stages": stages}
            h_blk = d & -d
            fused_kernel = decoded and dout <= d and ((h_blk == 1024 and d // h_blk <= 8) or
                                                (h_blk == 512 and d // h_blk <= 12))
            if fused_kernel:
                # the step runs the weight decode and the fused kernel: time
                # the fused kernel on its own
                ws_fd = torch.empty((max(B.oq_linear_fused_decoded_workspace_size(layer, T), 1),),
                                    dtype=torch.uint8, device=dev)
                runs["fused"] = [("fused", lambda: B.oq_linear_fused_decoded(layer, x, w16, r, y, ws_fd))]
            times = {}
            for name, st in runs.items():
                for _ in range(warm):
                    flush.zero_()
                    for _, fn in st:
                        fn()
                ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(st) + 1)] for _ in range(K)]
                torch.cuda.synchronize()
                for i in range(K):
                    flush.zero_()
                    ev[i][0].record(stream)
                    for j, (_, fn) in enumerate(st):
                        fn()
                        ev[i][j + 1].record(stream)
                torch.cuda.synchronize()
                for j, (kname, _) in enumerate(st):
                    times[kname] = statistics.mean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(K))
            B.oq_poll_error(layer)
            flops = 2.0 * T * d * dout
            rq_alg = T * (2 * d + d * lay.a_bits / 8 + 4)
            # the step's dominant kernel: the fused kernel where the step runs
            # one, else the contraction
            ck = "fused" if fused_kernel else "gemm"
            line = {
                "metric": METRIC, "sweep_point": True, "value": T / (times["step"] * 1e-3), "unit": UNIT,
                "n_gpus": 1, "steps": K, "warmup": warm, "ms_per_step": times["step"],
                "higher_is_better": True, "dtype": "f16", "data": "synthetic",
                "config": {"workload": f"stress: {wl.title}", "layer": lay.name, "tokens_per_gpu": T, "d_in": d,
                           "d_out": dout, "a_bits": lay.a_bits, "w_bits": lay.w_bits, "h": d & -d,
                           "x_bytes": T * d * 2,
                           "l2": "flushed (256 MiB write) before every step, outside the timed events",
                           "contraction": "decoded weights, both operands by TMA" if decoded else
                           ("GEMV kernel (warp MMAs, weight codes decoded in registers)" if T <= GEMV_MAX_T else
                            "small-batch split-K kernel" if T <= 256 else "CTA pair, weights decoded in the GEMM")},
                "roofline": {"kernel": "fused layer kernel (rotate-quantize and contraction)"
                             if fused_kernel else "contraction",
                             "bound": "tensor", "achieved": flops / (times[ck] * 1e-3) / 1e12,
                             "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                             "frac": flops / (times[ck] * 1e-3) / 1e12 / peaks["bf16_tflops"],
                             "traffic": None, "ms_per_launch": times[ck]},
                "contraction_alone": {"achieved": flops / (times["gemm"] * 1e-3) / 1e12,
                                      "frac": flops / (times["gemm"] * 1e-3) / 1e12 / peaks["bf16_tflops"],
                                      "ms_per_launch": times["gemm"]},
                "roofline_rotate_quantize": {"bound": "hbm", "achieved": rq_alg / (times["rq"] * 1e-3) / 1e9,
                                             "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                             "frac": rq_alg / (times["rq"] * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                             "bytes_per_launch": rq_alg, "ms_per_launch": times["rq"]},
                "step_tflops": flops / (times["step"] * 1e-3) / 1e12,
                "step_frac": flops / (times["step"] * 1e-3) / 1e12 / peaks["bf16_tflops"],
            }
            if T <= GEMV_MAX_T:
                # the batch-1 / GEMV end: the contraction streams the weight
                # codes once; its floor is their bytes at HBM speed
                gb = dout * d * lay.w_bits / 8 + T * d * 2 + dout * 4 + T * dout * 4
                line["roofline_tensor"] = line["roofline"]
                line["roofline"] = {
                    "kernel": "small-batch contraction (warp MMAs, weight codes decoded in registers)",
                    "bound": "hbm", "achieved": gb / (times["gemm"] * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": gb / (times["gemm"] * 1e-3) / 1e9 / peaks["hbm_gbs"],
                    "bytes_per_launch": gb, "ms_per_launch": times["gemm"],
                    "floor_ms": gb / (peaks["hbm_gbs"] * 1e9) * 1e3,
                    "bytes_rule": "weight codes + fp16 activation levels + r + fp32 y"}
            if decoded:
                wb = dout * d * (lay.w_bits / 8 + 2)
                line["roofline_weight_levels"] = {"bound": "hbm", "achieved": wb / (times["wlevels"] * 1e-3) / 1e9,
                                                  "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                                  "frac": wb / (times["wlevels"] * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                                  "bytes_per_launch": wb, "ms_per_launch": times["wlevels"]}
            print(json.dumps(line), flush=True)
            del y, ws, a16, s, w16


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.sweep:
        run_sweep(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
