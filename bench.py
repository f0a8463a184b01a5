"""Benchmark of the W4A4 WUSH linear layer hot path on B200.

One step = the whole hot path on one batch: wush_transform_quant of the
activations (WUSH block transform + MXFP4 quantisation) followed by wush_qgemm
(tcgen05 block-scaled FP4 GEMM) into fp32 y.  Weights are transformed and
quantised once, offline, outside the timed region.

Default workload (up_proj): X bf16 [4096 tokens, 4096] Student-t(3) with 41
outlier channels x50, W [12288, 4096] N(0, 0.02^2), per-block (b = 32) WUSH
transforms from 8192 seeded calibration tokens, MXFP4.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {wush,reference}]

N > 1 is launched by torchrun (one process per GPU); every rank runs its own
batch (weak scaling, no collective on the data path); timing is the max over
ranks of the device-timed region.  ``--impl reference`` times the CPU oracle on
the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

L2_BYTES = 126 * 2 ** 20
ROTATIONS = 3
STEPS_PER_GRAPH = 12            # steps captured per CUDA graph (four passes over the rotations)
FP4_OVER_BF16 = 4.0          # nominal dense FP4 : BF16 tensor ratio (9 : 2.25 PFLOP/s)


# --------------------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    bf16_tflops_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def dist_init(world: int):
    """One process per GPU: NCCL when CUDA is present, gloo otherwise (CPU tests)."""
    if world <= 1:
        return None
    import datetime

    import torch
    import torch.distributed as dist
    backend = "nccl" if torch.cuda.is_available() else "gloo"
    if backend == "nccl":
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int) -> float:
    """The largest ``value`` of all ranks (device time is taken as the slowest rank's)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def source_sha(source_file: str) -> str:
    """Hash of a kernel's source file together with the device headers it includes
    (quoted includes found beside it, followed recursively; the public C header, which
    holds declarations only, is left out)."""
    dirs = [os.path.dirname(source_file)]
    seen, order, todo = set(), [], [source_file]
    while todo:
        f = todo.pop(0)
        if f in seen:
            continue
        seen.add(f)
        order.append(f)
        for line in open(f, encoding="utf-8", errors="replace"):
            m = re.match(r'\s*#\s*include\s+"([^"]+)"', line)
            if m:
                for d in dirs:
                    cand = os.path.join(d, m.group(1))
                    if os.path.exists(cand):
                        todo.append(cand)
                        break
    h = hashlib.sha1()
    for f in [order[0]] + sorted(order[1:]):
        h.update(open(f, "rb").read())
    return h.hexdigest()[:12]


def traffic_from_profiles(kernel: str, workload: str, source_file: str):
    """DRAM bytes per launch recorded by an ncu capture, if the kernel source is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    sha = source_sha(source_file)
    for line in open(path):
        f = dict(kv.split("=", 1) for kv in line.split() if "=" in kv)
        if f.get("kernel") == kernel and f.get("workload") == workload and f.get("src_sha") == sha:
            return float(f["dram_bytes_per_launch"])
    return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the GPU is loaded."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "hw_power_brake_slowdown": 0x80, "sw_power_cap": 0x4}

    def __init__(self, index: int, period_s: float = 0.002):   # a timed region is a few ms
        self.samples, self.reasons = [], set()
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: report no samples
            self.nv = None
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                get = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
                r = get(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv is not None:
            self._t.join()

    def summary(self):
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}

    def rejected(self):
        bad = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"} & self.reasons
        stuck = (self.samples and self.max_mhz and statistics.median(self.samples) < 0.6 * self.max_mhz
                 and not self.reasons)
        return bool(bad) or bool(stuck)


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("num_threads")]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count()


# --------------------------------------------------------------------------- workload

WORKLOADS = {
    "tiny": dict(fmt="mxfp4", kind="wush"),          # 128 x 256 x 256: a quick check, not a bench line
    "up_proj": dict(fmt="mxfp4", kind="wush"),
    "down_proj": dict(fmt="nvfp4", kind="wush"),
    "int4": dict(fmt="int4", kind="wush"),
}


def build_inputs(name: str, tokens=None):
    w = synth.WORKLOADS[name]
    if tokens:
        import dataclasses
        w = dataclasses.replace(w, tokens=tokens)
    x = synth.activations(w)
    wt = synth.weights(w)
    xc = synth.activations(w, calib=True)
    return w, x, wt, xc


def describe(w, fmt, kind):
    return {"workload": (f"{w.name}: X bf16 [{w.tokens} tok, {w.d_in}] {w.x_dist} with {w.n_outlier} outlier "
                         f"channels x{w.outlier_factor:g}; W bf16 [{w.d_out}, {w.d_in}] N(0,0.02^2); "
                         f"{kind.upper()} b={w.block} from {w.n_calib} calib tokens; {fmt.upper()} W4A4, y fp32"),
            "M": w.tokens, "N": w.d_out, "K": w.d_in, "format": fmt, "transform": kind,
            "l2": f"inputs > L2: y is {w.tokens * w.d_out * 4 / 2**20:.0f} MiB per step; "
                  f"{ROTATIONS} rotating copies of X and of the weight codes"}


# --------------------------------------------------------------------------- CPU oracle leg

class OracleLeg:
    """The oracle on a sample of token rows of the step (T_X X -> quantise -> fp64 GEMM).

    Calibration and the weights' transform + quantisation are prepared once (offline
    work, as on the GPU side); ``step(rows)`` is the timed part.
    """

    def __init__(self, w, x, wt, xc, fmt, kind, groups=0):
        from oracle import calibrate as C
        from oracle import quant as Q
        from oracle import transforms as T
        self.w, self.x, self.fmt = w, x, fmt
        if groups:      # shared transforms, expanded to one per block
            sx, sw, idx = C.shared_transforms(C.block_moments(xc, w.block), C.block_moments(wt, w.block), kind, groups)
            tx, tw = sx[idx], sw[idx]
        else:
            tx, tw = C.calibrate(xc, wt, w.block, kind)
        self.tx, tw = tx.astype(np.float32), tw.astype(np.float32)
        self.gx = gw = None
        if fmt == "nvfp4":
            self.gx = C.nvfp4_global_scale(T.apply_block_transform(xc, self.tx).astype(np.float32))
            gw = C.nvfp4_global_scale(T.apply_block_transform(wt, tw).astype(np.float32))
        self.w_dq = Q.transform_quantize(wt, tw, fmt, gw)["dq"]

    def step(self, rows):
        from oracle import gemm as G
        from oracle import quant as Q
        a = Q.transform_quantize(self.x[:rows], self.tx, self.fmt, self.gx)["dq"]
        return G.gemm_dequantized(a, self.w_dq)

    def rows_for(self, seconds):
        t0 = time.perf_counter()
        self.step(16)
        dt = time.perf_counter() - t0
        return int(min(self.w.tokens, max(16, 16 * seconds / max(dt, 1e-3))))


def time_oracle(w, x, wt, xc, fmt, kind, target_s=12.0, groups=0):
    leg = OracleLeg(w, x, wt, xc, fmt, kind, groups)
    rows = leg.rows_for(target_s / 3)
    t0 = time.perf_counter()
    reps = 0
    while True:
        leg.step(rows)
        reps += 1
        if time.perf_counter() - t0 > target_s / 2 or reps >= 8:
            break
    dt = (time.perf_counter() - t0) / reps
    flops = 2.0 * rows * w.d_out * w.d_in
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{rows} of {w.tokens} token rows through the whole step (transform, quantise, fp64 "
                      f"GEMM against the offline-quantised {w.d_out}x{w.d_in} weights), {reps} reps, "
                      f"{dt:.2f} s each"}


# --------------------------------------------------------------------------- GPU leg

def run_gpu(args, rank, world):
    import torch
    import activation_quantization_b200 as aq

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    spec = dict(WORKLOADS[args.workload])
    if args.transform:
        spec["kind"] = args.transform
    fmt, kind = spec["fmt"], spec["kind"]
    w, x, wt, xc = build_inputs(args.workload, args.tokens)
    M, N, K = w.tokens, w.d_out, w.d_in
    b = w.block

    # offline: calibration (host C++), weight transform + quantisation (GPU), NVFP4 scales
    groups = args.share_groups
    if groups:
        if kind in ("identity", "hadamard"):
            raise SystemExit("--share-groups needs a dense transform (wus, wush, wush_diag)")
        tx_s, tw_s, t_idx = aq.wush_calibrate_shared(xc, wt, b, kind, groups)
        tx, tw = tx_s[t_idx], tw_s[t_idx]                  # expanded, for the offline NVFP4 scales
        t_xs, t_ws = torch.from_numpy(tx_s).to(dev), torch.from_numpy(tw_s).to(dev)
        t_idx_dev = torch.from_numpy(t_idx).to(dev)
    else:
        tx, tw = aq.wush_calibrate(xc, wt, b, kind)
    t_x, t_w = torch.from_numpy(tx).to(dev), torch.from_numpy(tw).to(dev)

    def quant(x_in, t_full, t_shared, fmt_, codes_, scales_, gs_, stream_=None):
        if groups:
            aq.wush_transform_quant_indexed(x_in, t_shared, t_idx_dev, kind, fmt_, codes_, scales_, gs_, stream=stream_)
        else:
            aq.wush_transform_quant(x_in, t_full, kind, fmt_, codes_, scales_, gs_, stream=stream_)
    gx = gw = 0.0
    if fmt == "nvfp4":
        amax = torch.empty(1, dtype=torch.float32, device=dev)
        aq.wush_transform_amax(torch.from_numpy(xc).to(torch.bfloat16).to(dev), t_x, kind, b, amax)
        gx = aq.wush_nvfp4_global_scale(amax.item())
        wt_dev = torch.from_numpy(wt).to(torch.bfloat16).to(dev)
        aq.wush_transform_amax(wt_dev, t_w, kind, b, amax)
        gw = aq.wush_nvfp4_global_scale(amax.item())
    alpha = aq.wush_nvfp4_alpha(gx, gw) if fmt == "nvfp4" else 1.0
    xs = [torch.from_numpy(x).to(torch.bfloat16).to(dev) for _ in range(ROTATIONS)]
    wcodes = []
    for _ in range(ROTATIONS):
        bc, bs = aq.alloc_quant_outputs(N, K, fmt, dev)
        quant(torch.from_numpy(wt).to(torch.bfloat16).to(dev), t_w, t_ws if groups else None, fmt, bc, bs, gw)
        wcodes.append((bc, bs))
    acodes = [aq.alloc_quant_outputs(M, K, fmt, dev) for _ in range(ROTATIONS)]
    y = torch.empty((M, N), dtype=torch.float32, device=dev)
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)

    # NVFP4 with --dynamic-scale: each step derives the activations' per-tensor scale
    # on the device (an amax pass over T x, then the quantiser and the GEMM's alpha
    # read it), instead of the static calibrated scale
    dynamic = fmt == "nvfp4" and args.dynamic_scale
    if dynamic and groups:
        raise SystemExit("--share-groups applies to the static-scale path only")
    dyn_amax = torch.zeros(1, dtype=torch.float32, device=dev)
    dyn_gs = torch.zeros(1, dtype=torch.float32, device=dev)

    def tq_into(x_in, acode):
        if dynamic:
            aq.wush_transform_amax(x_in, t_x, kind, b, dyn_amax, stream=stream)
            aq.wush_transform_quant_nvfp4_dynamic(x_in, t_x, kind, dyn_amax, acode[0], acode[1], dyn_gs,
                                                  stream=stream)
        else:
            quant(x_in, t_x, t_xs if groups else None, fmt, acode[0], acode[1], gx, stream)

    def tq(r):
        tq_into(xs[r], acodes[r])

    # INT4: the two-pass form (each operand dequantised once to fp16, then a CTA-pair
    # fp16 GEMM); its workspace is allocated once, outside the timed region
    ws = (torch.empty(aq.wush_qgemm_int4_workspace_bytes(M, N, K), dtype=torch.uint8, device=dev)
          if fmt == "int4" else None)

    def gemm_into(acode, wcode, y_out):
        if fmt == "int4":
            aq.wush_qgemm_int4_ws(acode[0], acode[1], wcode[0], wcode[1], M, N, K, ws, y_out, stream=stream)
        elif dynamic:
            aq.wush_qgemm_nvfp4_dynamic(acode[0], acode[1], wcode[0], wcode[1], M, N, K, dyn_gs, gw, y_out,
                                        stream=stream)
        else:
            aq.wush_qgemm(acode[0], acode[1], wcode[0], wcode[1], M, N, K, fmt, alpha, y_out, stream=stream)

    def gemm(r):
        gemm_into(acodes[r], wcodes[r], y)

    # The timed steps run as CUDA graphs of STEPS_PER_GRAPH consecutive steps
    # (rotating through the input copies), with event nodes between the kernels so
    # that each kernel's device time is read without the graph-launch latency.
    with torch.cuda.stream(stream):
        for r in range(ROTATIONS):
            tq(r)
            gemm(r)
    stream.synchronize()

    def capture(n_steps, start=0, events=True):
        """A graph of n_steps steps; with ``events`` an event node sits between the
        kernels (for per-kernel times), without them consecutive kernels are adjacent,
        so each may start its set-up under the previous one's tail (programmatic
        dependent launch)."""
        g = torch.cuda.CUDAGraph()
        evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in range(n_steps)]
        with torch.cuda.graph(g, stream=stream):
            for j in range(n_steps):
                r = (start + j) % ROTATIONS
                if events:
                    evs[j][0].record(stream)
                tq(r)
                if events:
                    evs[j][1].record(stream)
                gemm(r)
                if events:
                    evs[j][2].record(stream)
        return g, evs

    g_main, _ = capture(STEPS_PER_GRAPH, events=False)
    n_rem = args.steps % STEPS_PER_GRAPH
    g_rem, _ = capture(n_rem, events=False) if n_rem else (None, [])
    g_ev, ev_main = capture(STEPS_PER_GRAPH)
    # a graph's event nodes refer to its Event objects: keep every (graph, events) pair alive
    g_one = [capture(1, r) for r in range(ROTATIONS)]
    if aq.wush_check_device_status(stream) != 0:
        raise RuntimeError("device status after capture")

    def timed(steps):
        e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            e_start.record(stream)
            for _ in range(steps // STEPS_PER_GRAPH):
                g_main.replay()
            if g_rem is not None:
                g_rem.replay()
            e_end.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        total_ms = e_start.elapsed_time(e_end)
        return total_ms

    def kernel_times():
        """Per-kernel device times from the event nodes of one replay of the evented graph."""
        with torch.cuda.stream(stream):
            g_ev.replay()
        stream.synchronize()
        return ([e[0].elapsed_time(e[1]) for e in ev_main], [e[1].elapsed_time(e[2]) for e in ev_main])

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            g_one[i % ROTATIONS][0].replay()
    stream.synchronize()

    for attempt in range(2):
        sampler = ClockSampler(dev.index)
        with sampler:
            total_ms = timed(args.steps)
        if not sampler.rejected():
            break
    tq_ms, gm_ms = kernel_times()
    status = aq.wush_check_device_status(stream)
    if status != 0:
        raise RuntimeError(f"device status {status}")

    # The transform alone, as a burst of back-to-back launches over the rotating
    # inputs: inside a step it also absorbs the write-back of the GEMM's y from L2.
    g_tq = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_tq, stream=stream):
        for j in range(STEPS_PER_GRAPH):
            tq(j % ROTATIONS)
    with torch.cuda.stream(stream):
        g_tq.replay()
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        for _ in range(8):
            g_tq.replay()
        b1.record(stream)
    torch.cuda.synchronize()
    tq_burst_us = 1e3 * b0.elapsed_time(b1) / (8 * STEPS_PER_GRAPH)

    # Batches pipelined over two streams: the transform of batch j runs on a second
    # stream as soon as its output buffer is free again (the GEMM of batch j - 3 has
    # read it), so it overlaps the GEMM of batch j - 1, its tail and its y write-back.
    # Same work per step; reported beside the serial step, not as the headline.
    pipe_us = None
    if not dynamic:
        side = torch.cuda.Stream(device=dev)
        ev_tq = [torch.cuda.Event() for _ in range(STEPS_PER_GRAPH)]
        ev_gm = [torch.cuda.Event() for _ in range(STEPS_PER_GRAPH)]
        g_pipe = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_pipe, stream=stream):
            side.wait_stream(stream)
            for j in range(STEPS_PER_GRAPH):
                r = j % ROTATIONS
                if j >= ROTATIONS:
                    side.wait_event(ev_gm[j - ROTATIONS])
                quant(xs[r], t_x, t_xs if groups else None, fmt, acodes[r][0], acodes[r][1], gx, side)
                ev_tq[j].record(side)
                stream.wait_event(ev_tq[j])
                gemm(r)
                ev_gm[j].record(stream)
            stream.wait_stream(side)
        with torch.cuda.stream(stream):
            g_pipe.replay()
            p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            p0.record(stream)
            for _ in range(8):
                g_pipe.replay()
            p1.record(stream)
        torch.cuda.synchronize()
        pipe_us = 1e3 * p0.elapsed_time(p1) / (8 * STEPS_PER_GRAPH)
        del g_pipe

    total_ms = max_over_ranks(total_ms, world)

    flops_step = 2.0 * M * N * K
    value = flops_step * args.steps * world / (total_ms * 1e-3) / 1e12
    tq_us = 1e3 * float(np.mean(tq_ms))
    gm_us = 1e3 * float(np.mean(gm_ms))
    peaks = load_peaks()
    # the GEMM's own dtype: FP4 for MXFP4/NVFP4, fp16 for the dequantised INT4 path
    fp4_peak = peaks["bf16_tflops"] * (FP4_OVER_BF16 if fmt != "int4" else 1.0)
    tq_bytes = (M * K * 2 + aq.wush_codes_bytes(M, K, fmt) + aq.wush_scales_bytes(M, K, fmt)
                + (K // b) * b * b * 4)
    gemm_kernel = ("hgemm_pair_kernel" if fmt == "int4"
                   else "qgemm_pair_kernel" if M % 256 == 0 and N % 256 == 0 else "qgemm_kernel")
    gemm_peak_src = ("bf16 burst x 1 (the INT4 path multiplies fp16)" if fmt == "int4"
                     else f"bf16 burst x {FP4_OVER_BF16:g} (nominal dense FP4:BF16)")
    gemm_tflops = flops_step / (gm_us * 1e-6) / 1e12
    tq_gbs = tq_bytes / (tq_us * 1e-6) / 1e9
    qgemm_src = os.path.join(ROOT, "activation_quantization_b200", "csrc",
                             "qgemm_int4.cu" if fmt == "int4" else "qgemm.cu")
    tq_src = os.path.join(ROOT, "activation_quantization_b200", "csrc", "transform_quant_tc.cu")

    # End to end through the public API: every step uploads its X from pinned host
    # memory and downloads its fp32 y.  The copies run on their own streams and the
    # device buffers are double-buffered, so step i's kernels overlap step i+1's
    # upload and step i-1's download; the time runs from the first upload to the
    # last download.
    if True:
        x_host = torch.from_numpy(x).to(torch.bfloat16).pin_memory()
        y_host = [torch.empty((M, N), dtype=torch.float32).pin_memory() for _ in range(2)]
        y_dev = [y, torch.empty_like(y)]
        up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            sl = i % 2
            with torch.cuda.stream(up):
                up.wait_event(ev_done[sl])            # step i-2 has finished reading xs[sl]
                xs[sl].copy_(x_host, non_blocking=True)
                ev_in[sl].record(up)
            with torch.cuda.stream(stream):
                stream.wait_event(ev_in[sl])
                stream.wait_event(ev_out[sl])         # step i-2's y has been downloaded
                tq_into(xs[sl], acodes[sl])
                gemm_into(acodes[sl], wcodes[0], y_dev[sl])
                ev_done[sl].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev_done[sl])
                y_host[sl].copy_(y_dev[sl], non_blocking=True)
                ev_out[sl].record(down)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        e_steps = max(4, min(args.steps, 12))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(up)
        for i in range(e_steps):
            e2e_step(i)
        e1.record(down)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1) / e_steps, world)
        e2e = {"value": flops_step * world / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(x_host.numel() * 2), "d2h_bytes_per_step": int(y_host[0].numel() * 4),
               "ms_per_step": e_ms}

    result = None
    if rank == 0:
        traffic = traffic_from_profiles(gemm_kernel, args.workload, qgemm_src)
        tq_traffic = traffic_from_profiles("tq_tc_kernel", args.workload, tq_src)
        result = {
            "metric": "transform+quant HBM GB/s; W4A4 block-scaled GEMM TFLOP/s (% of peak)",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e2m1 x e2m1 -> fp32 (transform in fp32)", "data": "synthetic",
            "config": dict(describe(w, fmt, kind),
                           **({"nvfp4_scale": "dynamic: device amax pass + scale every step "
                                              "(inside the transform's time)"} if dynamic else {}),
                           **({"transform_sharing": f"{groups} shared transforms for {K // b} blocks "
                                                    f"({groups * b * b * 4} B of T_X instead of {K * b * 4} B)"}
                              if groups else {})),
            "transform_quant": {"us": tq_us, "GB_s": tq_gbs, "bytes_per_launch": tq_bytes,
                                "frac_of_hbm": tq_gbs / peaks["hbm_gbs"], "dram_bytes_per_launch": tq_traffic,
                                "burst_us": tq_burst_us,
                                "burst_frac_of_hbm": tq_bytes / (tq_burst_us * 1e-6) / 1e9 / peaks["hbm_gbs"]},
            "qgemm": {"us": gm_us, "TFLOP_s": gemm_tflops, "frac_of_peak": gemm_tflops / fp4_peak},
            "pipelined_step": None if pipe_us is None else {
                "us": pipe_us, "TFLOP_s": flops_step / (pipe_us * 1e-6) / 1e12,
                "how": "transform of batch j on a second stream, overlapping the GEMM of batch j - 1 "
                       f"({ROTATIONS} rotating code buffers); graph bursts of {STEPS_PER_GRAPH} steps"},
            "roofline": {"kernel": gemm_kernel, "bound": "tensor", "achieved": gemm_tflops, "peak": fp4_peak,
                         "unit": "TFLOP/s", "frac": gemm_tflops / fp4_peak, "traffic": traffic,
                         "peak_source": f"{peaks['source']} bf16 burst {peaks['bf16_tflops']:.1f} TFLOP/s, {gemm_peak_src}"},
            "e2e": e2e, "gpu_launches": (4 if fmt == "int4" else 3 if dynamic else 2) * args.steps,
            "clocks": sampler.summary(),
        }
    return result, (w, x, wt, xc, fmt, kind)


# --------------------------------------------------------------------------- ITQ3 GEMV

def measure_itq3(steps: int, warmup: int):
    """Times itq3_dequant_gemv (both modes) at 1, 4 and 16 tokens; one dict per (tokens, mode)."""
    import torch
    import activation_quantization_b200 as aq
    dev = torch.device("cuda", torch.cuda.current_device())
    w = synth.itq3_weights()
    d_out, d_in = w.shape
    codes, scales = aq.itq3_quantize_weights(w.astype(np.float16))
    copies = 24                                    # 24 x 6.4 MB of weights rotate: more than L2
    cs = [torch.from_numpy(codes).to(dev) for _ in range(copies)]
    ss = [torch.from_numpy(scales).to(dev) for _ in range(copies)]
    peaks = load_peaks()
    out = []
    for t in synth.ITQ3_TOKENS:
        x = torch.from_numpy(synth.itq3_activations(t).astype(np.float16)).to(dev)
        y = torch.empty((t, d_out), dtype=torch.float32, device=dev)
        ws = torch.empty((t, d_in), dtype=torch.float32, device=dev)
        for mode in (0, 1):
            # one CUDA graph holds a burst of calls over the rotating weight copies,
            # so the device time is not bounded by the host's launch rate
            burst = 2 * copies
            stream = torch.cuda.Stream(device=dev)
            with torch.cuda.stream(stream):
                for i in range(3):
                    aq.itq3_dequant_gemv(cs[i], ss[i], x, d_out, mode, y, ws, stream=stream)
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(burst):
                    aq.itq3_dequant_gemv(cs[i % copies], ss[i % copies], x, d_out, mode, y, ws, stream=stream)
            reps = max(1, steps // burst)
            with torch.cuda.stream(stream):
                for _ in range(max(1, warmup // burst)):
                    g.replay()
            stream.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                for _ in range(reps):
                    g.replay()
                e1.record(stream)
            stream.synchronize()
            us = e0.elapsed_time(e1) / (reps * burst) * 1e3
            byts = codes.nbytes + scales.nbytes + t * d_in * 2 + t * d_out * 4
            tc = mode == 1 and t >= 3 and d_out % 128 == 0
            out.append({"workload": f"itq3 W fp16 [{d_out}, {d_in}] 3-bit, {t} tokens", "tokens": t,
                        "mode": "fused inverse FWHT" if mode == 0 else "activation-side rotation",
                        "kernel": "itq3_tc_kernel (tcgen05, fp16 levels from TMEM)" if tc
                        else "itq3_gemv_kernel (CUDA cores)",
                        "us": us, "GB_s": byts / us / 1e3, "frac_of_hbm": byts / us / 1e3 / peaks["hbm_gbs"],
                        "bytes_per_call": byts})
            del g
    return out


def run_itq3(args):
    """Prints one JSON line per (tokens, mode) of the ITQ3 GEMV."""
    for line in measure_itq3(args.steps, args.warmup):
        print(json.dumps(line))


# --------------------------------------------------------------------------- the other workloads

EXTRA_STEPS = 24          # steps of each other workload: one CUDA graph, replayed after a warm replay


def _graph_kernel_times(stream, launches, n_steps, reps=3):
    """Captures n_steps steps, each the callables ``launches`` (called with the step
    index), into two CUDA graphs: one with event nodes between the kernels (per-kernel
    times), one without (the step time, kernels adjacent as in the headline step).
    Each is replayed once warm, then timed.  Returns (us per step, [us per launch kind])."""
    import torch
    g_plain, g_ev = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(launches) + 1)]
           for _ in range(n_steps)]
    with torch.cuda.graph(g_plain, stream=stream):
        for j in range(n_steps):
            for fn in launches:
                fn(j)
    with torch.cuda.graph(g_ev, stream=stream):
        for j in range(n_steps):
            for i, fn in enumerate(launches):
                evs[j][i].record(stream)
                fn(j)
            evs[j][-1].record(stream)
    with torch.cuda.stream(stream):
        g_plain.replay()
        g_ev.replay()
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            g_plain.replay()
        e1.record(stream)
        g_ev.replay()
    stream.synchronize()
    per_step = 1e3 * e0.elapsed_time(e1) / (reps * n_steps)
    per_kind = [1e3 * float(np.mean([e[i].elapsed_time(e[i + 1]) for e in evs])) for i in range(len(launches))]
    del g_plain, g_ev
    return per_step, per_kind


def measure_layer(dev, stream, inputs, fmt, kind, tokens=None):
    """The step (transform + quantise of X, then the GEMM) of one workload, timed as
    a graph of EXTRA_STEPS steps over rotating copies; weights prepared offline."""
    import torch
    import activation_quantization_b200 as aq
    w, x, wt, xc = inputs
    if tokens:
        x = x[:tokens]
    M, N, K, b = x.shape[0], w.d_out, w.d_in, w.block
    tx, tw = aq.wush_calibrate(xc, wt, b, kind)
    t_x, t_w = torch.from_numpy(tx).to(dev), torch.from_numpy(tw).to(dev)
    gx = gw = 0.0
    alpha = 1.0
    wt_dev = torch.from_numpy(wt).to(torch.bfloat16).to(dev)
    if fmt == "nvfp4":
        amax = torch.zeros(1, dtype=torch.float32, device=dev)
        aq.wush_transform_amax(torch.from_numpy(xc).to(torch.bfloat16).to(dev), t_x, kind, b, amax)
        gx = aq.wush_nvfp4_global_scale(amax.item())
        aq.wush_transform_amax(wt_dev, t_w, kind, b, amax)
        gw = aq.wush_nvfp4_global_scale(amax.item())
        alpha = aq.wush_nvfp4_alpha(gx, gw)
    xs = [torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).to(dev) for _ in range(ROTATIONS)]
    bc, bs = aq.alloc_quant_outputs(N, K, fmt, dev)
    aq.wush_transform_quant(wt_dev, t_w, kind, fmt, bc, bs, gw)
    del wt_dev
    wcodes = [(bc, bs)] + [(bc.clone(), bs.clone()) for _ in range(ROTATIONS - 1)]
    acodes = [aq.alloc_quant_outputs(M, K, fmt, dev) for _ in range(ROTATIONS)]
    y = torch.empty((M, N), dtype=torch.float32, device=dev)
    ws = (torch.empty(aq.wush_qgemm_int4_workspace_bytes(M, N, K), dtype=torch.uint8, device=dev)
          if fmt == "int4" else None)

    def tq(j):
        r = j % ROTATIONS
        aq.wush_transform_quant(xs[r], t_x, kind, fmt, acodes[r][0], acodes[r][1], gx, stream=stream)

    def gemm(j):
        r = j % ROTATIONS
        (a, sa), (bb, sb) = acodes[r], wcodes[r]
        if fmt == "int4":
            aq.wush_qgemm_int4_ws(a, sa, bb, sb, M, N, K, ws, y, stream=stream)
        else:
            aq.wush_qgemm(a, sa, bb, sb, M, N, K, fmt, alpha, y, stream=stream)

    with torch.cuda.stream(stream):
        for j in range(ROTATIONS):
            tq(j)
            gemm(j)
    stream.synchronize()
    step_us, (tq_us, gm_us) = _graph_kernel_times(stream, [tq, gemm], EXTRA_STEPS)
    if aq.wush_check_device_status(stream) != 0:
        raise RuntimeError(f"device status after {w.name} {kind}")
    peaks = load_peaks()
    tq_bytes = M * K * 2 + aq.wush_codes_bytes(M, K, fmt) + aq.wush_scales_bytes(M, K, fmt) + (K // b) * b * b * 4
    flops = 2.0 * M * N * K
    gemm_peak = peaks["bf16_tflops"] * (FP4_OVER_BF16 if fmt != "int4" else 1.0)
    gemm_tflops = flops / (gm_us * 1e-6) / 1e12
    return {"M": M, "N": N, "K": K, "format": fmt, "transform": kind, "step_us": step_us,
            "TFLOP_s": flops / (step_us * 1e-6) / 1e12,
            "transform_quant": {"us": tq_us, "GB_s": tq_bytes / (tq_us * 1e-6) / 1e9,
                                "frac_of_hbm": tq_bytes / (tq_us * 1e-6) / 1e9 / peaks["hbm_gbs"],
                                "bytes_per_launch": tq_bytes},
            "gemm": {"kernel": ("int4_dequant_kernel x2 + hgemm_pair_kernel (fp16 MMA)" if fmt == "int4"
                                else "qgemm_pair_kernel (block-scaled FP4 MMA)"),
                     "us": gm_us, "TFLOP_s": gemm_tflops, "frac_of_peak": gemm_tflops / gemm_peak,
                     "peak": gemm_peak}}


def tiny_losses(dev):
    """Loss l = ||y - W^T X||_F^2 / (d_out tokens) of the GPU layer on the tiny workload
    (MXFP4), for the identity, Hadamard and WUSH transforms."""
    import torch
    import activation_quantization_b200 as aq
    w, x, wt, xc = build_inputs("tiny")
    M, N, K = w.tokens, w.d_out, w.d_in
    ref = x.astype(np.float64) @ wt.astype(np.float64).T
    out = {}
    for kind in ("identity", "hadamard", "wush"):
        tx, tw = aq.wush_calibrate(xc, wt, w.block, kind)
        ac, as_ = aq.alloc_quant_outputs(M, K, "mxfp4", dev)
        bc, bs = aq.alloc_quant_outputs(N, K, "mxfp4", dev)
        aq.wush_transform_quant(torch.from_numpy(x).to(dev), torch.from_numpy(tx).to(dev), kind, "mxfp4", ac, as_)
        aq.wush_transform_quant(torch.from_numpy(wt).to(dev), torch.from_numpy(tw).to(dev), kind, "mxfp4", bc, bs)
        y = torch.empty((M, N), dtype=torch.float32, device=dev)
        aq.wush_qgemm(ac, as_, bc, bs, M, N, K, "mxfp4", 1.0, y)
        d = y.cpu().numpy().astype(np.float64) - ref
        out[kind] = float(np.sum(d * d) / (N * M))
    out["workload"] = (f"tiny: X fp32 [{M} tok, {K}] N(0,1) with {w.n_outlier} outlier channels "
                       f"x{w.outlier_factor:g}; W [{N}, {K}]; MXFP4 b=32 through the GPU path")
    return out


def run_extras(args):
    """The other workloads' kernels, each measured in this process, for the bench line."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.Stream(device=dev)
    extras = {}
    inp = build_inputs("down_proj")
    extras["down_proj"] = {k: measure_layer(dev, stream, inp, "nvfp4", k) for k in ("wus", "wush")}
    del inp
    inp = build_inputs("int4")
    extras["int4_2048"] = measure_layer(dev, stream, inp, "int4", "wush", tokens=2048)
    extras["int4_8192"] = measure_layer(dev, stream, inp, "int4", "wush")
    del inp
    torch.cuda.empty_cache()
    extras["itq3"] = measure_itq3(max(args.steps, 96), 48)
    extras["tiny_loss"] = tiny_losses(dev)
    torch.cuda.empty_cache()
    return extras


# --------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="wush", choices=["wush", "reference"])
    ap.add_argument("--workload", default="up_proj", choices=sorted(WORKLOADS) + ["itq3"])
    ap.add_argument("--tokens", type=int, default=None, help="override the workload's token count")
    ap.add_argument("--transform", default=None, choices=["identity", "hadamard", "wus", "wush", "wush_diag"],
                    help="override the workload's block transform (calibrated from the same tokens)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other workloads' kernel timings (down_proj, int4, itq3, tiny loss)")
    ap.add_argument("--share-groups", type=int, default=0,
                    help="share the dense transforms among this many groups of similar blocks")
    ap.add_argument("--dynamic-scale", action="store_true",
                    help="NVFP4: derive the activations' per-tensor scale on the device every step")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    if args.workload == "itq3":
        if rank == 0:               # a per-call latency benchmark: one rank times it
            run_itq3(args)
        return
    spec = dict(WORKLOADS[args.workload])
    if args.transform:
        spec["kind"] = args.transform

    if args.impl == "reference":
        if rank != 0:
            return
        w, x, wt, xc = build_inputs(args.workload, args.tokens)
        leg = OracleLeg(w, x, wt, xc, spec["fmt"], spec["kind"], args.share_groups)
        step_rows = leg.rows_for(1.5)
        times = []
        for i in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            leg.step(step_rows)
            if i >= args.warmup:
                times.append(time.perf_counter() - t0)
        dt = sum(times) / len(times)
        val = 2.0 * step_rows * w.d_out * w.d_in / dt / 1e12
        cb = {"value": val, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
              "sample": f"{step_rows} of {w.tokens} token rows per step through the whole step"}
        print(json.dumps({"impl": "reference", "metric": "transform+quant HBM GB/s; W4A4 block-scaled GEMM "
                          "TFLOP/s (% of peak)", "value": val, "unit": "TFLOP/s", "n_gpus": world,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                          "data": "synthetic", "config": describe(w, spec["fmt"], spec["kind"]),
                          "cpu_baseline": cb,
                          "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                                  "d2h_bytes_per_step": 0}}))
        return

    dist_init(world)
    result, ctx = run_gpu(args, rank, world)
    if rank == 0:
        if world == 1 and not args.no_extras:
            result.update(run_extras(args))
        if world == 1 and not args.no_cpu_baseline:
            w, x, wt, xc, fmt, kind = ctx
            result["cpu_baseline"] = time_oracle(w, x, wt, xc, fmt, kind, groups=args.share_groups)
        print(json.dumps(result))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
