#!/usr/bin/env python
"""Benchmark of the MicroQonv hot path on B200: one step = for every layer of
the workload, MX-quantize X, W and G_Y (each once, both code orders), then the
block-scaled forward, input-gradient and weight-gradient convolutions.

Prints one JSON line (rank 0).  `value` is the whole-job MX conv fwd+bwd
throughput in TFLOP/s (algorithmic 2*M*N*K of the three GEMMs of every layer,
divided by the device time of the full step, quantization included), with the
inputs already in HBM.  `e2e` is the same metric through the same C-ABI calls
with the fp32 inputs copied from pinned host memory and the three outputs
copied back inside the timed region.  `roofline` is for the launch that takes
the largest share of the step; `cpu_baseline` times the oracle (plain C,
double precision) on a bounded batch slice of the same workload.

--impl reference runs that oracle as the reference arm.
Multi-GPU (torchrun): each rank runs the full per-GPU workload on its own
batch (weak scaling) and the weight gradients are summed across ranks with
one NCCL all-reduce per step, the data-parallel exchange of training.
"""
from __future__ import annotations

import argparse
import ctypes
import glob
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

WORKLOAD_CFG = 3
METRIC = "MX conv fwd+bwd TFLOPS (quantizer GB/s and % of roofline alongside) at 1 B200"


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="mqc", choices=["mqc", "reference"])
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-extras", action="store_true",
                    help="skip the fused step, the tensor-bound layers and the stochastic-rounding quantizer")
    ap.add_argument("--profile", default=None, metavar="CALL[,CALL...]",
                    help="profiling mode: build one layer, then run the listed calls (quantize_x, quantize_w, quantize_g, fwd, "
                         "dgrad, wgrad) --reps times and exit")
    ap.add_argument("--layer", type=int, default=0)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--workload", default="3",
                    help="workload of --profile / --sweep: 3 (YOLO training step), 4, or 5:fp8:N / 5:fp4:N")
    ap.add_argument("--sweep", action="store_true",
                    help="time every call of every layer of --workload (the other configurations: parity-test "
                         "cases, reported separately from the bench line)")
    return ap.parse_args(argv)


# --------------------------------------------------------------------------- distributed plumbing
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def max_over_ranks(value: float, device) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def allreduce_weight_grads(tensors):
    """The data-parallel exchange of the step: every rank's weight gradients
    (partial sums over its own batch shard) are summed over the ranks in
    place, so each rank ends with the gradient of the whole global batch.
    The only collective of the path; nothing when running alone."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        for t in tensors:
            dist.all_reduce(t, op=dist.ReduceOp.SUM)


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix=f"mqc_clocks_gpu{self.idx}_", suffix=".csv")
            self.fh = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        try:
            os.unlink(self.path)
        except OSError:
            pass
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        load = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- peaks
def kernel_sources_sha256() -> str:
    """Hash of the CUDA sources and the C header: DRAM counters taken by ncu
    on one version of the kernels are reported only for that version."""
    h = hashlib.sha256()
    files = sorted(glob.glob(os.path.join(ROOT, "im2col_gemm_b200", "csrc", "*.cu*")))
    for f in files + [os.path.join(ROOT, "include", "mqc.h")]:
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(kernel: str):
    """dram__bytes_read.sum + dram__bytes_write.sum of one launch of `kernel`
    (e.g. "dgrad layer 0") from the ncu record under profiles/, or None when
    no record exists for the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("sources_sha256") != kernel_sources_sha256():
        return None
    k = rec.get("calls", {}).get(kernel)
    return None if k is None else k["dram_bytes_read"] + k["dram_bytes_write"]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# --------------------------------------------------------------------------- the step
class LayerBuffers:
    """Device (and pinned host) buffers of one layer of the training step."""

    def __init__(self, mqc, torch, L: synth.Layer, wl: synth.Workload, i: int, want_host: bool):
        dev = torch.device("cuda")
        x, w, g = synth.layer_inputs(wl, i)
        self.L = L
        self.cv = mqc.conv_desc(L.N, L.C, L.H, L.W, L.K, L.R, L.S, L.stride, L.pad)
        self.x = torch.from_numpy(x).to(dev)
        self.w = torch.from_numpy(w).to(dev)
        self.g = torch.from_numpy(g).to(dev)
        self.host_in = None
        if want_host:
            self.host_in = [torch.from_numpy(a).pin_memory() for a in (x, w, g)]
        blk = wl.block
        self.mx = {}
        self.q = {}
        for name, t, fmt in (("x", self.x, wl.fmt_x), ("w", self.w, wl.fmt_w), ("g", self.g, wl.fmt_g)):
            d = tuple(t.shape)
            mx = mqc.MX(fmt, blk, 0)
            nc = mqc.mqc_codes_bytes(mx, *d)
            nc2 = mqc.mqc_codes_bytes(mqc.MX(fmt, blk, 1), *d)
            ns = mqc.mqc_scales_bytes(mx, *d)
            codes = torch.empty(nc, dtype=torch.uint8, device=dev)
            alt = torch.empty(nc2, dtype=torch.uint8, device=dev)
            scales = torch.empty(ns, dtype=torch.uint8, device=dev)
            self.q[name] = mqc.Quantized(codes, scales, d, mx, alt)
            self.mx[name] = mx
            self.desc = getattr(self, "desc", {})
            self.desc[name] = mqc.T4(*d, *t.stride())
        self.y = torch.empty((L.N, L.K, L.P, L.Q), dtype=torch.float32, device=dev)
        self.gx = torch.empty((L.N, L.C, L.H, L.W), dtype=torch.float32, device=dev)
        self.gw = torch.empty((L.K, L.C, L.R, L.S), dtype=torch.float32, device=dev)
        qx, qw, qg = self.q["x"], self.q["w"], self.q["g"]
        self.ws_fwd = mqc.mqc_conv2d_fwd_workspace_bytes(self.cv, qx.mx, qw.mx)
        self.ws_dgrad = mqc.mqc_conv2d_bwd_data_workspace_bytes(self.cv, qw.other_order().mx, qg.mx)
        self.ws_wgrad = mqc.conv2d_bwd_weight_workspace_bytes(self.cv, qg.other_order().mx, qx.other_order().mx)
        # E2M1 operands are widened to E4M3 codes inside each GEMM call (one
        # launch per widened operand); the weight gradient reduces split-K
        # partials when its workspace holds more than the widened copies
        widen = {k: (2 * self.q[k].codes.numel() + 255) // 256 * 256 if self.q[k].mx.fmt == mqc.E2M1 else 0
                 for k in ("x", "w", "g")}
        self.n_widen = 2 * sum(1 for v in widen.values() if v)
        self.split_k = self.ws_wgrad > widen["g"] + widen["x"]
        self.ws_bytes = max(self.ws_fwd, self.ws_dgrad, self.ws_wgrad)
        self.host_out = None
        if want_host:
            self.host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (self.y, self.gx, self.gw)]

    # algorithmic work of each call
    def quant_bytes(self, name):
        t = {"x": self.x, "w": self.w, "g": self.g}[name]
        q = self.q[name]
        return 4 * t.numel() + q.codes.numel() + q.codes_alt.numel() + q.scales.numel()

    def gemm_flops(self):
        return self.L.gemm_flops()

    def gemm_bytes(self, op, nxt=None):
        qx, qw, qg = self.q["x"], self.q["w"], self.q["g"]
        if op == "fwd_quant":
            ny = nxt.q["x"]
            return (qx.codes.numel() + qx.scales.numel() + qw.codes.numel() + qw.scales.numel()
                    + ny.codes.numel() + ny.codes_alt.numel() + ny.scales.numel())
        if op == "fwd":
            return qx.codes.numel() + qx.scales.numel() + qw.codes.numel() + qw.scales.numel() + 4 * self.y.numel()
        if op == "dgrad":
            return qg.codes.numel() + qg.scales.numel() + qw.codes.numel() + qw.scales.numel() + 4 * self.gx.numel()
        return qg.codes.numel() + qg.scales.numel() + qx.codes.numel() + qx.scales.numel() + 4 * self.gw.numel()

    def launches(self, mqc):
        """Kernels one pass of this layer launches: 3 quantizations, the
        forward GEMM, the input gradient (as one sub-pixel GEMM after the
        kernel that builds its window weights when the 2 to 4 stride phases
        tile the input and C is a multiple of 16; else its stride phases
        share launches of up to 4 height phases), the weight-gradient GEMM
        and, with split-K partials, their reduction."""
        L = self.L
        subpix = 2 <= L.stride * L.stride <= 4 and L.H % L.stride == 0 and L.W % L.stride == 0 and L.C % 16 == 0
        dgrad = 2 if subpix else -(-L.stride // 4)
        return 3 + 1 + dgrad + (2 if self.split_k else 1) + self.n_widen


def run_layer(mqc, lb: LayerBuffers, workspace, stream, events=None, only=None, nxt=None, with_x=True):
    """All calls of one layer through the C ABI; `events` (optional) collects
    (name, start, end) CUDA events around every call on `stream`; `only`
    (a tuple of call names) restricts the run to those calls (profiling).
    With `nxt` (the next layer's buffers) the forward is "fwd_quant": its
    epilogue applies SiLU and writes the next layer's quantized input (both
    code orders) instead of the fp32 output; `with_x` False skips this
    layer's own quantize_x (its input came from the previous forward)."""
    c_void = ctypes.c_void_p
    P = lambda t: c_void(t.data_ptr())

    def timed(name, fn):
        if only is not None and name not in only:
            return
        if events is not None:
            import torch
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            mqc.check(fn())
            e1.record()
            events.append((name, e0, e1))
        else:
            mqc.check(fn())

    for name, t in (("x", lb.x), ("w", lb.w), ("g", lb.g)):
        if name == "x" and not with_x:
            continue
        q = lb.q[name]
        timed(f"quantize_{name}", lambda q=q, t=t, name=name: mqc.mqc_quantize_mx(
            P(t), lb.desc[name], q.mx, P(q.codes), P(q.scales), P(q.codes_alt), stream))
    if only is not None and "quantize_g_sr" in only:
        # the output gradient with stochastically rounded elements (timed alone)
        q = lb.q["g"]
        timed("quantize_g_sr", lambda: mqc.mqc_quantize_mx_sr(
            P(lb.g), lb.desc["g"], q.mx, P(q.codes), P(q.scales), P(q.codes_alt), 1234, 0, stream))
    qx, qw, qg = lb.q["x"], lb.q["w"], lb.q["g"]
    wq_ab, gq_ab, xq_ab = qw.other_order(), qg.other_order(), qx.other_order()
    wsp = P(workspace) if lb.ws_bytes else None
    if nxt is not None:
        ny = nxt.q["x"]
        timed("fwd_quant", lambda: mqc.mqc_conv2d_fwd_quant(
            P(qx.codes), P(qx.scales), qx.mx, P(qw.codes), P(qw.scales), qw.mx, lb.cv, mqc.ACT_SILU, ny.mx,
            P(ny.codes), P(ny.scales), P(ny.codes_alt), None, wsp, lb.ws_fwd, stream))
    else:
        timed("fwd", lambda: mqc.mqc_conv2d_fwd(P(qx.codes), P(qx.scales), qx.mx, P(qw.codes), P(qw.scales),
                                                qw.mx, lb.cv, P(lb.y), wsp, lb.ws_fwd, stream))
    timed("dgrad", lambda: mqc.mqc_conv2d_bwd_data(P(wq_ab.codes), P(wq_ab.scales), wq_ab.mx, P(qg.codes),
                                                   P(qg.scales), qg.mx, lb.cv, P(lb.gx), wsp, lb.ws_dgrad, stream))
    timed("wgrad", lambda: mqc.mqc_conv2d_bwd_weight(P(gq_ab.codes), P(gq_ab.scales), gq_ab.mx, P(xq_ab.codes),
                                                     P(xq_ab.scales), xq_ab.mx, lb.cv, P(lb.gw),
                                                     wsp, lb.ws_wgrad, stream))


# --------------------------------------------------------------------------- CPU oracle
def oracle_sample(wl: synth.Workload, n_images: int = 1, layers=None):
    """Times the oracle on a batch slice (n_images of N) of the same layers:
    quantize X, W, G_Y and the three convolutions in double.  Returns
    (algorithmic flops, seconds, threads, description)."""
    import oracle as orc
    orc.build()
    layers = range(len(wl.layers)) if layers is None else layers
    flops = 0
    t_total = 0.0
    for i in layers:
        L = wl.layers[i]
        x, w, g = synth.layer_inputs(wl, i)
        x, g = np.ascontiguousarray(x[:n_images]), np.ascontiguousarray(g[:n_images])
        t0 = time.perf_counter()
        cx, sx = orc.quantize(x, wl.fmt_x, wl.block, 0)
        cw, sw = orc.quantize(w, wl.fmt_w, wl.block, 0)
        cg, sg = orc.quantize(g, wl.fmt_g, wl.block, 0)
        xd = orc.dequantize(cx, sx, x.shape, wl.fmt_x, wl.block, 0)
        wd = orc.dequantize(cw, sw, w.shape, wl.fmt_w, wl.block, 0)
        gd = orc.dequantize(cg, sg, g.shape, wl.fmt_g, wl.block, 0)
        st, pd = L.stride, L.pad
        orc.conv_fwd(xd, wd, st, st, pd, pd)
        orc.conv_dgrad(wd, gd, L.H, L.W, st, st, pd, pd)
        orc.conv_wgrad(gd, xd, L.R, L.S, st, st, pd, pd)
        t_total += time.perf_counter() - t0
        flops += 3 * 2 * n_images * L.P * L.Q * L.K * L.C * L.R * L.S
    desc = (f"batch slice of {n_images} of {wl.layers[0].N} images, layers {list(layers)} of {wl.name}: "
            "quantize X/W/G_Y + fwd + dgrad + wgrad in double")
    return flops, t_total, orc.num_threads(), desc


def arm_config(wl, world):
    """The `config` object both arms print: the workload, its sizes and formats."""
    L0 = wl.layers[0]
    return {"workload": wl.name, "layers": len(wl.layers), "global_batch": L0.N * world,
            "input": f"{L0.C}x{L0.H}x{L0.W}", "block": "SQ32", "formats": "X,W e4m3; G_Y e5m2",
            "l2": "inputs larger than L2 (step working set well above 126 MB); no flush",
            "parallelism": f"dp{world}"}


def reference_arm(args):
    world, rank, local = dist_env()
    if rank != 0:
        return 0
    wl = synth.WORKLOADS[WORKLOAD_CFG]
    # bounded sample: the smallest-work layers first, sized for a few minutes in total
    per_step_layers = list(range(len(wl.layers)))
    flops_list, secs = [], []
    for step in range(args.warmup + args.steps):
        f, t, cores, desc = oracle_sample(wl, 1, per_step_layers)
        if step >= args.warmup:
            flops_list.append(f)
            secs.append(t)
    tot_f, tot_t = sum(flops_list), sum(secs)
    value = tot_f / tot_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / max(1, len(secs)),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(arm_config(wl, world), sample=desc),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_by_name(name: str) -> synth.Workload:
    if ":" in name:
        cfg, fmt, n = name.split(":")
        return synth.WORKLOADS[(int(cfg), fmt, int(n))]
    return synth.WORKLOADS[int(name)]


CALLS = ("quantize_x", "quantize_w", "quantize_g", "fwd", "dgrad", "wgrad")


def capture_graph(torch, fn):
    """One CUDA graph of `fn` (C-ABI calls on the capturing stream): replaying
    it runs the same kernels without the host's per-call argument marshalling
    and tensor-map encoding between launches."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        fn()
    return g


def graph_call_times(mqc, torch, lb, workspace, reps, names=CALLS, k=8, nxt=None):
    """Device time (ms) of each named call of one layer, launch cost
    amortised: one CUDA graph holds k (L2 flush, call) pairs, another the k
    flushes alone (a 256 MiB write each, larger than the 126 MB L2); each is
    replayed `reps` times between a pair of events and the call's time is
    (median with calls - median of flushes) / k.  Returns lists of per-call
    estimates (one per replay pair)."""
    cur = lambda: ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def body(name):
        for _ in range(k):
            flush.fill_(1)
            if name is not None:
                run_layer(mqc, lb, workspace, cur(), only=(name,), nxt=nxt if name == "fwd_quant" else None)

    def timed(g):
        out = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            out.append((e0, e1))
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in out]

    g_flush = capture_graph(torch, lambda: body(None))
    g_flush.replay()
    t_flush = statistics.median(timed(g_flush))
    out = {}
    for name in names:
        g = capture_graph(torch, lambda: body(name))
        g.replay()
        out[name] = [max(1e-6, (t - t_flush) / k) for t in timed(g)]
        del g
    del g_flush
    mqc.check(mqc.get_device_status())
    return out


def graph_fn_times(mqc, torch, fn, reps, k=8):
    """graph_call_times for any callable that issues C-ABI calls on the
    current stream: (median of k (flush, fn) pairs - median of k flushes) / k."""
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def body(with_fn):
        for _ in range(k):
            flush.fill_(1)
            if with_fn:
                fn()

    def timed(g):
        out = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            out.append((e0, e1))
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in out]

    gf = capture_graph(torch, lambda: body(False))
    gf.replay()
    t_flush = statistics.median(timed(gf))
    g = capture_graph(torch, lambda: body(True))
    g.replay()
    out = [max(1e-6, (t - t_flush) / k) for t in timed(g)]
    del g, gf
    mqc.check(mqc.get_device_status())
    return out


def quantize_weights(mqc, layers, stream):
    """Every layer's weights in one launch (mqc_quantize_mx_batch): the
    weights are quantized together once per weight update."""
    P = lambda t: t.data_ptr()
    qs = [lb.q["w"] for lb in layers]
    mqc.check(mqc.mqc_quantize_mx_batch([P(lb.w) for lb in layers], [lb.desc["w"] for lb in layers], qs[0].mx,
                                        [P(q.codes) for q in qs], [P(q.scales) for q in qs],
                                        [P(q.codes_alt) for q in qs], stream))


def sweep(mqc, torch, wl, args):
    """Per-call times of every layer of a workload, with roofline fractions."""
    pk = peaks()
    fp8_peak = 2.0 * pk["bf16_tflops"]
    out = []
    for i, L in enumerate(wl.layers):
        lb = LayerBuffers(mqc, torch, L, wl, i, False)
        workspace = torch.empty(max(lb.ws_bytes, 16), dtype=torch.uint8, device="cuda")
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        for _ in range(2):
            run_layer(mqc, lb, workspace, stream)
        per = graph_call_times(mqc, torch, lb, workspace, max(3, args.reps))
        for name, v in per.items():
            ms = statistics.median(v)
            if name.startswith("quantize"):
                byt, fl = lb.quant_bytes(name[-1]), 0
            else:
                byt, fl = lb.gemm_bytes(name), lb.gemm_flops()
            t_roof = max(byt / (pk["hbm_gbs"] * 1e9), fl / (fp8_peak * 1e12))
            out.append({"workload": wl.name, "layer": i, "call": name, "ms": round(ms, 5),
                        "tflops": round(fl / (ms * 1e-3) / 1e12, 1) if fl else None,
                        "gbs": round(byt / (ms * 1e-3) / 1e9, 1),
                        "frac_of_roofline": round(1e3 * t_roof / ms, 4),
                        "frac_of_mxfp8_peak": round(fl / (ms * 1e-3) / 1e12 / fp8_peak, 4) if fl else None})
        # the explicit channel-batch-first im2col of quantized X (the GEMMs
        # never call it): HBM-bound, source codes + scales read once and the
        # expansion written once, timed after a 256 MiB L2 flush
        xq = lb.q["x"]
        nc = mqc.lib.mqc_im2col_cbf_codes_bytes(ctypes.byref(lb.cv), ctypes.byref(xq.mx))
        ns = mqc.lib.mqc_im2col_cbf_scales_bytes(ctypes.byref(lb.cv), ctypes.byref(xq.mx))
        co = torch.empty(max(nc, 16), dtype=torch.uint8, device="cuda")
        so = torch.empty(max(ns, 16), dtype=torch.uint8, device="cuda")
        ptr = lambda t: ctypes.c_void_p(t.data_ptr())
        call = lambda: mqc.check(mqc.mqc_im2col_cbf(ptr(xq.codes), ptr(xq.scales), lb.cv, xq.mx, ptr(co), ptr(so),
                                                   stream))
        call()
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        ts = []
        for _ in range(max(3, args.reps)):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            call()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        ms = statistics.median(ts)
        byt = xq.codes.numel() + xq.scales.numel() + nc + ns
        out.append({"workload": wl.name, "layer": i, "call": "im2col_x", "ms": round(ms, 5), "tflops": None,
                    "gbs": round(byt / (ms * 1e-3) / 1e9, 1),
                    "frac_of_roofline": round(byt / (pk["hbm_gbs"] * 1e9) * 1e3 / ms, 4), "frac_of_mxfp8_peak": None})
        del lb, workspace, co, so, flush
        torch.cuda.empty_cache()
    for o in out:
        print(json.dumps(o), flush=True)
    return 0


# --------------------------------------------------------------------------- profiling driver
def profile_call(mqc, torch, wl, args):
    """Runs one layer's calls once (so every operand exists), then the chosen
    call `reps` more times; used as the small case of an ncu capture."""
    lb = LayerBuffers(mqc, torch, wl.layers[args.layer], wl, args.layer, False)
    names = tuple(args.profile.split(","))
    # fwd_quant writes the next layer's quantized input
    nxt = (LayerBuffers(mqc, torch, wl.layers[args.layer + 1], wl, args.layer + 1, False)
           if "fwd_quant" in names else None)
    workspace = torch.empty(max(lb.ws_bytes, 16), dtype=torch.uint8, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    run_layer(mqc, lb, workspace, stream)
    events = []
    for _ in range(args.reps):
        run_layer(mqc, lb, workspace, stream, events, only=names, nxt=nxt)
    torch.cuda.synchronize()
    mqc.check(mqc.get_device_status())
    ms = [e0.elapsed_time(e1) for _, e0, e1 in events]
    print(json.dumps({"profile": args.profile, "layer": args.layer, "ms": ms}), flush=True)
    return 0


# --------------------------------------------------------------------------- extras
def fused_step(mqc, torch, args, layers, workspace, layer_calls, allreduce_gw, step_flops, pk, world):
    """The training step with quantize-in-epilogue (the paper's section V /
    Fig. 4 flow): forwards 0-6 apply SiLU and write the next layer's SQ32
    E4M3 codes (both orders) and scales, so layers 1-7 skip quantize_x and
    no fp32 activation is written.  Same flops as the step; its own graph,
    timed like the step, plus the per-call time of every fused forward."""
    g = capture_graph(torch, lambda: layer_calls(fused=True))
    for _ in range(max(3, args.warmup)):
        g.replay()
        allreduce_gw()
    torch.cuda.synchronize()
    mqc.check(mqc.get_device_status())
    barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        g.replay()
        allreduce_gw()
    t1.record()
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, torch.device("cuda"))
    mqc.check(mqc.get_device_status())
    del g
    calls = []
    for i in range(len(layers) - 1):
        lb, nxt = layers[i], layers[i + 1]
        t = statistics.median(graph_call_times(mqc, torch, lb, workspace, 5, names=("fwd_quant",), nxt=nxt)["fwd_quant"])
        byt = lb.gemm_bytes("fwd_quant", nxt)
        calls.append({"layer": i, "call": "fwd_quant", "ms": round(t, 5), "bytes": byt,
                      "frac_of_hbm_roofline": round(byt / (pk["hbm_gbs"] * 1e9) * 1e3 / t, 4)})
    # one batched weight launch; layers 1-7 have no quantize_x
    launches = sum(lb.launches(mqc) for lb in layers) - 2 * (len(layers) - 1)
    return {"value": world * step_flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms,
            "gpu_launches_per_step": launches,
            "what": "forwards 0-6 quantize their SiLU output in the epilogue as the next layer's SQ32 E4M3 input "
                    "(both orders); layers 1-7 skip quantize_x; no fp32 activation written",
            "calls": calls}


TENSOR_BOUND = ((4, "latent-replay N=128 C=K=256 14x14, X E2M1, W E4M3, G_Y E5M2"),
                ((5, "fp8", 128), "large-batch N=128 C=K=128 80x80 MXFP8"),
                ((5, "fp4", 128), "large-batch N=128 C=K=128 80x80 MXFP4"))


def tensor_bound_layers(mqc, torch, pk):
    """Per-call TFLOP/s of the three GEMMs on the tensor-bound configurations
    (latent-replay block, large-batch layer at N=128 in MXFP8 and MXFP4) as
    fractions of the dense MXFP8 peak (2 x the measured bf16 peak) and, for
    all-FP4 operands, of the dense MXFP4 peak (2 x MXFP8, the nominal ratio)."""
    fp8_peak = 2.0 * pk["bf16_tflops"]
    out = []
    for key, what in TENSOR_BOUND:
        wl = synth.WORKLOADS[key]
        lb = LayerBuffers(mqc, torch, wl.layers[0], wl, 0, False)
        ws = torch.empty(max(lb.ws_bytes, 16), dtype=torch.uint8, device="cuda")
        run_layer(mqc, lb, ws, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        per = graph_call_times(mqc, torch, lb, ws, 5, names=("fwd", "dgrad", "wgrad"), k=4)
        all_fp4 = wl.fmt_x == wl.fmt_w == wl.fmt_g == synth.E2M1
        for name, v in per.items():
            ms = statistics.median(v)
            tf = lb.gemm_flops() / (ms * 1e-3) / 1e12
            out.append({"workload": wl.name, "what": what, "call": name, "ms": round(ms, 5), "tflops": round(tf, 1),
                        "frac_of_mxfp8_peak": round(tf / fp8_peak, 4),
                        "frac_of_mxfp4_peak": round(tf / (2 * fp8_peak), 4) if all_fp4 else None})
        del lb, ws
        torch.cuda.empty_cache()
    # NVFP4 (the paper's own format) forward on the large-batch layer: X and W
    # quantized with 16 x 16 squares, tcgen05 kind::mxf4nvf4 on packed codes
    wl = synth.WORKLOADS[(5, "fp4", 128)]
    L = wl.layers[0]
    x, w, _ = synth.layer_inputs(wl, 0)
    xq = mqc.quantize_nvfp4(torch.from_numpy(x).cuda(), mqc.NV_SQ16, 0)
    wq = mqc.quantize_nvfp4(torch.from_numpy(w).cuda(), mqc.NV_SQ16, 0)
    cv = mqc.conv_desc(L.N, L.C, L.H, L.W, L.K, L.R, L.S, L.stride, L.pad)
    y = torch.empty((L.N, L.K, L.P, L.Q), dtype=torch.float32, device="cuda")
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    fwd = lambda: mqc.check(mqc.lib.mqc_conv2d_fwd_nvfp4(
        ptr(xq.codes), ptr(xq.scales), ptr(xq.tscale), mqc.NV_SQ16, ptr(wq.codes), ptr(wq.scales), ptr(wq.tscale),
        mqc.NV_SQ16, ctypes.byref(cv), ptr(y), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)))
    fwd()
    ms = statistics.median(graph_fn_times(mqc, torch, fwd, 5, k=4))
    tf = L.gemm_flops() / (ms * 1e-3) / 1e12
    out.append({"workload": "large-batch-nvfp4-n128-c128-80x80",
                "what": "large-batch N=128 C=K=128 80x80, X and W NVFP4 (E2M1, E4M3 scales per 16x16, fp32 tensor scale)",
                "call": "fwd", "ms": round(ms, 5), "tflops": round(tf, 1), "frac_of_mxfp8_peak": round(tf / fp8_peak, 4),
                "frac_of_mxfp4_peak": round(tf / (2 * fp8_peak), 4)})
    del xq, wq, y
    torch.cuda.empty_cache()
    return out


# --------------------------------------------------------------------------- main arm
def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return reference_arm(args)
    world, rank, local = dist_env()
    import torch
    torch.cuda.set_device(local)
    init_dist(world, "nccl")
    import im2col_gemm_b200 as mqc

    wl = synth.WORKLOADS[WORKLOAD_CFG]
    if args.profile or args.sweep:
        wl = workload_by_name(args.workload)
        if args.sweep:
            return sweep(mqc, torch, wl, args)
        return profile_call(mqc, torch, wl, args)
    pk = peaks()
    want_host = not args.skip_e2e
    layers = [LayerBuffers(mqc, torch, L, wl, i, want_host) for i, L in enumerate(wl.layers)]
    ws_max = max(lb.ws_bytes for lb in layers)
    workspace = torch.empty(max(ws_max, 16), dtype=torch.uint8, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    step_flops = sum(3 * lb.gemm_flops() for lb in layers)
    # one batched launch quantizes every layer's weights
    launches_per_step = sum(lb.launches(mqc) for lb in layers) - (len(layers) - 1)
    gws = [lb.gw for lb in layers]

    def allreduce_gw():
        allreduce_weight_grads(gws)

    def cur_stream():
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    wstream = torch.cuda.Stream()
    rest = tuple(c for c in CALLS if c != "quantize_w") + ("fwd_quant",)

    def layer_calls(events=None, fused=False):
        # the weights are known when the step starts (as right after a weight
        # update), so their quantizations run on a second stream, overlapping
        # the activation work; each layer's GEMMs wait for its own weights.
        # fused: each forward but the last applies SiLU and writes the next
        # layer's quantized input in its epilogue (section V / Fig. 4 of the
        # paper), so layers 1-7 have no quantize_x and no fp32 activation
        # is written or read again
        main = torch.cuda.current_stream()
        fork = torch.cuda.Event()
        fork.record(main)
        wstream.wait_event(fork)
        with torch.cuda.stream(wstream):
            quantize_weights(mqc, layers, cur_stream())
            ready = torch.cuda.Event()
            ready.record(wstream)
        for i, lb in enumerate(layers):
            if i == 0:
                main.wait_event(ready)
            nxt = layers[i + 1] if fused and i + 1 < len(layers) else None
            run_layer(mqc, lb, workspace, cur_stream(), events, only=rest, nxt=nxt, with_x=not fused or i == 0)

    def step(events=None):
        layer_calls(events)
        allreduce_gw()


    # clocks are sampled from the start of the warm-up to the end of the timed
    # region (nvidia-smi needs a few hundred ms to produce its first sample)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.5)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    mqc.check(mqc.get_device_status())
    # the step's kernels as one CUDA graph (the weight-gradient all-reduce of
    # a multi-GPU run stays outside it)
    step_graph = capture_graph(torch, layer_calls)
    for _ in range(args.warmup):
        step_graph.replay()
        allreduce_gw()
    torch.cuda.synchronize()
    mqc.check(mqc.get_device_status())

    # ---- timed region: inputs resident in HBM
    barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        step_graph.replay()
        allreduce_gw()
    t1.record()
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = t0.elapsed_time(t1) / args.steps
    ms = max_over_ranks(ms, torch.device("cuda"))
    mqc.check(mqc.get_device_status())
    value = world * step_flops / (ms * 1e-3) / 1e12

    # per-call durations: each call as its own graph (cold L2, no host gaps)
    per = {}
    for li, lb in enumerate(layers):
        for name, v in graph_call_times(mqc, torch, lb, workspace, max(3, min(args.steps, 10)),
                                        names=tuple(c for c in CALLS if c != "quantize_w")).items():
            per[(li, name)] = v
    cur = lambda: ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    per[("all", "quantize_w")] = graph_fn_times(mqc, torch, lambda: quantize_weights(mqc, layers, cur()),
                                                max(3, min(args.steps, 10)))
    calls = []
    for (li, name), v in per.items():
        d = statistics.mean(v)
        if li == "all":
            byt = sum(lb.quant_bytes("w") for lb in layers)
            calls.append({"layer": "all", "call": name, "ms": d, "bytes": byt, "flops": 0})
            continue
        lb = layers[li]
        if name.startswith("quantize"):
            byt = lb.quant_bytes(name[-1])
            calls.append({"layer": li, "call": name, "ms": d, "bytes": byt, "flops": 0})
        else:
            calls.append({"layer": li, "call": name, "ms": d, "bytes": lb.gemm_bytes(name), "flops": lb.gemm_flops()})
    fp8_peak = 2.0 * pk["bf16_tflops"]          # MXFP8 dense = 2x bf16 (nominal ratio) x measured bf16
    for c in calls:
        t_hbm = c["bytes"] / (pk["hbm_gbs"] * 1e9)
        t_tc = c["flops"] / (fp8_peak * 1e12) if c["flops"] else 0.0
        c["bound"] = "tensor" if t_tc > t_hbm else "hbm"
        c["roofline_ms"] = 1e3 * max(t_hbm, t_tc)
        c["frac"] = c["roofline_ms"] / c["ms"]
    total_call_ms = sum(c["ms"] for c in calls)
    top = max(calls, key=lambda c: c["ms"])
    if top["bound"] == "hbm":
        achieved = top["bytes"] / (top["ms"] * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"]}
    else:
        achieved = top["flops"] / (top["ms"] * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": fp8_peak, "unit": "TFLOP/s",
                "frac": achieved / fp8_peak}
    top_name = f"{top['call']} layer {top['layer']}"
    roof.update({"traffic": measured_traffic(top_name), "kernel": top_name,
                 "share": top["ms"] / total_call_ms, "peak_source": pk["source"] + " (MXFP8 = 2 x bf16)"
                 if roof["bound"] == "tensor" else pk["source"]})
    qcalls = [c for c in calls if c["call"].startswith("quantize")]
    quant_gbs = sum(c["bytes"] for c in qcalls) / (sum(c["ms"] for c in qcalls) * 1e-3) / 1e9

    # ---- end to end: host fp32 inputs -> device -> step -> outputs back to host
    e2e = None
    if not args.skip_e2e:
        h2d = sum(h.numel() * h.element_size() for lb in layers for h in lb.host_in)
        d2h = sum(h.numel() * h.element_size() for lb in layers for h in lb.host_out)
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            for lb in layers:
                for dst, src in zip((lb.x, lb.w, lb.g), lb.host_in):
                    dst.copy_(src, non_blocking=True)
            step()      # the 48 C-ABI calls of the step, issued one by one from the host
            for lb in layers:
                for dst, src in zip(lb.host_out, (lb.y, lb.gx, lb.gw)):
                    dst.copy_(src, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        barrier()
        ems = max_over_ranks(e0.elapsed_time(e1) / args.steps, torch.device("cuda"))
        e2e = {"value": world * step_flops / (ems * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ems,
               "how": "fp32 X, W, G_Y of every layer copied from pinned host memory, the step's C-ABI calls "
                      "issued one by one (no graph), Y, G_X, G_W copied back, every step"}

    # ---- extras: the fused step, the tensor-bound layers, the stochastic-rounding quantizer
    fused = tensor_bound = sr_quant = None
    if not args.skip_extras:
        fused = fused_step(mqc, torch, args, layers, workspace, layer_calls, allreduce_gw, step_flops, pk, world)
        for c in fused["calls"]:       # what the fused forward replaces: the fp32 forward + the next quantize_x
            c["ms_unfused"] = round(statistics.mean(per[(c["layer"], "fwd")])
                                    + statistics.mean(per[(c["layer"] + 1, "quantize_x")]), 5)
        tensor_bound = tensor_bound_layers(mqc, torch, pk)
        lb0 = layers[0]
        t_sr = statistics.median(graph_call_times(mqc, torch, lb0, workspace, 5, names=("quantize_g_sr",))
                                 ["quantize_g_sr"])
        t_rn = statistics.median(graph_call_times(mqc, torch, lb0, workspace, 5, names=("quantize_g",))["quantize_g"])
        byt = lb0.quant_bytes("g")
        sr_quant = {"call": "quantize_g_sr layer 0", "ms": t_sr, "gbs": byt / (t_sr * 1e-3) / 1e9,
                    "frac_of_hbm": byt / (t_sr * 1e-3) / 1e9 / pk["hbm_gbs"], "ms_round_to_nearest": t_rn,
                    "what": "G_Y 16x32x320x320 fp32 -> E5M2 SQ32, both orders, elements rounded stochastically "
                            "with Philox4x64-10 bits"}

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        f, t, cores, desc = oracle_sample(wl, 4)
        cpu = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc,
               "seconds": t}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "mxfp8 (e4m3/e5m2 x e8m0) -> fp32", "data": "synthetic",
            "config": arm_config(wl, world),
            "quantizer_gbs": quant_gbs, "quantizer_frac_of_hbm": quant_gbs / pk["hbm_gbs"],
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
            "fused_step": fused, "tensor_bound": tensor_bound, "sr_quantizer": sr_quant,
            "calls": [{k: (round(v, 5) if isinstance(v, float) else v) for k, v in c.items()} for c in calls],
        }
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
