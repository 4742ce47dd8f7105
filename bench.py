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
        self.path = os.path.join(ROOT, "gpurun_out", f"clocks_rank{gpu_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
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

    def gemm_bytes(self, op):
        qx, qw, qg = self.q["x"], self.q["w"], self.q["g"]
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


def run_layer(mqc, lb: LayerBuffers, workspace, stream, events=None, only=None):
    """All calls of one layer through the C ABI; `events` (optional) collects
    (name, start, end) CUDA events around every call on `stream`; `only`
    (a tuple of call names) restricts the run to those calls (profiling)."""
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
        q = lb.q[name]
        timed(f"quantize_{name}", lambda q=q, t=t, name=name: mqc.mqc_quantize_mx(
            P(t), lb.desc[name], q.mx, P(q.codes), P(q.scales), P(q.codes_alt), stream))
    qx, qw, qg = lb.q["x"], lb.q["w"], lb.q["g"]
    wq_ab, gq_ab, xq_ab = qw.other_order(), qg.other_order(), qx.other_order()
    wsp = P(workspace) if lb.ws_bytes else None
    timed("fwd", lambda: mqc.mqc_conv2d_fwd(P(qx.codes), P(qx.scales), qx.mx, P(qw.codes), P(qw.scales), qw.mx,
                                            lb.cv, P(lb.y), wsp, lb.ws_fwd, stream))
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


def graph_call_times(mqc, torch, lb, workspace, reps, names=CALLS):
    """Device time (ms) of each named call of one layer: the call captured as
    a CUDA graph and replayed `reps` times, each replay between a pair of
    events and preceded by an L2 flush (a 256 MiB write)."""
    cur = lambda: ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    out = {}
    for name in names:
        g = capture_graph(torch, lambda: run_layer(mqc, lb, workspace, cur(), only=(name,)))
        g.replay()
        ev = []
        for _ in range(reps):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            ev.append((e0, e1))
        torch.cuda.synchronize()
        out[name] = [a.elapsed_time(b) for a, b in ev]
        del g
    mqc.check(mqc.get_device_status())
    return out


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
    workspace = torch.empty(max(lb.ws_bytes, 16), dtype=torch.uint8, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    run_layer(mqc, lb, workspace, stream)
    events = []
    for _ in range(args.reps):
        run_layer(mqc, lb, workspace, stream, events, only=tuple(args.profile.split(",")))
    torch.cuda.synchronize()
    mqc.check(mqc.get_device_status())
    ms = [e0.elapsed_time(e1) for _, e0, e1 in events]
    print(json.dumps({"profile": args.profile, "layer": args.layer, "ms": ms}), flush=True)
    return 0


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
    launches_per_step = sum(lb.launches(mqc) for lb in layers)
    gws = [lb.gw for lb in layers]

    def allreduce_gw():
        allreduce_weight_grads(gws)

    def cur_stream():
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    wstream = torch.cuda.Stream()
    rest = tuple(c for c in CALLS if c != "quantize_w")

    def layer_calls(events=None):
        # the weights are known when the step starts (as right after a weight
        # update), so their quantizations run on a second stream, overlapping
        # the activation work; each layer's GEMMs wait for its own weights
        main = torch.cuda.current_stream()
        fork = torch.cuda.Event()
        fork.record(main)
        wstream.wait_event(fork)
        ready = []
        with torch.cuda.stream(wstream):
            for lb in layers:
                run_layer(mqc, lb, workspace, cur_stream(), only=("quantize_w",))
                ev = torch.cuda.Event()
                ev.record(wstream)
                ready.append(ev)
        for lb, ev in zip(layers, ready):
            main.wait_event(ev)
            run_layer(mqc, lb, workspace, cur_stream(), events, only=rest)

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
        for name, v in graph_call_times(mqc, torch, lb, workspace, max(3, min(args.steps, 10))).items():
            per[(li, name)] = v
    calls = []
    for (li, name), v in per.items():
        lb = layers[li]
        d = statistics.mean(v)
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
            step_graph.replay()
            allreduce_gw()
            for lb in layers:
                for dst, src in zip(lb.host_out, (lb.y, lb.gx, lb.gw)):
                    dst.copy_(src, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        barrier()
        ems = max_over_ranks(e0.elapsed_time(e1) / args.steps, torch.device("cuda"))
        e2e = {"value": world * step_flops / (ems * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ems}

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
            "calls": [{k: (round(v, 5) if isinstance(v, float) else v) for k, v in c.items()} for c in calls],
        }
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
