"""Seeded synthetic inputs and workload shapes for the MicroQonv hot path.

This module is shared by the tests, the smoke check and the benchmark, and it
feeds both the CUDA library and the oracle.  It holds NO arithmetic of the
method (no quantization, no im2col, no convolution): only layer shapes, the
MX formats each tensor uses, and seeded random fp32 tensors with the value
distributions of the paper's workloads (post-activation feature maps, small
weights, small output gradients, heavy-tailed stress inputs).

The paper trains on CIFAR-100, ImageNet-100, PascalVOC and KITTI with ResNet
and YOLO networks; none of those datasets or weights are used.  Seeded
synthetic layers with the same tensor shapes stand in for them.

Generator: numpy PCG64 (``numpy.random.default_rng(seed)``).  Seeds: for the
layer ``i`` of configuration ``cfg``, X uses ``1000*cfg + 10*i``, W that plus
1 and G_Y that plus 2.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# element formats, block modes (same small integers as the C ABI)
E4M3, E5M2, E2M1 = 0, 1, 2
A32, B32, SQ32 = 0, 1, 2
FMT_NAME = {E4M3: "e4m3", E5M2: "e5m2", E2M1: "e2m1"}


@dataclass(frozen=True)
class Layer:
    """One convolution layer: X [N][C][H][W], W [K][C][R][S], stride, padding."""
    N: int
    C: int
    H: int
    W: int
    K: int
    R: int
    S: int
    stride: int = 1
    pad: int = 0

    @property
    def P(self) -> int:
        return (self.H + 2 * self.pad - self.R) // self.stride + 1

    @property
    def Q(self) -> int:
        return (self.W + 2 * self.pad - self.S) // self.stride + 1

    def gemm_flops(self) -> int:
        """2*M*N*K of one of the three GEMMs (they all have the same count)."""
        return 2 * self.N * self.P * self.Q * self.K * self.C * self.R * self.S


@dataclass(frozen=True)
class Workload:
    name: str
    cfg: int
    layers: tuple
    fmt_x: int
    fmt_w: int
    fmt_g: int
    block: int               # block mode used for the product path
    backward: bool           # fwd only, or fwd + dgrad + wgrad
    dist: str                # "normal", "silu", "relu", "student_t"
    w_std: float = 1.0
    g_std: float = 1e-3
    note: str = ""


def _yolo_stack(N: int = 16, size: int = 640):
    """YOLOv8n-shaped backbone stem at the literal reading of the workload:
    3x3 stride-2 convs C 16->32->64->128->256 each followed by a 1x1 conv."""
    layers = []
    c, hw = 16, size
    for cout in (32, 64, 128, 256):
        layers.append(Layer(N, c, hw, hw, cout, 3, 3, 2, 1))
        hw = (hw + 2 - 3) // 2 + 1
        layers.append(Layer(N, cout, hw, hw, cout, 1, 1, 1, 0))
        c = cout
    return tuple(layers)


WORKLOADS = {
    1: Workload("single-conv-n2-c32-8x8", 1, (Layer(2, 32, 8, 8, 32, 3, 3, 1, 1),),
                E4M3, E4M3, E5M2, A32, False, "normal", 1.0),
    2: Workload("yolov8n-stack-fwd-n16-640", 2, _yolo_stack(), E4M3, E4M3, E5M2, A32, False, "silu", 0.02),
    3: Workload("yolov8n-stack-train-n16-640", 3, _yolo_stack(), E4M3, E4M3, E5M2, SQ32, True, "silu", 0.02),
    4: Workload("latent-replay-n128-c256-14x14", 4, (Layer(128, 256, 14, 14, 256, 3, 3, 1, 1),),
                E2M1, E4M3, E5M2, SQ32, True, "relu", 0.02),
}
for _n in (32, 64, 128, 256):
    WORKLOADS[(5, "fp8", _n)] = Workload(f"large-batch-mxfp8-n{_n}-c128-80x80", 5,
                                         (Layer(_n, 128, 80, 80, 128, 3, 3, 1, 1),),
                                         E4M3, E4M3, E5M2, SQ32, True, "student_t", 1.0)
    WORKLOADS[(5, "fp4", _n)] = Workload(f"large-batch-mxfp4-n{_n}-c128-80x80", 5,
                                         (Layer(_n, 128, 80, 80, 128, 3, 3, 1, 1),),
                                         E2M1, E2M1, E2M1, SQ32, True, "student_t", 1.0)


def seeds(cfg: int, i: int) -> tuple[int, int, int]:
    base = 1000 * cfg + 10 * i
    return base, base + 1, base + 2


def _normal(rng, shape) -> np.ndarray:
    return rng.standard_normal(size=shape, dtype=np.float32)


def _student_t(rng, shape, dof=3.0) -> np.ndarray:
    out = np.empty(int(np.prod(shape)), dtype=np.float32)
    step = 1 << 24
    for i in range(0, out.size, step):
        out[i:i + step] = rng.standard_t(dof, size=min(step, out.size - i))
    return out.reshape(shape)


def activation(shape, seed: int, dist: str) -> np.ndarray:
    """Input feature map [N][C][H][W] with the workload's value distribution."""
    rng = np.random.default_rng(seed)
    if dist == "student_t":
        return _student_t(rng, shape)
    x = _normal(rng, shape)
    if dist == "silu":          # post-SiLU feature maps: x * sigmoid(x)
        x = x / (np.float32(1.0) + np.exp(-x))
    elif dist == "relu":        # non-negative post-ReLU feature maps
        np.maximum(x, np.float32(0.0), out=x)
    return x.astype(np.float32, copy=False)


def weight(shape, seed: int, dist: str, std: float) -> np.ndarray:
    rng = np.random.default_rng(seed)
    if dist == "student_t":
        return _student_t(rng, shape)
    w = _normal(rng, shape)
    if std != 1.0:
        w *= np.float32(std)
    return w


def grad(shape, seed: int, dist: str, std: float) -> np.ndarray:
    rng = np.random.default_rng(seed)
    g = _student_t(rng, shape) if dist == "student_t" else _normal(rng, shape)
    g *= np.float32(std)
    return g


def layer_inputs(wl: Workload, i: int, n_override: int | None = None):
    """(X, W, G_Y) fp32 arrays for layer i of a workload (G_Y None if fwd only)."""
    L = wl.layers[i]
    N = L.N if n_override is None else n_override
    sx, sw, sg = seeds(wl.cfg, i)
    x = activation((N, L.C, L.H, L.W), sx, wl.dist)
    w = weight((L.K, L.C, L.R, L.S), sw, wl.dist, wl.w_std)
    g = grad((N, L.K, L.P, L.Q), sg, wl.dist, wl.g_std) if wl.backward else None
    return x, w, g


def random_tensor(shape, seed: int, dist: str = "normal", scale: float = 1.0) -> np.ndarray:
    """Generic seeded tensor for property and edge-case tests."""
    rng = np.random.default_rng(seed)
    if dist == "student_t":
        t = _student_t(rng, shape)
    elif dist == "uniform_exp":
        # magnitudes spread over many binades: sign * 2^U(-20, 20) * U(1, 2)
        e = rng.uniform(-20, 20, size=shape)
        m = rng.uniform(1, 2, size=shape)
        s = np.where(rng.random(size=shape) < 0.5, -1.0, 1.0)
        t = (s * m * np.exp2(e)).astype(np.float32)
    else:
        t = _normal(rng, shape)
    if scale != 1.0:
        t = t * np.float32(scale)
    return t.astype(np.float32, copy=False)
