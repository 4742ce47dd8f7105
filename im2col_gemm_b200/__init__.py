"""Python binding of libmqc, the B200 implementation of the MicroQonv hot path
("MicroQonv: Reshaping Convolution Tensors for Efficient Microscaling in
Training and Inference", arXiv:2609.28358).

Argument marshalling only: every computation runs in the CUDA kernels of
``libmqc.so`` (built from ``csrc/`` for sm_100a).  PyTorch supplies device
memory and the current stream.  There is no fallback: importing this module
fails loudly when the library is missing.

The ``mqc_*`` names mirror the C ABI in ``include/mqc.h`` one to one (raw
pointers, sizes, streams).  The lower-case helpers below them allocate the
output tensors with torch and call the same entry points.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmqc.so")

E4M3, E5M2, E2M1 = 0, 1, 2
A32, B32, SQ32 = 0, 1, 2
ORDER_BA, ORDER_AB = 0, 1
ROLE_X, ROLE_W, ROLE_G = 0, 1, 2

STATUS = {0: "MQC_OK", -1: "MQC_ERR_INVALID", -2: "MQC_ERR_UNSUPPORTED", -3: "MQC_ERR_CUDA",
          -4: "MQC_ERR_DEVICE_TIMEOUT", -5: "MQC_ERR_ALIGNMENT", -6: "MQC_ERR_WORKSPACE"}

# every symbol include/mqc.h declares
EXPORTS = ("mqc_codes_bytes", "mqc_scales_bytes", "mqc_tensor_dims", "mqc_quantize_mx", "mqc_im2col_cbf",
           "mqc_im2col_cbf_scales_bytes", "mqc_im2col_cbf_codes_bytes", "mqc_conv2d_fwd", "mqc_conv2d_bwd_data",
           "mqc_conv2d_bwd_weight", "mqc_conv2d_bwd_weight_workspace_bytes", "mqc_get_device_status",
           "mqc_debug_expire_wait", "mqc_status_string", "mqc_last_error_message", "mqc_version",
           "mqc_conv2d_bwd_weight_noalloc", "mqc_conv2d_fwd_workspace_bytes", "mqc_conv2d_bwd_data_workspace_bytes",
           "mqc_quantize_mx_sr", "mqc_conv2d_fwd_quant", "mqc_quantize_mx_batch", "mqc_quantize_nvfp4",
           "mqc_nvfp4_scales_bytes", "mqc_conv2d_fwd_nvfp4")
NV_A16, NV_B16, NV_SQ16 = 0, 1, 2
ACT_NONE, ACT_RELU, ACT_SILU = 0, 1, 2
NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


class MqcError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class T4(ctypes.Structure):
    _fields_ = [("d0", ctypes.c_int32), ("d1", ctypes.c_int32), ("d2", ctypes.c_int32), ("d3", ctypes.c_int32),
                ("s0", ctypes.c_int64), ("s1", ctypes.c_int64), ("s2", ctypes.c_int64), ("s3", ctypes.c_int64)]


class MX(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("block", ctypes.c_int32), ("order", ctypes.c_int32)]


class Conv(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("N", "C", "H", "W", "K", "R", "S", "stride_h", "stride_w",
                                               "pad_h", "pad_w")]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python im2col_gemm_b200/build.py` "
                          "(nvcc, sm_100a); there is no fallback implementation")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    P = ctypes.POINTER
    sig = {
        "mqc_codes_bytes": (i64, [P(MX), i32, i32, i32, i32]),
        "mqc_scales_bytes": (i64, [P(MX), i32, i32, i32, i32]),
        "mqc_tensor_dims": (i32, [i32, P(Conv), P(i32)]),
        "mqc_quantize_mx": (i32, [vp, P(T4), P(MX), vp, vp, vp, vp]),
        "mqc_quantize_mx_sr": (i32, [vp, P(T4), P(MX), vp, vp, vp, ctypes.c_uint64, ctypes.c_uint64, vp]),
        "mqc_quantize_mx_batch": (i32, [i32, P(vp), P(T4), P(MX), P(vp), P(vp), P(vp), vp]),
        "mqc_quantize_nvfp4": (i32, [vp, P(T4), i32, i32, vp, vp, vp, vp, vp]),
        "mqc_nvfp4_scales_bytes": (i64, [i32, i32, i32, i32, i32, i32]),
        "mqc_conv2d_fwd_nvfp4": (i32, [vp, vp, vp, i32, vp, vp, vp, i32, P(Conv), vp, vp]),
        "mqc_im2col_cbf": (i32, [vp, vp, P(Conv), P(MX), vp, vp, vp]),
        "mqc_im2col_cbf_scales_bytes": (i64, [P(Conv), P(MX)]),
        "mqc_im2col_cbf_codes_bytes": (i64, [P(Conv), P(MX)]),
        "mqc_conv2d_fwd": (i32, [vp, vp, P(MX), vp, vp, P(MX), P(Conv), vp, vp, sz, vp]),
        "mqc_conv2d_fwd_workspace_bytes": (sz, [P(Conv), P(MX), P(MX)]),
        "mqc_conv2d_fwd_quant": (i32, [vp, vp, P(MX), vp, vp, P(MX), P(Conv), i32, P(MX), vp, vp, vp, vp, vp, sz,
                                       vp]),
        "mqc_conv2d_bwd_data": (i32, [vp, vp, P(MX), vp, vp, P(MX), P(Conv), vp, vp, sz, vp]),
        "mqc_conv2d_bwd_data_workspace_bytes": (sz, [P(Conv), P(MX), P(MX)]),
        "mqc_conv2d_bwd_weight": (i32, [vp, vp, P(MX), vp, vp, P(MX), P(Conv), vp, vp, sz, vp]),
        "mqc_conv2d_bwd_weight_workspace_bytes": (sz, [P(Conv), P(MX), P(MX)]),
        "mqc_conv2d_bwd_weight_noalloc": (i32, [vp, vp, P(MX), vp, vp, P(MX), P(Conv), vp, vp]),
        "mqc_get_device_status": (i32, [vp]),
        "mqc_debug_expire_wait": (i32, [i64, vp]),
        "mqc_status_string": (ctypes.c_char_p, [i32]),
        "mqc_last_error_message": (ctypes.c_char_p, []),
        "mqc_version": (i32, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


lib = _load()


def check(status: int) -> None:
    if status != 0:
        raise MqcError(status, lib.mqc_last_error_message().decode())


# ------------------------------------------------------------------ C ABI, same names
def mqc_codes_bytes(mx: MX, d0, d1, d2, d3) -> int:
    return lib.mqc_codes_bytes(ctypes.byref(mx), d0, d1, d2, d3)


def mqc_scales_bytes(mx: MX, d0, d1, d2, d3) -> int:
    return lib.mqc_scales_bytes(ctypes.byref(mx), d0, d1, d2, d3)


def mqc_quantize_mx(src_ptr, desc: T4, mx: MX, codes_ptr, scales_ptr, codes_alt_ptr, stream) -> int:
    return lib.mqc_quantize_mx(src_ptr, ctypes.byref(desc), ctypes.byref(mx), codes_ptr, scales_ptr,
                               codes_alt_ptr, stream)


def mqc_quantize_mx_sr(src_ptr, desc: T4, mx: MX, codes_ptr, scales_ptr, codes_alt_ptr, seed, offset, stream) -> int:
    return lib.mqc_quantize_mx_sr(src_ptr, ctypes.byref(desc), ctypes.byref(mx), codes_ptr, scales_ptr,
                                  codes_alt_ptr, seed, offset, stream)


def mqc_quantize_mx_batch(srcs, descs, mx: MX, codes, scales, codes_alt, stream) -> int:
    """One launch for len(srcs) tensors; pointer lists (ints or c_void_p),
    T4 descriptors, one shared MX; codes_alt a list or None."""
    n = len(srcs)
    arr = lambda xs: (ctypes.c_void_p * n)(*[x.value if isinstance(x, ctypes.c_void_p) else x for x in xs])
    alt = arr(codes_alt) if codes_alt is not None else None
    return lib.mqc_quantize_mx_batch(n, arr(srcs), (T4 * n)(*descs), ctypes.byref(mx), arr(codes), arr(scales),
                                     alt, stream)


def mqc_im2col_cbf(codes_ptr, scales_ptr, conv: Conv, mx: MX, codes_out_ptr, scales_out_ptr, stream) -> int:
    return lib.mqc_im2col_cbf(codes_ptr, scales_ptr, ctypes.byref(conv), ctypes.byref(mx), codes_out_ptr,
                              scales_out_ptr, stream)


def mqc_conv2d_fwd(xq, xs, xf: MX, wq, ws, wf: MX, conv: Conv, y, workspace, workspace_bytes, stream) -> int:
    return lib.mqc_conv2d_fwd(xq, xs, ctypes.byref(xf), wq, ws, ctypes.byref(wf), ctypes.byref(conv), y, workspace,
                              workspace_bytes, stream)


def mqc_conv2d_fwd_quant(xq, xs, xf: MX, wq, ws, wf: MX, conv: Conv, act: int, yf: MX, yq, ys, yq_alt, y, workspace,
                         workspace_bytes, stream) -> int:
    return lib.mqc_conv2d_fwd_quant(xq, xs, ctypes.byref(xf), wq, ws, ctypes.byref(wf), ctypes.byref(conv), act,
                                    ctypes.byref(yf), yq, ys, yq_alt, y, workspace, workspace_bytes, stream)


def mqc_conv2d_fwd_workspace_bytes(conv: Conv, xf: MX, wf: MX) -> int:
    return lib.mqc_conv2d_fwd_workspace_bytes(ctypes.byref(conv), ctypes.byref(xf), ctypes.byref(wf))


def mqc_conv2d_bwd_data(wq, ws, wf: MX, gq, gs, gf: MX, conv: Conv, gx, workspace, workspace_bytes, stream) -> int:
    return lib.mqc_conv2d_bwd_data(wq, ws, ctypes.byref(wf), gq, gs, ctypes.byref(gf), ctypes.byref(conv), gx,
                                   workspace, workspace_bytes, stream)


def mqc_conv2d_bwd_data_workspace_bytes(conv: Conv, wf: MX, gf: MX) -> int:
    return lib.mqc_conv2d_bwd_data_workspace_bytes(ctypes.byref(conv), ctypes.byref(wf), ctypes.byref(gf))


def mqc_conv2d_bwd_weight(gq, gs, gf: MX, xq, xs, xf: MX, conv: Conv, gw, workspace, workspace_bytes,
                          stream) -> int:
    return lib.mqc_conv2d_bwd_weight(gq, gs, ctypes.byref(gf), xq, xs, ctypes.byref(xf), ctypes.byref(conv),
                                     gw, workspace, workspace_bytes, stream)


def mqc_conv2d_bwd_weight_workspace_bytes(conv: Conv, gf: MX, xf: MX) -> int:
    return lib.mqc_conv2d_bwd_weight_workspace_bytes(ctypes.byref(conv), ctypes.byref(gf), ctypes.byref(xf))


def mqc_conv2d_bwd_weight_noalloc(gq, gs, gf: MX, xq, xs, xf: MX, conv: Conv, gw, stream) -> int:
    """Weight gradient with the library's static split-K scratch: no workspace
    argument and no allocation (see include/mqc.h)."""
    return lib.mqc_conv2d_bwd_weight_noalloc(gq, gs, ctypes.byref(gf), xq, xs, ctypes.byref(xf),
                                             ctypes.byref(conv), gw, stream)


def mqc_get_device_status(stream) -> int:
    return lib.mqc_get_device_status(stream)


def mqc_debug_expire_wait(limit_ns: int, stream) -> int:
    return lib.mqc_debug_expire_wait(limit_ns, stream)


# ------------------------------------------------------------------ torch helpers
def _torch():
    import torch
    return torch


def _stream():
    torch = _torch()
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def conv_desc(N, C, H, W, K, R, S, stride=1, pad=0) -> Conv:
    sh, sw = (stride, stride) if isinstance(stride, int) else stride
    ph, pw = (pad, pad) if isinstance(pad, int) else pad
    return Conv(N, C, H, W, K, R, S, sh, sw, ph, pw)


def conv_out_hw(cv: Conv) -> tuple[int, int]:
    return ((cv.H + 2 * cv.pad_h - cv.R) // cv.stride_h + 1, (cv.W + 2 * cv.pad_w - cv.S) // cv.stride_w + 1)


def tensor_dims(role: int, cv: Conv) -> tuple[int, int, int, int]:
    d = (ctypes.c_int32 * 4)()
    check(lib.mqc_tensor_dims(role, ctypes.byref(cv), d))
    return tuple(d)


class Quantized:
    """Codes + scales of one tensor (device uint8 buffers) and how they are laid out."""

    def __init__(self, codes, scales, dims, mx: MX, codes_alt=None):
        self.codes, self.scales, self.dims, self.mx, self.codes_alt = codes, scales, tuple(dims), mx, codes_alt

    def other_order(self) -> "Quantized":
        """View of the second code order written by the same quantization."""
        if self.codes_alt is None:
            raise ValueError("quantized without the second code order")
        return Quantized(self.codes_alt, self.scales, self.dims, MX(self.mx.fmt, self.mx.block, 1 - self.mx.order),
                         self.codes)


def quantize_mx(src, fmt: int, block: int, order: int, both_orders: bool = False, sr_seed: int | None = None,
                sr_offset: int = 0) -> Quantized:
    """MX-quantize a 4-D fp32 CUDA tensor [d0=B][d1=A][d2][d3] (any strides);
    with `sr_seed`, the elements are rounded stochastically
    (mqc_quantize_mx_sr, order BA, NCHW-like source)."""
    torch = _torch()
    assert src.is_cuda and src.dtype == torch.float32 and src.dim() == 4
    d0, d1, d2, d3 = src.shape
    mx = MX(fmt, block, order)
    nc = mqc_codes_bytes(mx, d0, d1, d2, d3)
    ns = mqc_scales_bytes(mx, d0, d1, d2, d3)
    if nc < 0 or ns < 0:
        raise MqcError(-1, "bad quantization descriptor")
    codes = torch.empty(nc, dtype=torch.uint8, device=src.device)
    scales = torch.empty(ns, dtype=torch.uint8, device=src.device)
    alt = None
    if both_orders:
        alt = torch.empty(mqc_codes_bytes(MX(fmt, block, 1 - order), d0, d1, d2, d3), dtype=torch.uint8,
                          device=src.device)
    desc = T4(d0, d1, d2, d3, *src.stride())
    if sr_seed is None:
        check(mqc_quantize_mx(_ptr(src), desc, mx, _ptr(codes), _ptr(scales), _ptr(alt), _stream()))
    else:
        check(mqc_quantize_mx_sr(_ptr(src), desc, mx, _ptr(codes), _ptr(scales), _ptr(alt), sr_seed, sr_offset,
                                 _stream()))
    return Quantized(codes, scales, (d0, d1, d2, d3), mx, alt)


def quantize_mx_batch(srcs, fmt: int, block: int, order: int, both_orders: bool = False) -> list:
    """MX-quantize several 4-D fp32 CUDA tensors in one launch (same format,
    block mode and order): one Quantized per tensor."""
    torch = _torch()
    mx = MX(fmt, block, order)
    outs = []
    for src in srcs:
        assert src.is_cuda and src.dtype == torch.float32 and src.dim() == 4
        d = tuple(src.shape)
        codes = torch.empty(mqc_codes_bytes(mx, *d), dtype=torch.uint8, device=src.device)
        scales = torch.empty(mqc_scales_bytes(mx, *d), dtype=torch.uint8, device=src.device)
        alt = (torch.empty(mqc_codes_bytes(MX(fmt, block, 1 - order), *d), dtype=torch.uint8, device=src.device)
               if both_orders else None)
        outs.append(Quantized(codes, scales, d, mx, alt))
    descs = [T4(*s.shape, *s.stride()) for s in srcs]
    check(mqc_quantize_mx_batch([s.data_ptr() for s in srcs], descs, mx, [q.codes.data_ptr() for q in outs],
                                [q.scales.data_ptr() for q in outs],
                                [q.codes_alt.data_ptr() for q in outs] if both_orders else None, _stream()))
    return outs


class QuantizedNV(Quantized):
    """NVFP4 codes + E4M3 block scales + the per-tensor fp32 scale (a 2-float
    device buffer: [0] T, [1] scratch)."""

    def __init__(self, codes, scales, dims, block, order, tscale, codes_alt=None):
        super().__init__(codes, scales, dims, MX(E2M1, block, order), codes_alt)
        self.nv_block, self.tscale = block, tscale

    def other_order(self) -> "QuantizedNV":
        if self.codes_alt is None:
            raise ValueError("quantized without the second code order")
        return QuantizedNV(self.codes_alt, self.scales, self.dims, self.nv_block, 1 - self.mx.order, self.tscale,
                           self.codes)


def quantize_nvfp4(src, block: int, order: int, both_orders: bool = False) -> QuantizedNV:
    """NVFP4-quantize a 4-D fp32 CUDA tensor [d0=B][d1=A][d2][d3] (NCHW-like)."""
    torch = _torch()
    assert src.is_cuda and src.dtype == torch.float32 and src.dim() == 4
    d = tuple(src.shape)
    codes = torch.empty(mqc_codes_bytes(MX(E2M1, 0, order), *d), dtype=torch.uint8, device=src.device)
    scales = torch.empty(lib.mqc_nvfp4_scales_bytes(block, order, *d), dtype=torch.uint8, device=src.device)
    alt = (torch.empty(mqc_codes_bytes(MX(E2M1, 0, 1 - order), *d), dtype=torch.uint8, device=src.device)
           if both_orders else None)
    ts = torch.zeros(2, dtype=torch.float32, device=src.device)
    check(lib.mqc_quantize_nvfp4(_ptr(src), ctypes.byref(T4(*d, *src.stride())), block, order, _ptr(codes),
                                 _ptr(scales), _ptr(alt), _ptr(ts), _stream()))
    return QuantizedNV(codes, scales, d, block, order, ts, alt)


def conv2d_fwd_nvfp4(xq: QuantizedNV, wq: QuantizedNV, cv: Conv, out=None):
    """Forward convolution of NVFP4 operands on the tensor core (kind::mxf4nvf4)."""
    torch = _torch()
    P, Q = conv_out_hw(cv)
    y = out if out is not None else torch.empty((cv.N, cv.K, P, Q), dtype=torch.float32, device=xq.codes.device)
    check(lib.mqc_conv2d_fwd_nvfp4(_ptr(xq.codes), _ptr(xq.scales), _ptr(xq.tscale), xq.nv_block, _ptr(wq.codes),
                                   _ptr(wq.scales), _ptr(wq.tscale), wq.nv_block, ctypes.byref(cv), _ptr(y),
                                   _stream()))
    return y


def im2col_cbf(xq: Quantized, cv: Conv):
    """Explicit channel-batch-first im2col of quantized X: (codes, scales)."""
    torch = _torch()
    nc = lib.mqc_im2col_cbf_codes_bytes(ctypes.byref(cv), ctypes.byref(xq.mx))
    ns = lib.mqc_im2col_cbf_scales_bytes(ctypes.byref(cv), ctypes.byref(xq.mx))
    if nc < 0 or ns < 0:
        raise MqcError(-1, "bad im2col descriptor")
    co = torch.empty(nc, dtype=torch.uint8, device=xq.codes.device)
    so = torch.empty(ns, dtype=torch.uint8, device=xq.codes.device)
    check(mqc_im2col_cbf(_ptr(xq.codes), _ptr(xq.scales), cv, xq.mx, _ptr(co), _ptr(so), _stream()))
    return co, so


def conv2d_fwd(xq: Quantized, wq: Quantized, cv: Conv, out=None, workspace=None):
    torch = _torch()
    P, Q = conv_out_hw(cv)
    y = out if out is not None else torch.empty((cv.N, cv.K, P, Q), dtype=torch.float32, device=xq.codes.device)
    nws = mqc_conv2d_fwd_workspace_bytes(cv, xq.mx, wq.mx)
    if workspace is None and nws > 0:
        workspace = torch.empty(nws, dtype=torch.uint8, device=xq.codes.device)
    check(mqc_conv2d_fwd(_ptr(xq.codes), _ptr(xq.scales), xq.mx, _ptr(wq.codes), _ptr(wq.scales), wq.mx, cv,
                         _ptr(y), _ptr(workspace), nws, _stream()))
    return y


def conv2d_fwd_quant(xq: Quantized, wq: Quantized, cv: Conv, fmt: int, block: int, act: int = ACT_NONE,
                     both_orders: bool = False, keep_fp32: bool = False, workspace=None):
    """Forward convolution whose output is returned MX-quantized (order BA,
    and AB with `both_orders`) as the next layer's input: (Quantized, y)
    where y is the fp32 activated output when `keep_fp32`, else None."""
    torch = _torch()
    P, Q = conv_out_hw(cv)
    dev = xq.codes.device
    mx = MX(fmt, block, ORDER_BA)
    dims = (cv.N, cv.K, P, Q)
    codes = torch.empty(mqc_codes_bytes(mx, *dims), dtype=torch.uint8, device=dev)
    scales = torch.empty(mqc_scales_bytes(mx, *dims), dtype=torch.uint8, device=dev)
    alt = (torch.empty(mqc_codes_bytes(MX(fmt, block, ORDER_AB), *dims), dtype=torch.uint8, device=dev)
           if both_orders else None)
    y = torch.empty(dims, dtype=torch.float32, device=dev) if keep_fp32 else None
    nws = mqc_conv2d_fwd_workspace_bytes(cv, xq.mx, wq.mx)
    if workspace is None and nws > 0:
        workspace = torch.empty(nws, dtype=torch.uint8, device=dev)
    check(mqc_conv2d_fwd_quant(_ptr(xq.codes), _ptr(xq.scales), xq.mx, _ptr(wq.codes), _ptr(wq.scales), wq.mx, cv,
                               act, mx, _ptr(codes), _ptr(scales), _ptr(alt), _ptr(y), _ptr(workspace), nws,
                               _stream()))
    return Quantized(codes, scales, dims, mx, alt), y


def conv2d_bwd_data(wq: Quantized, gq: Quantized, cv: Conv, out=None, workspace=None):
    torch = _torch()
    gx = out if out is not None else torch.empty((cv.N, cv.C, cv.H, cv.W), dtype=torch.float32,
                                                 device=gq.codes.device)
    nws = mqc_conv2d_bwd_data_workspace_bytes(cv, wq.mx, gq.mx)
    if workspace is None and nws > 0:
        workspace = torch.empty(nws, dtype=torch.uint8, device=gq.codes.device)
    check(mqc_conv2d_bwd_data(_ptr(wq.codes), _ptr(wq.scales), wq.mx, _ptr(gq.codes), _ptr(gq.scales), gq.mx, cv,
                              _ptr(gx), _ptr(workspace), nws, _stream()))
    return gx


def conv2d_bwd_weight_workspace_bytes(cv: Conv, gf: MX, xf: MX) -> int:
    return mqc_conv2d_bwd_weight_workspace_bytes(cv, gf, xf)


def conv2d_bwd_weight(gq: Quantized, xq: Quantized, cv: Conv, out=None, workspace=None):
    torch = _torch()
    gw = out if out is not None else torch.empty((cv.K, cv.C, cv.R, cv.S), dtype=torch.float32,
                                                 device=gq.codes.device)
    nws = mqc_conv2d_bwd_weight_workspace_bytes(cv, gq.mx, xq.mx)
    if workspace is None and nws > 0:
        workspace = torch.empty(nws, dtype=torch.uint8, device=gq.codes.device)
    check(mqc_conv2d_bwd_weight(_ptr(gq.codes), _ptr(gq.scales), gq.mx, _ptr(xq.codes), _ptr(xq.scales), xq.mx,
                                cv, _ptr(gw), _ptr(workspace), nws, _stream()))
    return gw


def get_device_status() -> int:
    return mqc_get_device_status(_stream())


def debug_expire_wait(limit_ns: int) -> None:
    check(mqc_debug_expire_wait(limit_ns, _stream()))
