"""Python access to the plain-C oracle of the MicroQonv hot path.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  This package never
imports the CUDA library, and the CUDA library never imports it.

Every function takes and returns numpy arrays.  The arithmetic is all in
``mqc_oracle.c`` (double precision, plain loops); this module only marshals
arguments.  Formats, block modes and code orders use the same small integers
as the C file: fmt E4M3=0, E5M2=1, E2M1=2; block A32=0, B32=1, SQ32=2;
order BA=0 (A-axis innermost), AB=1 (B-axis innermost).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

E4M3, E5M2, E2M1 = 0, 1, 2
A32, B32, SQ32 = 0, 1, 2
ORDER_BA, ORDER_AB = 0, 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mqc_oracle.c")
_LIB = os.path.join(_HERE, "libmqc_oracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        vp = ctypes.c_void_p
        L.oracle_decode.argtypes = [i32, i32, ctypes.POINTER(i32)]
        L.oracle_decode.restype = dbl
        L.oracle_encode.argtypes = [i32, dbl]
        L.oracle_encode.restype = i32
        L.oracle_scale_code.argtypes = [i32, dbl]
        L.oracle_scale_code.restype = i32
        L.oracle_emax_elem.argtypes = [i32]
        L.oracle_emax_elem.restype = i32
        L.oracle_max_finite.argtypes = [i32]
        L.oracle_max_finite.restype = dbl
        L.oracle_padded_extents.argtypes = [i32, i32, i64, i64, ctypes.POINTER(i64), ctypes.POINTER(i64)]
        L.oracle_codes_bytes.argtypes = [i32, i32, i64, i64, i64, i64]
        L.oracle_codes_bytes.restype = i64
        L.oracle_scales_bytes.argtypes = [i32, i32, i32, i64, i64, i64, i64]
        L.oracle_scales_bytes.restype = i64
        L.oracle_quantize.argtypes = [vp, i64, i64, i64, i64, vp, i32, i32, i32, vp, vp]
        L.oracle_dequantize.argtypes = [vp, vp, i64, i64, i64, i64, i32, i32, i32, vp]
        L.oracle_im2col_fp32.argtypes = [vp] + [i64] * 10 + [vp]
        L.oracle_im2col_cbf.argtypes = [vp, vp] + [i64] * 10 + [i32, i32, i32, vp, vp]
        for name in ("oracle_conv_fwd", "oracle_conv_dgrad", "oracle_conv_wgrad"):
            getattr(L, name).argtypes = [vp, vp] + [i64] * 11 + [vp, vp]
        for name in ("oracle_conv_fwd_at", "oracle_conv_dgrad_at", "oracle_conv_wgrad_at"):
            getattr(L, name).argtypes = [vp, vp] + [i64] * 11 + [vp, i64, vp, vp]
        L.oracle_im2col_counts.argtypes = [i64] * 10 + [vp]
        L.oracle_im2col_counts.restype = i64
        L.oracle_num_threads.restype = i32
        u64, u32 = ctypes.c_uint64, ctypes.c_uint32
        L.oracle_philox4x64.argtypes = [vp, vp, vp]
        L.oracle_sr_bits.argtypes = [u64, u64, i64, i64, i64, i64, i64]
        L.oracle_sr_bits.restype = u32
        L.oracle_encode_sr.argtypes = [i32, dbl, u32]
        L.oracle_encode_sr.restype = i32
        L.oracle_quantize_sr.argtypes = [vp, i64, i64, i64, i64, vp, i32, i32, i32, u64, u64, vp, vp]
        L.oracle_nvfp4_scales_bytes.argtypes = [i32, i32, i64, i64, i64, i64]
        L.oracle_nvfp4_scales_bytes.restype = i64
        L.oracle_quantize_nvfp4.argtypes = [vp, i64, i64, i64, i64, vp, i32, i32, vp, vp, vp]
        L.oracle_dequantize_nvfp4.argtypes = [vp, vp, ctypes.c_float, i64, i64, i64, i64, i32, i32, vp]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# element formats and scales
# --------------------------------------------------------------------------
def fmt_bits(fmt: int) -> int:
    return 4 if fmt == E2M1 else 8


def decode(fmt: int, code: int) -> tuple[float, bool]:
    fin = ctypes.c_int(0)
    v = lib().oracle_decode(fmt, int(code), ctypes.byref(fin))
    return v, bool(fin.value)


def decode_table(fmt: int) -> np.ndarray:
    """Value of every code 0 .. 2^bits-1 (NaN/Inf where the format says so)."""
    return np.array([decode(fmt, c)[0] for c in range(1 << fmt_bits(fmt))], dtype=np.float64)


def encode(fmt: int, v: float) -> int:
    return int(lib().oracle_encode(fmt, float(v)))


def scale_code(fmt: int, amax: float) -> int:
    return int(lib().oracle_scale_code(fmt, float(amax)))


def emax_elem(fmt: int) -> int:
    return int(lib().oracle_emax_elem(fmt))


def max_finite(fmt: int) -> float:
    return float(lib().oracle_max_finite(fmt))


# --------------------------------------------------------------------------
# quantized layout
# --------------------------------------------------------------------------
def padded_extents(fmt: int, order: int, A: int, B: int) -> tuple[int, int]:
    """(Ap, Bp): only the innermost axis is padded, to whole 16-byte rows."""
    ap, bp = ctypes.c_int64(), ctypes.c_int64()
    lib().oracle_padded_extents(fmt, order, A, B, ctypes.byref(ap), ctypes.byref(bp))
    return ap.value, bp.value


def codes_bytes(fmt, order, d0, d1, d2, d3) -> int:
    return int(lib().oracle_codes_bytes(fmt, order, d0, d1, d2, d3))


def scales_bytes(fmt, block, order, d0, d1, d2, d3) -> int:
    return int(lib().oracle_scales_bytes(fmt, block, order, d0, d1, d2, d3))


def quantize(x: np.ndarray, fmt: int, block: int, order: int) -> tuple[np.ndarray, np.ndarray]:
    """MX-quantize a 4-D fp32 tensor [d0=B][d1=A][d2][d3] into (codes, scales)."""
    assert x.dtype == np.float32 and x.ndim == 4
    d0, d1, d2, d3 = x.shape
    strides = np.array([s // 4 for s in x.strides], dtype=np.int64)
    codes = np.zeros(codes_bytes(fmt, order, d0, d1, d2, d3), dtype=np.uint8)
    scales = np.zeros(scales_bytes(fmt, block, order, d0, d1, d2, d3), dtype=np.uint8)
    lib().oracle_quantize(_p(x), d0, d1, d2, d3, _p(strides), fmt, block, order, _p(codes), _p(scales))
    return codes, scales


def philox4x64(ctr, key) -> np.ndarray:
    """One Philox4x64-10 block (four uint64 words) for a counter and a key."""
    c = np.ascontiguousarray(ctr, dtype=np.uint64)
    k = np.ascontiguousarray(key, dtype=np.uint64)
    out = np.zeros(4, dtype=np.uint64)
    lib().oracle_philox4x64(_p(c), _p(k), _p(out))
    return out


def sr_bits(seed, offset, B, A, pix, b, a) -> int:
    """The 16 random bits stochastic rounding uses for element (pix, b, a)."""
    return int(lib().oracle_sr_bits(seed, offset, B, A, pix, b, a))


def encode_sr(fmt: int, v: float, r: int) -> int:
    return int(lib().oracle_encode_sr(fmt, float(v), int(r)))


def quantize_sr(x: np.ndarray, fmt: int, block: int, order: int, seed: int, offset: int = 0):
    """MX quantization with stochastically rounded elements: (codes, scales)."""
    assert x.dtype == np.float32 and x.ndim == 4
    d0, d1, d2, d3 = x.shape
    strides = np.array([s // 4 for s in x.strides], dtype=np.int64)
    codes = np.zeros(codes_bytes(fmt, order, d0, d1, d2, d3), dtype=np.uint8)
    scales = np.zeros(scales_bytes(fmt, block, order, d0, d1, d2, d3), dtype=np.uint8)
    lib().oracle_quantize_sr(_p(x), d0, d1, d2, d3, _p(strides), fmt, block, order, seed, offset, _p(codes),
                             _p(scales))
    return codes, scales


NV_A16, NV_B16, NV_SQ16 = 0, 1, 2


def quantize_nvfp4(x: np.ndarray, block: int, order: int):
    """NVFP4 quantization (paper, Eq. 4-6) of a 4-D fp32 tensor: (codes,
    E4M3 block scales, per-tensor fp32 scale T)."""
    assert x.dtype == np.float32 and x.ndim == 4
    d0, d1, d2, d3 = x.shape
    strides = np.array([s // 4 for s in x.strides], dtype=np.int64)
    codes = np.zeros(codes_bytes(E2M1, order, d0, d1, d2, d3), dtype=np.uint8)
    scales = np.zeros(int(lib().oracle_nvfp4_scales_bytes(block, order, d0, d1, d2, d3)), dtype=np.uint8)
    t = np.zeros(1, dtype=np.float32)
    lib().oracle_quantize_nvfp4(_p(x), d0, d1, d2, d3, _p(strides), block, order, _p(codes), _p(scales), _p(t))
    return codes, scales, float(t[0])


def dequantize_nvfp4(codes, scales, tscale, shape, block, order) -> np.ndarray:
    d0, d1, d2, d3 = shape
    out = np.empty((d0, d1, d2, d3), dtype=np.float64)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    lib().oracle_dequantize_nvfp4(_p(codes), _p(scales), float(tscale), d0, d1, d2, d3, block, order, _p(out))
    return out


ACT_NONE, ACT_RELU, ACT_SILU = 0, 1, 2


def activation(y: np.ndarray, act: int) -> np.ndarray:
    """The activation a layer applies to its convolution output before the
    result is quantized as the next layer's input (the paper's section V and
    Fig. 4 flow): none, ReLU max(y, 0), or SiLU y / (1 + exp(-y)), in float64."""
    y = np.asarray(y, dtype=np.float64)
    if act == ACT_RELU:
        return np.maximum(y, 0.0)
    if act == ACT_SILU:
        return y / (1.0 + np.exp(-y))
    return y


def dequantize(codes, scales, shape, fmt, block, order) -> np.ndarray:
    d0, d1, d2, d3 = shape
    out = np.empty((d0, d1, d2, d3), dtype=np.float64)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    lib().oracle_dequantize(_p(codes), _p(scales), d0, d1, d2, d3, fmt, block, order, _p(out))
    return out


# --------------------------------------------------------------------------
# conv geometry
# --------------------------------------------------------------------------
def out_hw(H, W, R, S, sh, sw, ph, pw) -> tuple[int, int]:
    return (H + 2 * ph - R) // sh + 1, (W + 2 * pw - S) // sw + 1


def im2col_fp32(x: np.ndarray, R, S, sh, sw, ph, pw) -> np.ndarray:
    N, C, H, W = x.shape
    P, Q = out_hw(H, W, R, S, sh, sw, ph, pw)
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty((N, R * S * C, P, Q), dtype=np.float32)
    lib().oracle_im2col_fp32(_p(x), N, C, H, W, R, S, sh, sw, ph, pw, _p(out))
    return out


def im2col_cbf(codes, scales, N, C, H, W, R, S, sh, sw, ph, pw, fmt, block, order):
    """Channel-batch-first im2col on quantized X; returns (codes, scales) of the
    expanded tensor (spatial P x Q, B = N, A = R*S*Ap)."""
    Ap, Bp = padded_extents(fmt, order, C, N)
    P, Q = out_hw(H, W, R, S, sh, sw, ph, pw)
    nsa = Ap if block == B32 else -(-Ap // 32)
    nsb = Bp if block == A32 else -(-Bp // 32)
    co = np.zeros(codes_bytes(fmt, order, Bp, R * S * Ap, P, Q), dtype=np.uint8)
    so = np.zeros(P * Q * nsb * R * S * nsa, dtype=np.uint8)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    lib().oracle_im2col_cbf(_p(codes), _p(scales), N, C, H, W, R, S, sh, sw, ph, pw,
                            fmt, block, order, _p(co), _p(so))
    return co, so


def _conv_args(N, C, H, W, K, R, S, sh, sw, ph, pw):
    return [N, C, H, W, K, R, S, sh, sw, ph, pw]


def conv_fwd(x: np.ndarray, w: np.ndarray, sh=1, sw=1, ph=0, pw=0):
    """Eq. 1 in double: returns (Y, sum|a*b|) as [N][K][P][Q]."""
    N, C, H, W = x.shape
    K, C2, R, S = w.shape
    assert C == C2
    P, Q = out_hw(H, W, R, S, sh, sw, ph, pw)
    x = np.ascontiguousarray(x, dtype=np.float64)
    w = np.ascontiguousarray(w, dtype=np.float64)
    y = np.empty((N, K, P, Q))
    ya = np.empty((N, K, P, Q))
    lib().oracle_conv_fwd(_p(x), _p(w), *_conv_args(N, C, H, W, K, R, S, sh, sw, ph, pw), _p(y), _p(ya))
    return y, ya


def conv_dgrad(w: np.ndarray, gy: np.ndarray, H: int, W: int, sh=1, sw=1, ph=0, pw=0):
    """Eq. 2 in double: returns (G_X, sum|a*b|) as [N][C][H][W]."""
    K, C, R, S = w.shape
    N, K2, P, Q = gy.shape
    assert K == K2 and (P, Q) == out_hw(H, W, R, S, sh, sw, ph, pw)
    w = np.ascontiguousarray(w, dtype=np.float64)
    gy = np.ascontiguousarray(gy, dtype=np.float64)
    gx = np.empty((N, C, H, W))
    gxa = np.empty((N, C, H, W))
    lib().oracle_conv_dgrad(_p(w), _p(gy), *_conv_args(N, C, H, W, K, R, S, sh, sw, ph, pw), _p(gx), _p(gxa))
    return gx, gxa


def conv_wgrad(gy: np.ndarray, x: np.ndarray, R: int, S: int, sh=1, sw=1, ph=0, pw=0):
    """Eq. 3 in double: returns (G_W, sum|a*b|) as [K][C][R][S]."""
    N, C, H, W = x.shape
    N2, K, P, Q = gy.shape
    assert N == N2 and (P, Q) == out_hw(H, W, R, S, sh, sw, ph, pw)
    x = np.ascontiguousarray(x, dtype=np.float64)
    gy = np.ascontiguousarray(gy, dtype=np.float64)
    gw = np.empty((K, C, R, S))
    gwa = np.empty((K, C, R, S))
    lib().oracle_conv_wgrad(_p(gy), _p(x), *_conv_args(N, C, H, W, K, R, S, sh, sw, ph, pw), _p(gw), _p(gwa))
    return gw, gwa


def _at(name, a, b, dims, idx):
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    val = np.empty(idx.size)
    vab = np.empty(idx.size)
    a = np.ascontiguousarray(a, dtype=np.float64)
    b = np.ascontiguousarray(b, dtype=np.float64)
    getattr(lib(), name)(_p(a), _p(b), *dims, _p(idx), idx.size, _p(val), _p(vab))
    return val, vab


def conv_fwd_at(x, w, idx, sh=1, sw=1, ph=0, pw=0):
    N, C, H, W = x.shape
    K, _, R, S = w.shape
    return _at("oracle_conv_fwd_at", x, w, _conv_args(N, C, H, W, K, R, S, sh, sw, ph, pw), idx)


def conv_dgrad_at(w, gy, H, W, idx, sh=1, sw=1, ph=0, pw=0):
    K, C, R, S = w.shape
    N = gy.shape[0]
    return _at("oracle_conv_dgrad_at", w, gy, _conv_args(N, C, H, W, K, R, S, sh, sw, ph, pw), idx)


def conv_wgrad_at(gy, x, R, S, idx, sh=1, sw=1, ph=0, pw=0):
    N, C, H, W = x.shape
    K = gy.shape[1]
    return _at("oracle_conv_wgrad_at", gy, x, _conv_args(N, C, H, W, K, R, S, sh, sw, ph, pw), idx)


def im2col_counts(N, C, H, W, R, S, sh=1, sw=1, ph=0, pw=0):
    """(per-element occurrence counts in X', total entries of X')."""
    counts = np.empty((N, C, H, W), dtype=np.int32)
    entries = lib().oracle_im2col_counts(N, C, H, W, R, S, sh, sw, ph, pw, _p(counts))
    return counts, int(entries)


def num_threads() -> int:
    return int(lib().oracle_num_threads())
