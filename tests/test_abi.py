"""The C-ABI library loads, exports every entry point include/mqc.h declares,
and its host-only logic (buffer sizes, argument checks) is right.  No kernel
is launched: these run without a GPU."""
import ctypes
import os
import re

import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def mqc():
    import __graft_entry__
    __graft_entry__.build()
    import im2col_gemm_b200
    return im2col_gemm_b200


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "mqc.h")).read()
    return sorted(set(re.findall(r"MQC_API [^;(]*?\b(mqc_\w+)\(", text)))


def test_exports_every_declared_symbol(mqc):
    names = declared_symbols()
    assert len(names) >= 16
    assert set(names) == set(mqc.EXPORTS)
    lib = ctypes.CDLL(mqc.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert mqc.lib.mqc_version() == 100
    assert mqc.lib.mqc_status_string(-4).decode() == "device wait timed out"


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("block", [0, 1, 2])
@pytest.mark.parametrize("order", [0, 1])
def test_sizes_match_oracle(mqc, orc, fmt, block, order):
    for dims in [(2, 32, 8, 8), (16, 16, 640, 640), (37, 45, 3, 2), (1, 1, 1, 1), (256, 128, 80, 80)]:
        mx = mqc.MX(fmt, block, order)
        assert mqc.mqc_codes_bytes(mx, *dims) == orc.codes_bytes(fmt, order, *dims)
        assert mqc.mqc_scales_bytes(mx, *dims) == orc.scales_bytes(fmt, block, order, *dims)


@pytest.mark.parametrize("fmt,block,order", [(0, 0, 0), (0, 1, 1), (2, 2, 0), (1, 2, 1)])
def test_im2col_sizes_match_oracle(mqc, orc, fmt, block, order):
    import numpy as np
    for (N, C, H, W, R, S, st, pad) in [(2, 32, 8, 8, 3, 3, 1, 1), (3, 48, 9, 7, 3, 3, 2, 1), (5, 16, 4, 4, 1, 1, 1, 0)]:
        cv = mqc.conv_desc(N, C, H, W, 8, R, S, st, pad)
        x = np.zeros((N, C, H, W), dtype=np.float32)
        codes, scales = orc.quantize(x, fmt, block, order)
        co, so = orc.im2col_cbf(codes, scales, N, C, H, W, R, S, st, st, pad, pad, fmt, block, order)
        assert mqc.lib.mqc_im2col_cbf_codes_bytes(ctypes.byref(cv), ctypes.byref(mqc.MX(fmt, block, order))) == co.size
        assert mqc.lib.mqc_im2col_cbf_scales_bytes(ctypes.byref(cv), ctypes.byref(mqc.MX(fmt, block, order))) == so.size


def test_tensor_dims(mqc):
    cv = mqc.conv_desc(16, 32, 320, 320, 64, 3, 3, 2, 1)
    assert mqc.tensor_dims(mqc.ROLE_X, cv) == (16, 32, 320, 320)
    assert mqc.tensor_dims(mqc.ROLE_W, cv) == (64, 32, 3, 3)
    assert mqc.tensor_dims(mqc.ROLE_G, cv) == (16, 64, 160, 160)
    for L in synth.WORKLOADS[2].layers:
        cv = mqc.conv_desc(L.N, L.C, L.H, L.W, L.K, L.R, L.S, L.stride, L.pad)
        assert mqc.tensor_dims(mqc.ROLE_G, cv)[2:] == (L.P, L.Q)


def test_invalid_arguments_rejected_before_launch(mqc):
    mx = mqc.MX(0, 0, 0)
    d = mqc.T4(2, 32, 8, 8, 2048, 64, 8, 1)
    # null source / codes
    assert mqc.mqc_quantize_mx(None, d, mx, ctypes.c_void_p(16), ctypes.c_void_p(16), None, None) == -1
    # bad enum
    assert mqc.mqc_quantize_mx(ctypes.c_void_p(16), d, mqc.MX(7, 0, 0), ctypes.c_void_p(16), ctypes.c_void_p(16),
                               None, None) == -1
    # misaligned codes
    assert mqc.mqc_quantize_mx(ctypes.c_void_p(16), d, mx, ctypes.c_void_p(17), ctypes.c_void_p(16), None,
                               None) == -5
    assert "aligned" in mqc.lib.mqc_last_error_message().decode()
    # zero extent
    bad = mqc.T4(0, 32, 8, 8, 1, 1, 1, 1)
    assert mqc.mqc_quantize_mx(ctypes.c_void_p(16), bad, mx, ctypes.c_void_p(16), ctypes.c_void_p(16), None,
                               None) == -1
    # GEMM operand in the wrong block mode / order / format
    cv = mqc.conv_desc(2, 32, 8, 8, 32, 3, 3, 1, 1)
    p = ctypes.c_void_p(256)
    assert mqc.mqc_conv2d_fwd(p, p, mqc.MX(0, 1, 0), p, p, mqc.MX(0, 0, 0), cv, p, None, 0, None) == -2
    assert mqc.mqc_conv2d_fwd(p, p, mqc.MX(0, 0, 1), p, p, mqc.MX(0, 0, 0), cv, p, None, 0, None) == -2
    assert mqc.mqc_conv2d_bwd_data(p, p, mqc.MX(0, 0, 1), p, p, mqc.MX(1, 0, 0), cv, p, None, 0, None) == -2
    assert mqc.mqc_conv2d_bwd_weight(p, p, mqc.MX(1, 0, 1), p, p, mqc.MX(0, 1, 1), cv, p, None, 0, None) == -2
    # a convolution whose kernel is larger than the padded input
    assert mqc.mqc_conv2d_fwd(p, p, mx, p, p, mx, mqc.conv_desc(1, 32, 2, 2, 8, 5, 5, 1, 1), p, None, 0, None) == -1
    assert mqc.lib.mqc_debug_expire_wait(10, None) == -1
    # batched quantization: 1 .. 16 tensors, all codes_alt or none
    one = [ctypes.c_void_p(16)]
    assert mqc.mqc_quantize_mx_batch([], [], mx, [], [], None, None) == -1
    assert mqc.mqc_quantize_mx_batch(one * 17, [d] * 17, mx, one * 17, one * 17, None, None) == -1
    assert mqc.mqc_quantize_mx_batch(one * 2, [d, d], mx, one * 2, one * 2, [16, 0], None) == -1
    assert mqc.mqc_quantize_mx_batch(one * 2, [d, bad], mx, one * 2, one * 2, None, None) == -1
    assert mqc.mqc_quantize_mx_batch(one * 2, [d, d], mx, [16, 17], one * 2, None, None) == -5
    # stochastic rounding: primary order BA and an NCHW-like source only
    assert mqc.mqc_quantize_mx_sr(ctypes.c_void_p(16), d, mqc.MX(0, 2, 1), ctypes.c_void_p(16), ctypes.c_void_p(16),
                                  None, 1, 0, None) == -2
    dt = mqc.T4(2, 32, 8, 8, 2048, 64, 1, 8)     # H and W swapped in memory
    assert mqc.mqc_quantize_mx_sr(ctypes.c_void_p(16), dt, mx, ctypes.c_void_p(16), ctypes.c_void_p(16),
                                  None, 1, 0, None) == -2
    assert "quantize_mx_sr" in mqc.lib.mqc_last_error_message().decode()
    # forward and weight gradient: at most four stride phases (stride_h * stride_w <= 4)
    s3 = mqc.conv_desc(2, 32, 12, 12, 32, 3, 3, 3, 1)
    assert mqc.mqc_conv2d_fwd(p, p, mx, p, p, mx, s3, p, None, 0, None) == -2
    assert "stride product" in mqc.lib.mqc_last_error_message().decode()
    sq_ab = mqc.MX(0, 2, 1)
    assert mqc.mqc_conv2d_bwd_weight(p, p, sq_ab, p, p, sq_ab, s3, p, None, 0, None) == -2
    assert mqc.mqc_conv2d_bwd_weight_noalloc(p, p, sq_ab, p, p, sq_ab, s3, p, None) == -2


def test_gemm_workspace_sizes_cover_widened_fp4_operands(mqc):
    """E2M1 GEMM operands are widened to one byte per element in the caller's
    workspace: the size queries give twice the packed code bytes (rounded up
    to 256), and nothing for FP8 operands unless the input gradient runs as a
    sub-pixel GEMM (its window weights)."""
    cv = mqc.conv_desc(4, 40, 9, 11, 24, 3, 3, 2, 1)
    P, Q = (9 + 2 - 3) // 2 + 1, (11 + 2 - 3) // 2 + 1
    fp8_a, fp4_a = mqc.MX(0, 2, 0), mqc.MX(2, 2, 0)
    fp8_b, fp4_b = mqc.MX(0, 2, 1), mqc.MX(2, 2, 1)
    r = lambda n: (2 * n + 255) // 256 * 256
    assert mqc.mqc_conv2d_fwd_workspace_bytes(cv, fp8_a, fp8_a) == 0
    assert mqc.mqc_conv2d_fwd_workspace_bytes(cv, fp4_a, fp8_a) == r(mqc.mqc_codes_bytes(fp4_a, 4, 40, 9, 11))
    assert mqc.mqc_conv2d_fwd_workspace_bytes(cv, fp4_a, fp4_a) == (r(mqc.mqc_codes_bytes(fp4_a, 4, 40, 9, 11))
                                                                     + r(mqc.mqc_codes_bytes(fp4_a, 24, 40, 3, 3)))
    assert mqc.mqc_conv2d_bwd_data_workspace_bytes(cv, fp8_b, fp8_a) == 0
    # sub-pixel input gradient (C = 32, even H and W, stride 2): the window
    # weights, 2 x 2 offsets x (4 phases x 32 channels) rows of 48 code bytes,
    # and their scales, 2 K-blocks per row
    sub = mqc.conv_desc(2, 32, 8, 8, 48, 3, 3, 2, 1)
    assert mqc.mqc_conv2d_bwd_data_workspace_bytes(sub, fp8_b, fp8_a) == 4 * 128 * 48 + (4 * 2 * 128 + 255) // 256 * 256
    assert mqc.mqc_conv2d_bwd_data_workspace_bytes(cv, fp4_b, fp4_a) == (r(mqc.mqc_codes_bytes(fp4_b, 24, 40, 3, 3))
                                                                          + r(mqc.mqc_codes_bytes(fp4_a, 4, 24, P, Q)))


@pytest.mark.parametrize("block", [0, 1, 2])
@pytest.mark.parametrize("order", [0, 1])
def test_nvfp4_scale_sizes_match_oracle(mqc, orc, block, order):
    for dims in [(2, 32, 8, 8), (37, 45, 3, 2), (1, 1, 1, 1), (128, 128, 80, 80)]:
        assert mqc.lib.mqc_nvfp4_scales_bytes(block, order, *dims) == \
            int(orc.lib().oracle_nvfp4_scales_bytes(block, order, *dims))
    assert mqc.lib.mqc_nvfp4_scales_bytes(3, order, 2, 32, 8, 8) == -1
