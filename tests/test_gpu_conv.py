"""Parity of the block-scaled tensor-core convolutions with the oracle.

The CUDA path quantizes the fp32 inputs with its own quantizer and runs its
GEMM; the oracle quantizes the same inputs, dequantizes them and evaluates
Eq. 1-3 directly in double, with sum |a*b| alongside.  Every output element
must satisfy |err| <= 1e-3 * sum|a*b| + 1e-6.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu
RTOL, ATOL = 1e-3, 1e-6


@pytest.fixture(scope="module")
def mqc():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import im2col_gemm_b200
    return im2col_gemm_b200


def _dev(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _host(t):
    import torch
    torch.cuda.synchronize()
    return t.cpu().numpy().astype(np.float64)


def _check(name, got, ref, refabs):
    err = np.abs(got - ref)
    bound = RTOL * refabs + ATOL
    bad = ~(err <= bound)
    if bad.any():
        idx = np.argwhere(bad)
        first = [tuple(int(v) for v in i) for i in idx[:6]]
        vals = [(float(got[tuple(i)]), float(ref[tuple(i)])) for i in idx[:6]]
        raise AssertionError(f"{name}: {bad.sum()} of {bad.size} outside tolerance; max err/bound "
                             f"{float((err / bound).max()):.3g}; first {first} got/want {vals}")


# (N, C, H, W, K, R, S, stride, pad)
FWD_CASES = [
    (2, 32, 8, 8, 32, 3, 3, 1, 1),        # the single-conv workload
    (64, 64, 4, 4, 64, 1, 1, 1, 0),       # plain GEMM: 1x1 conv
    (4, 48, 9, 11, 40, 3, 3, 2, 1),       # ragged, stride 2
    (16, 16, 20, 20, 32, 3, 3, 2, 1),     # C = 16 (half a block), stride 2
    (3, 128, 10, 9, 160, 3, 3, 1, 1),     # two column tiles, 4-block boxes
    (8, 96, 7, 6, 256, 1, 1, 1, 0),       # C with 3 blocks
    (5, 32, 12, 12, 24, 2, 3, 1, 0),      # non-square kernel, K < 32
    # batch 16 with 16-byte code rows (C <= 16): whole-batch pixel runs,
    # batch-first rows; Q a multiple of 4 takes the staged epilogue
    (16, 16, 24, 24, 32, 3, 3, 2, 1),     # Q = 12: the last 8-wide tile half empty
    (16, 3, 17, 33, 40, 3, 3, 1, 1),      # C = 3, odd Q (plain stores), K = 40 (48-column tile)
    (16, 8, 16, 16, 96, 1, 1, 1, 0),      # 1x1, three 32-column chunks
    (16, 16, 10, 17, 20, 2, 3, 2, 0),     # non-square kernel, Q = 8, K = 20
    (6, 40, 12, 20, 30, 3, 3, 1, 1),      # Q = 20, K = 30 (ragged columns)
    # 16-byte runs of 4 q per lane quad: the 32-bit scale gather (C = 128),
    # and units of several 128-row tiles (many tiles, one K-block)
    (4, 128, 8, 12, 30, 1, 1, 1, 0),
    (16, 32, 80, 80, 30, 1, 1, 1, 0),
]


@pytest.mark.parametrize("case", FWD_CASES)
@pytest.mark.parametrize("blocks", [(0, 0), (2, 2)])
def test_conv_fwd_parity(mqc, orc, case, blocks):
    N, C, H, W, K, R, S, st, pad = case
    bx, bw = blocks
    x = synth.random_tensor((N, C, H, W), seed=700 + N + C, dist="student_t")
    w = synth.random_tensor((K, C, R, S), seed=701 + K, scale=0.05)
    fx, fw = 0, (1 if (K // 8) % 2 else 0)
    cv = mqc.conv_desc(N, C, H, W, K, R, S, st, pad)
    y = mqc.conv2d_fwd(mqc.quantize_mx(_dev(x), fx, bx, 0), mqc.quantize_mx(_dev(w), fw, bw, 0), cv)
    xd = orc.dequantize(*orc.quantize(x, fx, bx, 0), x.shape, fx, bx, 0)
    wd = orc.dequantize(*orc.quantize(w, fw, bw, 0), w.shape, fw, bw, 0)
    ref, refabs = orc.conv_fwd(xd, wd, st, st, pad, pad)
    _check(f"fwd {case} blocks {blocks}", _host(y), ref, refabs)


BWD_CASES = [
    (2, 32, 8, 8, 32, 3, 3, 1, 1),
    (32, 64, 6, 5, 64, 1, 1, 1, 0),
    (4, 40, 9, 11, 48, 3, 3, 2, 1),
    (16, 16, 12, 12, 32, 3, 3, 2, 1),
    (40, 96, 5, 6, 130, 3, 3, 1, 1),
    (64, 32, 6, 6, 32, 3, 3, 1, 0),
    (6, 160, 5, 5, 48, 3, 3, 1, 1),       # C > 128: one tap per weight-gradient unit, two column tiles
]


# input-gradient cases beyond the shared ones: output stride phases without
# taps (1x1 stride 2), nine phases over three launches (stride 3), a 5x5
# kernel with uneven tap counts per phase, unequal phase extents (odd H, W)
DGRAD_CASES = BWD_CASES + [
    (4, 32, 10, 9, 32, 1, 1, 2, 0),
    (2, 32, 11, 10, 48, 3, 3, 3, 1),
    (3, 16, 13, 12, 32, 5, 5, 2, 2),
    (2, 64, 7, 9, 160, 3, 3, 2, 1),
    (6, 30, 12, 20, 40, 3, 3, 1, 1),      # stride 1, W = 20: 16-byte runs of 4 w, C = 30 (ragged columns)
]
# the sub-pixel GEMM (stride 2, even H and W, C in 16s): phases no tap reaches
# (1x1), a 3x3 window of offsets (5x5), column tiles that split the phases
# (C = 48, 192 columns) with ragged K, a 4x4 kernel
DGRAD_CASES += [
    (4, 32, 10, 8, 32, 1, 1, 2, 0),
    (3, 16, 12, 10, 32, 5, 5, 2, 2),
    (2, 48, 6, 8, 40, 3, 3, 2, 1),
    (2, 16, 8, 8, 32, 4, 4, 2, 1),
    (4, 32, 14, 24, 48, 3, 3, 2, 1),      # W = 24: 16-byte runs of 4 column pairs per lane quad
]


@pytest.mark.parametrize("case", DGRAD_CASES)
@pytest.mark.parametrize("sq", [False, True])
def test_conv_bwd_data_parity(mqc, orc, case, sq):
    N, C, H, W, K, R, S, st, pad = case
    P, Q = orc.out_hw(H, W, R, S, st, st, pad, pad)
    w = synth.random_tensor((K, C, R, S), seed=801 + K, scale=0.05)
    g = synth.random_tensor((N, K, P, Q), seed=802 + N, scale=1e-3)
    bw, bg = (2, 2) if sq else (1, 0)
    cv = mqc.conv_desc(N, C, H, W, K, R, S, st, pad)
    gx = mqc.conv2d_bwd_data(mqc.quantize_mx(_dev(w), 0, bw, 1), mqc.quantize_mx(_dev(g), 1, bg, 0), cv)
    wd = orc.dequantize(*orc.quantize(w, 0, bw, 1), w.shape, 0, bw, 1)
    gd = orc.dequantize(*orc.quantize(g, 1, bg, 0), g.shape, 1, bg, 0)
    ref, refabs = orc.conv_dgrad(wd, gd, H, W, st, st, pad, pad)
    _check(f"dgrad {case} sq={sq}", _host(gx), ref, refabs)


# weight-gradient cases beyond the shared ones: tap groups of whole kernel
# rows loaded as one window box per pixel with channels beyond C (C = 3), with
# 128-byte rows (N = 128), and with a partial last group (5x5, two rows each)
WGRAD_CASES = BWD_CASES + [
    (2, 3, 16, 16, 16, 3, 3, 2, 1),
    (128, 16, 6, 6, 32, 3, 3, 2, 1),
    (4, 24, 11, 10, 40, 5, 5, 2, 2),
]


@pytest.mark.parametrize("case", WGRAD_CASES)
@pytest.mark.parametrize("sq", [False, True])
def test_conv_bwd_weight_parity(mqc, orc, case, sq):
    N, C, H, W, K, R, S, st, pad = case
    P, Q = orc.out_hw(H, W, R, S, st, st, pad, pad)
    x = synth.random_tensor((N, C, H, W), seed=901 + C, dist="student_t")
    g = synth.random_tensor((N, K, P, Q), seed=902 + K, scale=1e-3)
    b = 2 if sq else 1
    cv = mqc.conv_desc(N, C, H, W, K, R, S, st, pad)
    gw = mqc.conv2d_bwd_weight(mqc.quantize_mx(_dev(g), 1, b, 1), mqc.quantize_mx(_dev(x), 0, b, 1), cv)
    gd = orc.dequantize(*orc.quantize(g, 1, b, 1), g.shape, 1, b, 1)
    xd = orc.dequantize(*orc.quantize(x, 0, b, 1), x.shape, 0, b, 1)
    ref, refabs = orc.conv_wgrad(gd, xd, R, S, st, st, pad, pad)
    _check(f"wgrad {case} sq={sq}", _host(gw), ref, refabs)


# FP4 (E2M1) operands, alone or mixed with FP8: (case, format of the first
# operand, format of the second) for each GEMM
FP4_CASES = [((4, 48, 9, 11, 40, 3, 3, 2, 1), 2, 0), ((16, 16, 12, 12, 32, 3, 3, 2, 1), 2, 2),
             ((3, 128, 10, 9, 160, 3, 3, 1, 1), 0, 2), ((40, 96, 5, 6, 130, 1, 1, 1, 0), 2, 1),
             # both operands MXFP4: native kind::mxf4 forward and per-phase input
             # gradient (odd H: the stride phases do not tile; C, K ragged)
             ((6, 40, 9, 7, 24, 3, 3, 2, 1), 2, 2), ((5, 70, 8, 8, 100, 3, 3, 1, 1), 2, 2)]


@pytest.mark.parametrize("case,fa,fb", FP4_CASES)
def test_conv_fp4_operands(mqc, orc, case, fa, fb):
    """E2M1 operands run through the same tensor-core path (widened to the
    E4M3 codes of the same values): forward (X, W), input gradient (W, G_Y)
    and weight gradient (G_Y, X) against the oracle on its own E2M1
    dequantization."""
    N, C, H, W, K, R, S, st, pad = case
    P, Q = orc.out_hw(H, W, R, S, st, st, pad, pad)
    x = synth.random_tensor((N, C, H, W), seed=950 + C, dist="student_t")
    w = synth.random_tensor((K, C, R, S), seed=951 + K, scale=0.05)
    g = synth.random_tensor((N, K, P, Q), seed=952 + N, scale=1e-3)
    cv = mqc.conv_desc(N, C, H, W, K, R, S, st, pad)
    deq = lambda t, f, o: orc.dequantize(*orc.quantize(t, f, 2, o), t.shape, f, 2, o)
    y = mqc.conv2d_fwd(mqc.quantize_mx(_dev(x), fa, 2, 0), mqc.quantize_mx(_dev(w), fb, 2, 0), cv)
    ref, refabs = orc.conv_fwd(deq(x, fa, 0), deq(w, fb, 0), st, st, pad, pad)
    _check(f"fwd fp4 {case} {fa}/{fb}", _host(y), ref, refabs)
    gx = mqc.conv2d_bwd_data(mqc.quantize_mx(_dev(w), fa, 2, 1), mqc.quantize_mx(_dev(g), fb, 2, 0), cv)
    ref, refabs = orc.conv_dgrad(deq(w, fa, 1), deq(g, fb, 0), H, W, st, st, pad, pad)
    _check(f"dgrad fp4 {case} {fa}/{fb}", _host(gx), ref, refabs)
    gw = mqc.conv2d_bwd_weight(mqc.quantize_mx(_dev(g), fa, 2, 1), mqc.quantize_mx(_dev(x), fb, 2, 1), cv)
    ref, refabs = orc.conv_wgrad(deq(g, fa, 1), deq(x, fb, 1), R, S, st, st, pad, pad)
    _check(f"wgrad fp4 {case} {fa}/{fb}", _host(gw), ref, refabs)


def test_training_step_shares_one_quantization(mqc, orc):
    """SQ32: each tensor is quantized once, in both code orders, and the
    three GEMMs read those copies (paper, section IV-B: quantized once)."""
    N, C, H, W, K, R, S, st, pad = 32, 64, 10, 10, 96, 3, 3, 1, 1
    P, Q = orc.out_hw(H, W, R, S, st, st, pad, pad)
    x = synth.random_tensor((N, C, H, W), seed=11, dist="student_t")
    w = synth.random_tensor((K, C, R, S), seed=12, scale=0.02)
    g = synth.random_tensor((N, K, P, Q), seed=13, scale=1e-3)
    cv = mqc.conv_desc(N, C, H, W, K, R, S, st, pad)
    xq = mqc.quantize_mx(_dev(x), 0, 2, 0, both_orders=True)
    wq = mqc.quantize_mx(_dev(w), 0, 2, 0, both_orders=True)
    gq = mqc.quantize_mx(_dev(g), 1, 2, 0, both_orders=True)
    y = mqc.conv2d_fwd(xq, wq, cv)
    gx = mqc.conv2d_bwd_data(wq.other_order(), gq, cv)
    gw = mqc.conv2d_bwd_weight(gq.other_order(), xq.other_order(), cv)
    xd = orc.dequantize(*orc.quantize(x, 0, 2, 0), x.shape, 0, 2, 0)
    wd = orc.dequantize(*orc.quantize(w, 0, 2, 0), w.shape, 0, 2, 0)
    gd = orc.dequantize(*orc.quantize(g, 1, 2, 0), g.shape, 1, 2, 0)
    _check("step fwd", _host(y), *orc.conv_fwd(xd, wd, st, st, pad, pad))
    _check("step dgrad", _host(gx), *orc.conv_dgrad(wd, gd, H, W, st, st, pad, pad))
    _check("step wgrad", _host(gw), *orc.conv_wgrad(gd, xd, R, S, st, st, pad, pad))


def test_device_wait_timeout_is_reported(mqc):
    """A bounded kernel-side wait that runs out sets the device error flag; the
    host reads and clears it and the context stays usable."""
    import torch
    assert mqc.get_device_status() == 0
    mqc.debug_expire_wait(2_000_000)          # 2 ms
    assert mqc.get_device_status() == -4
    assert mqc.get_device_status() == 0
    t = torch.ones(4, device="cuda")
    assert float(t.sum()) == 4.0


def test_tensor_map_cache_same_address_other_shape(mqc, orc):
    """Forwards whose activation codes start at the same device address with
    other extents (and the first shape again): the library reuses encoded
    tensor maps keyed by every encoder input, so each call must still see its
    own geometry."""
    import torch
    buf = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    for case in [(2, 32, 8, 8, 32, 3, 3, 1, 1), (4, 32, 6, 10, 32, 3, 3, 1, 1), (2, 32, 8, 8, 32, 3, 3, 1, 1)]:
        N, C, H, W, K, R, S, st, pad = case
        x = synth.random_tensor((N, C, H, W), seed=1200 + N * H, dist="student_t")
        w = synth.random_tensor((K, C, R, S), seed=1201 + W, scale=0.05)
        xq = mqc.quantize_mx(_dev(x), 0, 2, 0)
        n = xq.codes.numel()
        buf[:n].copy_(xq.codes)
        xs = mqc.Quantized(buf[:n], xq.scales, xq.dims, xq.mx)
        cv = mqc.conv_desc(N, C, H, W, K, R, S, st, pad)
        y = mqc.conv2d_fwd(xs, mqc.quantize_mx(_dev(w), 0, 2, 0), cv)
        xd = orc.dequantize(*orc.quantize(x, 0, 2, 0), x.shape, 0, 2, 0)
        wd = orc.dequantize(*orc.quantize(w, 0, 2, 0), w.shape, 0, 2, 0)
        ref, refabs = orc.conv_fwd(xd, wd, st, st, pad, pad)
        _check(f"fwd {case} at a shared address", _host(y), ref, refabs)
