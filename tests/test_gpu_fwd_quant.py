"""Parity of the forward convolution with a quantized output
(mqc_conv2d_fwd_quant: the activation and the next layer's MX quantization in
the GEMM epilogue, the flow of the MicroQonv paper's section V / Fig. 4).

The oracle composes the pieces: its direct convolution of the dequantized
operands (Eq. 1), the activation in float64, and its quantizer.  The kernel
also returns the fp32 activated output it quantized, so that:
- that fp32 output is within the convolution tolerance (1e-3 * sum|a*b| +
  1e-6) of the oracle's activated convolution, widened by the activation's
  Lipschitz constant (1 for ReLU, 1.1 for SiLU) plus the fp32 evaluation of
  the activation (a relative 1e-6);
- the codes (order BA, and AB when asked for) and the E8M0 scales are bit
  for bit those of the oracle's quantizer applied to that same fp32 tensor
  (the floating-point values that decide the codes are the kernel's own).
A call without the fp32 copy writes the same codes.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu
LIP = {0: 1.0, 1: 1.0, 2: 1.1}


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
    return t.cpu().numpy()


def _run(mqc, orc, L, x, w, xfmt, wfmt, block, yfmt, yblock, act, full_conv=True, seed=0):
    cv = mqc.conv_desc(L.N, L.C, L.H, L.W, L.K, L.R, L.S, L.stride, L.pad)
    xq = mqc.quantize_mx(_dev(x), xfmt, block, mqc.ORDER_BA)
    wq = mqc.quantize_mx(_dev(w), wfmt, block, mqc.ORDER_BA)
    yq, y = mqc.conv2d_fwd_quant(xq, wq, cv, yfmt, yblock, act, both_orders=True, keep_fp32=True)
    yq2, _ = mqc.conv2d_fwd_quant(xq, wq, cv, yfmt, yblock, act, both_orders=False, keep_fp32=False)
    mqc.check(mqc.get_device_status())
    yh = _host(y)
    # codes and scales: the oracle's quantizer on the kernel's own fp32 output
    rc, rs = orc.quantize(yh, yfmt, yblock, 0)
    rc2, _ = orc.quantize(yh, yfmt, yblock, 1)
    assert np.array_equal(_host(yq.scales), rs), "scales differ"
    got = _host(yq.codes)
    if not np.array_equal(got, rc):
        bad = np.nonzero(got != rc)[0][:8]
        raise AssertionError(f"codes (BA) differ at {bad.tolist()}: got {got[bad]} want {rc[bad]}")
    assert np.array_equal(_host(yq.codes_alt), rc2), "codes (AB) differ"
    assert np.array_equal(_host(yq2.codes), got) and np.array_equal(_host(yq2.scales), rs)
    # the fp32 output: activated convolution of the dequantized operands
    xd = orc.dequantize(*orc.quantize(x, xfmt, block, 0), x.shape, xfmt, block, 0)
    wd = orc.dequantize(*orc.quantize(w, wfmt, block, 0), w.shape, wfmt, block, 0)
    st, pd = L.stride, L.pad
    if full_conv:
        ref, refabs = orc.conv_fwd(xd, wd, st, st, pd, pd)
        idx = np.arange(ref.size)
        ref, refabs = ref.reshape(-1), refabs.reshape(-1)
    else:
        rng = np.random.default_rng(seed)
        nn_, kk, pp, qq = yh.shape
        idx = ((np.arange(nn_)[:, None] * kk + rng.integers(0, kk, (nn_, pp * qq))) * (pp * qq)
               + np.arange(pp * qq)[None, :]).ravel()
        ref, refabs = orc.conv_fwd_at(xd, wd, idx, st, st, pd, pd)
    want = orc.activation(ref, act)
    g = yh.reshape(-1)[idx].astype(np.float64)
    tol = LIP[act] * (1e-3 * refabs + 1e-6) + 1e-6 * np.abs(want)
    bad = ~(np.abs(g - want) <= tol)
    assert not bad.any(), f"{bad.sum()} of {idx.size} fp32 outputs outside tolerance"


CASES = [  # (N, C, H, W, K, R, S, stride, pad)
    (16, 16, 32, 32, 32, 3, 3, 2, 1),      # batch 16: two pixels per warp, stride 2
    (32, 32, 12, 10, 64, 3, 3, 1, 1),      # batch 32: one pixel per warp
    (40, 48, 9, 7, 40, 3, 3, 1, 1),        # ragged batch and channels (padding rows and columns)
    (8, 32, 10, 10, 48, 1, 1, 1, 0),       # batch below 16
    (64, 64, 8, 8, 160, 3, 3, 1, 1),       # two column tiles, K not a multiple of 128
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("yfmt,yblock,act", [(0, 2, 2), (0, 0, 1), (1, 2, 0), (2, 2, 1), (2, 0, 2)])
def test_fwd_quant_parity(mqc, orc, case, yfmt, yblock, act):
    L = synth.Layer(*case)
    x = synth.random_tensor((L.N, L.C, L.H, L.W), seed=sum(case), dist="normal")
    w = synth.random_tensor((L.K, L.C, L.R, L.S), seed=sum(case) + 1, scale=0.05)
    _run(mqc, orc, L, x, w, 0, 0, 2, yfmt, yblock, act)


@pytest.mark.parametrize("layer", range(7))
def test_fwd_quant_yolo_layers(mqc, orc, layer):
    """Every layer of the YOLOv8n training stack that feeds another (0-6),
    at full size, SiLU and SQ32 E4M3 output as the next layer's activation;
    the fp32 output is compared at one seeded channel of every pixel."""
    wl = synth.WORKLOADS[3]
    L = wl.layers[layer]
    x, w, _ = synth.layer_inputs(wl, layer)
    _run(mqc, orc, L, x, w, wl.fmt_x, wl.fmt_w, wl.block, 0, 2, 2, full_conv=False, seed=layer)
