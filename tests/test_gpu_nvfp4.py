"""Parity of the CUDA NVFP4 quantizer (mqc_quantize_nvfp4; MicroQonv paper,
section III-A, Eq. 4-6) with the oracle: the per-tensor scale, the E4M3
block scales and the E2M1 codes in both orders must be bit-identical, for
lines of 16 along either axis and 16 x 16 squares, on ragged shapes and a
full-size large-batch activation."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


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


def _check(mqc, orc, x, block, order):
    q = mqc.quantize_nvfp4(_dev(x), block, order, both_orders=True)
    mqc.check(mqc.get_device_status())
    rc, rs, rt = orc.quantize_nvfp4(x, block, order)
    assert _host(q.tscale)[0] == np.float32(rt)
    assert np.array_equal(_host(q.scales), rs), "block scales differ"
    got = _host(q.codes)
    if not np.array_equal(got, rc):
        bad = np.nonzero(got != rc)[0][:8]
        raise AssertionError(f"codes differ at {bad.tolist()}: got {got[bad]} want {rc[bad]}")
    rc2, _, _ = orc.quantize_nvfp4(x, block, 1 - order)
    assert np.array_equal(_host(q.codes_alt), rc2), "second-order codes differ"


@pytest.mark.parametrize("block", [0, 1, 2])
@pytest.mark.parametrize("order", [0, 1])
@pytest.mark.parametrize("shape", [(37, 45, 3, 4), (16, 40, 6, 6), (64, 96, 4, 4), (5, 16, 11, 12), (20, 33, 1, 1)])
def test_nvfp4_quantize_parity(mqc, orc, block, order, shape):
    x = synth.random_tensor(shape, seed=sum(shape) + 7 * block + order, dist="student_t")
    _check(mqc, orc, x, block, order)


def test_nvfp4_zero_tensor_and_signed_zero(mqc, orc):
    z = np.zeros((4, 32, 2, 2), dtype=np.float32)
    _check(mqc, orc, z, 2, 0)
    x = synth.random_tensor((4, 32, 2, 2), seed=3)
    x[:, :16] = np.float32(-0.0)            # blocks of negative zeros next to real blocks
    _check(mqc, orc, x, 0, 0)


@pytest.mark.parametrize("block", [0, 2])
def test_nvfp4_full_size_large_batch(mqc, orc, block):
    """The MXFP4 large-batch activation (128 x 128 x 80 x 80, Student-t) in
    NVFP4 instead, compared in full."""
    wl = synth.WORKLOADS[(5, "fp4", 128)]
    x, _, _ = synth.layer_inputs(wl, 0)
    _check(mqc, orc, x, block, 0)


FWD_CASES = [  # (N, C, H, W, K, R, S, stride, pad)
    (2, 32, 8, 8, 32, 3, 3, 1, 1),
    (16, 16, 32, 32, 32, 3, 3, 2, 1),      # C = 16: half of each 64-code K-block is padding
    (32, 64, 12, 10, 64, 3, 3, 1, 1),
    (8, 128, 10, 10, 160, 1, 1, 1, 0),     # two column tiles, K not a multiple of 128
    (5, 40, 9, 7, 40, 3, 3, 1, 1),         # ragged channels and batch
    (128, 256, 14, 14, 256, 3, 3, 1, 1),   # the latent-replay block's shape
]


@pytest.mark.parametrize("case", FWD_CASES)
@pytest.mark.parametrize("xb,wb", [(0, 0), (2, 2), (0, 2)])
def test_nvfp4_forward_parity(mqc, orc, case, xb, wb):
    """mqc_conv2d_fwd_nvfp4 (tcgen05 kind::mxf4nvf4 with the per-tensor scales
    in the epilogue) against the oracle's double convolution of the
    dequantized NVFP4 operands: |err| <= 1e-3 * sum|a*b| + 1e-6 per element
    (every element for the small cases, one channel of every pixel for the
    largest)."""
    N, C, H, W, K, R, S, st, pad = case
    x = synth.random_tensor((N, C, H, W), seed=sum(case) + xb, dist="student_t")
    w = synth.random_tensor((K, C, R, S), seed=sum(case) + 10 + wb, scale=0.05)
    xq = mqc.quantize_nvfp4(_dev(x), xb, 0)
    wq = mqc.quantize_nvfp4(_dev(w), wb, 0)
    cv = mqc.conv_desc(N, C, H, W, K, R, S, st, pad)
    y = mqc.conv2d_fwd_nvfp4(xq, wq, cv)
    mqc.check(mqc.get_device_status())
    xd = orc.dequantize_nvfp4(*orc.quantize_nvfp4(x, xb, 0), x.shape, xb, 0)
    wd = orc.dequantize_nvfp4(*orc.quantize_nvfp4(w, wb, 0), w.shape, wb, 0)
    yh = _host(y).astype(np.float64)
    if N * K * H * W <= 2_000_000:
        ref, refabs = orc.conv_fwd(xd, wd, st, st, pad, pad)
        got, ref, refabs = yh.reshape(-1), ref.reshape(-1), refabs.reshape(-1)
    else:
        rng = np.random.default_rng(1)
        nn_, kk, pp, qq = yh.shape
        idx = ((np.arange(nn_)[:, None] * kk + rng.integers(0, kk, (nn_, pp * qq))) * (pp * qq)
               + np.arange(pp * qq)[None, :]).ravel()
        ref, refabs = orc.conv_fwd_at(xd, wd, idx, st, st, pad, pad)
        got = yh.reshape(-1)[idx]
    bad = ~(np.abs(got - ref) <= 1e-3 * refabs + 1e-6)
    assert not bad.any(), f"{bad.sum()} of {got.size} outputs outside tolerance"
