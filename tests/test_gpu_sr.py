"""Parity of the stochastically rounded CUDA quantizer (mqc_quantize_mx_sr)
with the oracle (MicroQonv paper, section III-A, Eq. 6: gradients are
rounded stochastically).  Both sides draw the same Philox4x64-10 bits from
(seed, offset) and the element position, so codes and scales must be
bit-identical, in both code orders, for every format and block mode, on
ragged shapes that span several tiles and at the full size of the training
benchmark's output gradients."""
import ctypes

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


def _check(mqc, orc, x, fmt, block, seed, offset, dual=True):
    q = mqc.quantize_mx(_dev(x), fmt, block, mqc.ORDER_BA, both_orders=dual, sr_seed=seed, sr_offset=offset)
    mqc.check(mqc.get_device_status())
    rc, rs = orc.quantize_sr(x, fmt, block, 0, seed, offset)
    assert np.array_equal(_host(q.scales), rs), "scales differ"
    got = _host(q.codes)
    if not np.array_equal(got, rc):
        bad = np.nonzero(got != rc)[0][:8]
        raise AssertionError(f"codes (BA) differ at {bad}: got {got[bad]} want {rc[bad]}")
    if dual:
        rc2, _ = orc.quantize_sr(x, fmt, block, 1, seed, offset)
        assert np.array_equal(_host(q.codes_alt), rc2), "codes (AB) differ"
    return q


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("block", [0, 1, 2])
# ragged B and A axes; spatial planes of whole 16-byte rows (the NCHW-like
# sources the stochastic path takes), not multiples of a tile's positions
@pytest.mark.parametrize("shape", [(37, 45, 3, 4), (16, 40, 6, 6), (64, 96, 4, 4), (5, 16, 11, 12), (33, 70, 5, 4)])
def test_sr_quantize_parity(mqc, orc, fmt, block, shape):
    x = synth.random_tensor(shape, seed=hash((fmt, block, shape)) % 1000, dist="student_t", scale=1e-3)
    _check(mqc, orc, x, fmt, block, seed=2024 + fmt, offset=7, dual=True)
    _check(mqc, orc, x, fmt, block, seed=2024 + fmt, offset=8, dual=False)


def test_sr_differs_from_nearest_and_between_offsets(mqc, orc):
    x = synth.random_tensor((32, 64, 8, 8), seed=3, scale=1e-3)
    a = _check(mqc, orc, x, 1, 2, seed=11, offset=0)
    b = _check(mqc, orc, x, 1, 2, seed=11, offset=1)
    rn = mqc.quantize_mx(_dev(x), 1, 2, mqc.ORDER_BA)
    ca, cb, cr = _host(a.codes), _host(b.codes), _host(rn.codes)
    assert not np.array_equal(ca, cb)
    assert not np.array_equal(ca, cr)
    assert np.array_equal(_host(a.scales), _host(rn.scales))


@pytest.mark.parametrize("wl_key,fmt_attr", [(3, "fmt_g"), ((5, "fp4", 128), "fmt_g")])
def test_sr_full_size_output_gradient(mqc, orc, wl_key, fmt_attr):
    """The output gradient of the largest layer of the YOLOv8n training step
    (16 x 32 x 320 x 320, E5M2) and of the MXFP4 large-batch layer (128 x 128
    x 80 x 80, E2M1), SQ32 blocks, both orders, compared in full."""
    wl = synth.WORKLOADS[wl_key]
    _, _, g = synth.layer_inputs(wl, 0)
    _check(mqc, orc, g, getattr(wl, fmt_attr), wl.block, seed=5, offset=123456789)


def test_sr_rejects_unsupported_layouts_before_launch(mqc):
    import torch
    x = torch.zeros((4, 32, 8, 8), dtype=torch.float32, device="cuda")
    codes = torch.zeros(4 * 32 * 8 * 8, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(4 * 32 * 8 * 8, dtype=torch.uint8, device="cuda")
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    d = mqc.T4(4, 32, 8, 8, *x.stride())
    # the primary order must be BA
    assert mqc.mqc_quantize_mx_sr(P(x), d, mqc.MX(0, 2, 1), P(codes), P(scales), None, 1, 0, s) == -2
    # positions must be contiguous
    xt = x.permute(0, 1, 3, 2)
    dt = mqc.T4(4, 32, 8, 8, *xt.stride())
    assert mqc.mqc_quantize_mx_sr(P(xt), dt, mqc.MX(0, 2, 0), P(codes), P(scales), None, 1, 0, s) == -2
    torch.cuda.synchronize()
    mqc.check(mqc.get_device_status())
    assert (codes == 0).all()
