"""Parity of the CUDA quantizer and the explicit channel-batch-first im2col
with the oracle: codes and scales must be bit-identical."""
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


EMAX = {0: 8, 1: 15, 2: 2}
LOW_BINADE = {0: -12, 1: -18, 2: -3}   # below half the smallest subnormal everything rounds to 0


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_element_encoding_every_fp32_in_range(mqc, orc, fmt):
    """Every fp32 bit pattern whose binade can round to a non-zero code, in
    blocks whose maximum fixes the scale at 2^0, encodes exactly as the oracle
    encodes it (RNE, saturation, subnormals, signed zero)."""
    emax = EMAX[fmt]
    mant = np.arange(1 << 23, dtype=np.uint32)
    for e in range(LOW_BINADE[fmt], emax + 1):
        for sign in (0, 1):
            bits = (np.uint32(sign << 31) | np.uint32((e + 127) << 23) | mant)
            vals = bits.view(np.float32)
            nb = -(-vals.size // 31)
            x = np.zeros((1, 32, 1, nb), dtype=np.float32)
            x[0, 0, 0, :] = np.float32(2.0 ** emax)     # block max in [2^emax, 2^(emax+1)) -> scale 2^0
            flat = np.zeros(nb * 31, dtype=np.float32)
            flat[:vals.size] = vals
            x[0, 1:, 0, :] = flat.reshape(nb, 31).T
            q = mqc.quantize_mx(_dev(x), fmt, 0, 0)
            ref_c, ref_s = orc.quantize(x, fmt, 0, 0)
            got_c, got_s = _host(q.codes), _host(q.scales)
            assert (ref_s == 127).all()
            assert np.array_equal(got_s, ref_s), (fmt, e, sign)
            if not np.array_equal(got_c, ref_c):
                bad = np.nonzero(got_c != ref_c)[0][:8]
                raise AssertionError(f"fmt {fmt} binade 2^{e} sign {sign}: first mismatches at {bad}: "
                                     f"got {got_c[bad]} want {ref_c[bad]}")
    # zeros of both signs and the saturation end of the top binade
    x = np.zeros((1, 32, 1, 1), dtype=np.float32)
    x[0, :, 0, 0] = [2.0 ** emax, -0.0, 0.0, orc.max_finite(fmt), -orc.max_finite(fmt)] + \
                    [np.nextafter(np.float32(2.0 ** (emax + 1)), np.float32(0)) * (-1) ** i for i in range(27)]
    q = mqc.quantize_mx(_dev(x), fmt, 0, 0)
    assert np.array_equal(_host(q.codes), orc.quantize(x, fmt, 0, 0)[0])


SHAPES = [(2, 32, 8, 8), (37, 45, 3, 5), (16, 16, 33, 17), (64, 96, 4, 6), (5, 3, 2, 40), (40, 70, 1, 1),
          (24, 40, 4, 8)]


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("block", [0, 1, 2])
@pytest.mark.parametrize("order", [0, 1])
def test_quantize_parity(mqc, orc, fmt, block, order):
    for i, shape in enumerate(SHAPES):
        x = synth.random_tensor(shape, seed=300 + i, dist="uniform_exp" if i % 2 else "student_t")
        q = mqc.quantize_mx(_dev(x), fmt, block, order, both_orders=True)
        rc, rs = orc.quantize(x, fmt, block, order)
        rc2, _ = orc.quantize(x, fmt, block, 1 - order)
        assert np.array_equal(_host(q.scales), rs), (shape, "scales")
        assert np.array_equal(_host(q.codes), rc), (shape, "codes")
        assert np.array_equal(_host(q.codes_alt), rc2), (shape, "codes in the second order")


def test_quantize_strided_source(mqc, orc):
    import torch
    x = synth.random_tensor((24, 40, 6, 7), seed=41)
    xt = torch.from_numpy(x).cuda().permute(2, 3, 0, 1).contiguous().permute(2, 3, 0, 1)   # not NCHW-contiguous
    for block in (0, 1, 2):
        q = mqc.quantize_mx(xt, 0, block, 0)
        rc, rs = orc.quantize(x, 0, block, 0)
        assert np.array_equal(_host(q.codes), rc) and np.array_equal(_host(q.scales), rs)


def test_quantize_edge_values(mqc, orc):
    """All-zero blocks (scale 0x00), tiny maxima clamped at 2^-127, fp32
    subnormals, huge values, exact powers of two and ties."""
    x = np.zeros((32, 64, 2, 3), dtype=np.float32)
    x[:, :32, 0, 0] = 1e-40                        # subnormal block max -> clamped scale
    x[:, :32, 0, 1] = np.float32(3.0e38)           # near FLT_MAX
    x[:, 32:, 0, 1] = 2.0 ** np.arange(-16, 16, dtype=np.float32)[None, :]
    x[:5, :, 1, 0] = 1.0 + 2.0 ** -4               # E4M3 tie (between 1 and 1.125)
    x[5:9, :, 1, 2] = -(1.0 + 3 * 2.0 ** -5)
    for fmt in (0, 1, 2):
        for block in (0, 1, 2):
            q = mqc.quantize_mx(_dev(x), fmt, block, 0)
            rc, rs = orc.quantize(x, fmt, block, 0)
            assert np.array_equal(_host(q.codes), rc) and np.array_equal(_host(q.scales), rs), (fmt, block)


GEOMS = [(2, 32, 8, 8, 3, 3, 1, 1), (3, 64, 9, 7, 3, 3, 2, 1), (32, 32, 5, 5, 1, 1, 1, 0), (4, 48, 6, 6, 2, 2, 1, 1),
         (40, 16, 7, 5, 3, 3, 2, 0)]


@pytest.mark.parametrize("fmt", [0, 2])
@pytest.mark.parametrize("block", [0, 1, 2])
@pytest.mark.parametrize("order", [0, 1])
def test_im2col_cbf_parity(mqc, orc, fmt, block, order):
    for i, (N, C, H, W, R, S, st, pad) in enumerate(GEOMS):
        x = synth.random_tensor((N, C, H, W), seed=500 + i, dist="student_t")
        xq = mqc.quantize_mx(_dev(x), fmt, block, order)
        cv = mqc.conv_desc(N, C, H, W, 8, R, S, st, pad)
        co, so = mqc.im2col_cbf(xq, cv)
        rc, rs = orc.quantize(x, fmt, block, order)
        eco, eso = orc.im2col_cbf(rc, rs, N, C, H, W, R, S, st, st, pad, pad, fmt, block, order)
        assert np.array_equal(_host(co), eco), (N, C, H, W, R, S, st, pad)
        assert np.array_equal(_host(so), eso), (N, C, H, W, R, S, st, pad)


def test_quantize_batch_equals_single_calls(mqc, orc):
    """mqc_quantize_mx_batch: the eight weight tensors of the YOLOv8n training
    stack (3x3 and 1x1 kernels, E4M3, SQ32, both orders) in one launch, and a
    set of small ragged tensors in A32 / B32 and E2M1, bit-identical to the
    oracle's quantization of each tensor."""
    wl = synth.WORKLOADS[3]
    ws = [synth.layer_inputs(wl, i)[1] for i in range(len(wl.layers))]
    qs = mqc.quantize_mx_batch([_dev(w) for w in ws], 0, 2, 0, both_orders=True)
    for w, q in zip(ws, qs):
        rc, rs = orc.quantize(w, 0, 2, 0)
        assert np.array_equal(_host(q.codes), rc) and np.array_equal(_host(q.scales), rs)
        assert np.array_equal(_host(q.codes_alt), orc.quantize(w, 0, 2, 1)[0])
    small = [synth.random_tensor(s, seed=40 + i, dist="student_t")
             for i, s in enumerate([(37, 45, 3, 3), (16, 40, 1, 1), (70, 33, 2, 5), (5, 16, 4, 4)])]
    for fmt, blk, order in ((2, 0, 0), (0, 1, 1), (1, 1, 0)):
        qs = mqc.quantize_mx_batch([_dev(x) for x in small], fmt, blk, order, both_orders=(fmt == 0))
        for x, q in zip(small, qs):
            rc, rs = orc.quantize(x, fmt, blk, order)
            assert np.array_equal(_host(q.codes), rc), (fmt, blk, order, x.shape)
            assert np.array_equal(_host(q.scales), rs), (fmt, blk, order, x.shape)
            if fmt == 0:
                assert np.array_equal(_host(q.codes_alt), orc.quantize(x, fmt, blk, 1 - order)[0])
    mqc.check(mqc.get_device_status())
