"""The weight gradient that allocates nothing (mqc_conv2d_bwd_weight_noalloc).

Some callers cannot allocate device memory at the call site: plugin hosts
whose memory belongs to someone else and is frozen after start-up, or tight
loops that cannot pay for an allocation per call.  This entry point keeps its
split-K partial sums in a fixed array inside the library instead of a caller
workspace.  Here it is called twice in a row through the C ABI (different
problems, so the second call reuses the array the first one filled) and each
result is compared with the workspace entry point's.  Both run the same plan
and the same fixed-order split-K reduction, so the results must be identical
bit for bit (a partial sum left over from the previous call would show); they
are also checked against the oracle's tolerance, |diff| <= 1e-3 * sum|a*b| +
1e-6 per element.  A problem whose scratch exceeds the array is rejected with
MQC_ERR_WORKSPACE before anything runs, leaving the output untouched.  The
file sorts last so that a failure here stops a run only after every other
test has run.
"""
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


def test_noalloc_weight_gradient_matches_workspace_entry_point(mqc, orc):
    import torch
    cases = [  # (N, C, H, W, K, R, S, stride, pad), both need split-K scratch
        (32, 64, 12, 10, 96, 3, 3, 1, 1),
        (16, 128, 20, 20, 128, 3, 3, 2, 1),
    ]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for i, (N, C, H, W, K, R, S, st, pad) in enumerate(cases):
        P, Q = orc.out_hw(H, W, R, S, st, st, pad, pad)
        x = synth.random_tensor((N, C, H, W), seed=60 + i, dist="student_t")
        g = synth.random_tensor((N, K, P, Q), seed=70 + i, scale=1e-3)
        cv = mqc.conv_desc(N, C, H, W, K, R, S, st, pad)
        gq = mqc.quantize_mx(torch.from_numpy(g).cuda(), mqc.E5M2, mqc.SQ32, mqc.ORDER_AB)
        xq = mqc.quantize_mx(torch.from_numpy(x).cuda(), mqc.E4M3, mqc.SQ32, mqc.ORDER_AB)
        assert 0 < mqc.conv2d_bwd_weight_workspace_bytes(cv, gq.mx, xq.mx) <= mqc.NOALLOC_SCRATCH_BYTES
        ref = mqc.conv2d_bwd_weight(gq, xq, cv)
        out = torch.full((K, C, R, S), float("nan"), dtype=torch.float32, device="cuda")
        P_ = lambda t: ctypes.c_void_p(t.data_ptr())
        st_code = mqc.mqc_conv2d_bwd_weight_noalloc(P_(gq.codes), P_(gq.scales), gq.mx, P_(xq.codes),
                                                    P_(xq.scales), xq.mx, cv, P_(out), stream)
        mqc.check(st_code)
        torch.cuda.synchronize()
        mqc.check(mqc.get_device_status())
        gd = orc.dequantize(*orc.quantize(g, 1, 2, 1), g.shape, 1, 2, 1)
        xd = orc.dequantize(*orc.quantize(x, 0, 2, 1), x.shape, 0, 2, 1)
        _, sabs = orc.conv_wgrad(gd, xd, R, S, st, st, pad, pad)
        a = out.cpu().numpy().astype(np.float64)
        b = ref.cpu().numpy().astype(np.float64)
        assert np.isfinite(a).all()
        assert torch.equal(out, ref), f"call {i}: no-alloc result is not bit-identical to the workspace call"
        assert (np.abs(a - b) <= 1e-3 * sabs + 1e-6).all(), f"call {i}: no-alloc result differs"


def test_noalloc_rejects_problems_above_the_static_scratch(mqc):
    """A weight gradient whose split-K partials need more than the static
    array returns MQC_ERR_WORKSPACE and launches nothing: the NaN-filled
    output is left as it was."""
    import torch
    # E2M1 output gradients: their widened copy alone (one byte per element,
    # 64 x 128 x 56 x 56 = 25.7 MB) is larger than the array, whatever the
    # split-K plan
    N, C, H, W, K, R, S, st, pad = 64, 128, 56, 56, 128, 3, 3, 1, 1
    cv = mqc.conv_desc(N, C, H, W, K, R, S, st, pad)
    gmx, xmx = mqc.MX(mqc.E2M1, mqc.SQ32, mqc.ORDER_AB), mqc.MX(mqc.E4M3, mqc.SQ32, mqc.ORDER_AB)
    need = mqc.conv2d_bwd_weight_workspace_bytes(cv, gmx, xmx)
    assert need > mqc.NOALLOC_SCRATCH_BYTES
    # operands of the right sizes (zeros), so that nothing could read out of bounds
    gq = torch.zeros(mqc.mqc_codes_bytes(gmx, N, K, H, W), dtype=torch.uint8, device="cuda")
    gs = torch.zeros(mqc.mqc_scales_bytes(gmx, N, K, H, W), dtype=torch.uint8, device="cuda")
    xq = torch.zeros(mqc.mqc_codes_bytes(xmx, N, C, H, W), dtype=torch.uint8, device="cuda")
    xs = torch.zeros(mqc.mqc_scales_bytes(xmx, N, C, H, W), dtype=torch.uint8, device="cuda")
    out = torch.full((K, C, R, S), float("nan"), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    P_ = lambda t: ctypes.c_void_p(t.data_ptr())
    code = mqc.mqc_conv2d_bwd_weight_noalloc(P_(gq), P_(gs), gmx, P_(xq), P_(xs), xmx, cv, P_(out), stream)
    assert code == -6, mqc.STATUS.get(code, code)
    assert "static" in mqc.lib.mqc_last_error_message().decode()
    torch.cuda.synchronize()
    mqc.check(mqc.get_device_status())
    assert torch.isnan(out).all()
