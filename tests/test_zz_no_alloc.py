"""The weight gradient that allocates nothing (mqc_conv2d_bwd_weight_noalloc).

Some callers cannot allocate device memory at the call site: plugin hosts
whose memory belongs to someone else and is frozen after start-up, or tight
loops that cannot pay for an allocation per call.  This entry point keeps its
split-K partial sums in a fixed array inside the library instead of a caller
workspace.  Here it is called twice in a row through the C ABI (different
problems, so the second call reuses the array the first one filled) and each
result is compared with the workspace entry point's, within the tolerance the
parity tests use: |diff| <= 1e-3 * sum|a*b| + 1e-6 per element, sum|a*b| from
the oracle.  The file sorts last so that a failure here stops a run only
after every other test has run.
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
        assert (np.abs(a - b) <= 1e-3 * sabs + 1e-6).all(), f"call {i}: no-alloc result differs"
