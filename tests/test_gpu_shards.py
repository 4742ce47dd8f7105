"""The data-parallel split of the path on one GPU: the weight gradients of two
batch shards of 32 images, computed by the library shard by shard and summed
(the sum the NCCL all-reduce of a two-GPU run performs), match the oracle's
weight gradient of the concatenated batch of 64 within 1e-3 * sum|ab| + 1e-6.
With the per-shard batch a multiple of 32, the 32-long blocks along N (B32,
SQ32) never straddle two shards, so each shard's codes and scales are those
of the global batch's quantization, sliced (checked first)."""
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


@pytest.mark.parametrize("case", [(64, 32, 20, 20, 64, 3, 3, 1, 1), (64, 16, 32, 32, 32, 3, 3, 2, 1)])
def test_two_shards_sum_to_the_global_weight_gradient(mqc, orc, case):
    N, C, H, W, K, R, S, st, pad = case
    P, Q = orc.out_hw(H, W, R, S, st, st, pad, pad)
    x = synth.random_tensor((N, C, H, W), seed=sum(case), dist="student_t")
    g = synth.random_tensor((N, K, P, Q), seed=sum(case) + 1, scale=1e-3)
    half = N // 2
    cvh = mqc.conv_desc(half, C, H, W, K, R, S, st, pad)
    gw = None
    for sh in range(2):
        xs, gs = x[sh * half:(sh + 1) * half], g[sh * half:(sh + 1) * half]
        xq = mqc.quantize_mx(_dev(xs), mqc.E4M3, mqc.SQ32, mqc.ORDER_AB)
        gq = mqc.quantize_mx(_dev(gs), mqc.E5M2, mqc.SQ32, mqc.ORDER_AB)
        # the shard's quantization is the global one restricted to the shard
        for t, q, f in ((xs, xq, 0), (gs, gq, 1)):
            rc, rs = orc.quantize(np.ascontiguousarray(t), f, 2, 1)
            assert np.array_equal(_host(q.codes), rc) and np.array_equal(_host(q.scales), rs)
        part = mqc.conv2d_bwd_weight(gq, xq, cvh)
        gw = part if gw is None else gw + part
    mqc.check(mqc.get_device_status())
    # global batch: the oracle's quantization of all 64 images, one weight gradient
    gd = orc.dequantize(*orc.quantize(g, 1, 2, 1), g.shape, 1, 2, 1)
    xd = orc.dequantize(*orc.quantize(x, 0, 2, 1), x.shape, 0, 2, 1)
    # slices of the global dequantization equal the shards' (blocks do not straddle)
    for sh in range(2):
        sl = slice(sh * half, (sh + 1) * half)
        xs = np.ascontiguousarray(x[sl])
        assert np.array_equal(orc.dequantize(*orc.quantize(xs, 0, 2, 1), xs.shape, 0, 2, 1), xd[sl])
    ref, refabs = orc.conv_wgrad(gd, xd, R, S, st, st, pad, pad)
    err = np.abs(_host(gw).astype(np.float64) - ref)
    assert (err <= 1e-3 * refabs + 1e-6).all()
