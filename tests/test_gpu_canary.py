"""No write lands outside an output or a workspace, and every output element
is written: each GEMM plan (units of several row tiles, column tiles, the
sub-pixel input gradient with paired and unpaired depth-to-space stores, the
per-phase input gradient, the weight gradient with 16-byte rows and window
boxes, with per-tap boxes and with 128-byte rows) runs into buffers with
16 KB guard bands filled with a sentinel.  The guarded result must also equal
an unguarded call bit for bit (the kernels are deterministic, the split-K
sum has a fixed order)."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu
GUARD = 4096                 # fp32 elements (16 KB) on each side
SENT = -12345.5              # never a result of these inputs
WS_SENT = 0xA5

# (N, C, H, W, K, R, S, stride, pad)
FWD = [(16, 16, 20, 20, 32, 3, 3, 2, 1), (3, 128, 10, 9, 160, 3, 3, 1, 1)]
DGRAD = [(16, 16, 12, 12, 32, 3, 3, 2, 1), (2, 48, 6, 8, 40, 3, 3, 2, 1), (2, 32, 11, 10, 48, 3, 3, 3, 1),
         (4, 40, 9, 11, 48, 3, 3, 2, 1)]
WGRAD = [(16, 16, 12, 12, 32, 3, 3, 2, 1), (40, 96, 5, 6, 130, 3, 3, 1, 1), (128, 16, 6, 6, 32, 3, 3, 2, 1)]


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


def _guarded_out(shape):
    import torch
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * GUARD,), SENT, dtype=torch.float32, device="cuda")
    return buf, buf[GUARD:GUARD + n].view(shape)


def _guarded_ws(nbytes):
    import torch
    if nbytes == 0:
        return None, None
    buf = torch.full((nbytes + 8 * GUARD,), WS_SENT, dtype=torch.uint8, device="cuda")
    return buf, buf[4 * GUARD:4 * GUARD + nbytes]


def _check(name, buf, out, ref, wbuf, nbytes):
    import torch
    torch.cuda.synchronize()
    h = buf.cpu().numpy()
    n = out.numel()
    assert (h[:GUARD] == SENT).all() and (h[GUARD + n:] == SENT).all(), f"{name}: a write outside the output"
    assert not (h[GUARD:GUARD + n] == SENT).any(), f"{name}: output elements left unwritten"
    if wbuf is not None:
        w = wbuf.cpu().numpy()
        assert (w[:4 * GUARD] == WS_SENT).all() and (w[4 * GUARD + nbytes:] == WS_SENT).all(), \
            f"{name}: a write outside the workspace"
    assert torch.equal(out, ref), f"{name}: guarded and unguarded results differ"


def _inputs(case):
    N, C, H, W, K, R, S, st, pad = case
    P, Q = (H + 2 * pad - R) // st + 1, (W + 2 * pad - S) // st + 1
    x = synth.random_tensor((N, C, H, W), seed=71, dist="student_t")
    w = synth.random_tensor((K, C, R, S), seed=72, scale=0.05)
    g = synth.random_tensor((N, K, P, Q), seed=73, scale=1e-3)
    return x, w, g, P, Q


@pytest.mark.parametrize("case", FWD)
def test_forward_writes_stay_inside(mqc, case):
    N, C, H, W, K, R, S, st, pad = case
    x, w, _, P, Q = _inputs(case)
    cv = mqc.conv_desc(N, C, H, W, K, R, S, st, pad)
    xq, wq = mqc.quantize_mx(_dev(x), 0, 2, 0), mqc.quantize_mx(_dev(w), 0, 2, 0)
    ref = mqc.conv2d_fwd(xq, wq, cv)
    nbytes = mqc.mqc_conv2d_fwd_workspace_bytes(cv, xq.mx, wq.mx)
    buf, out = _guarded_out((N, K, P, Q))
    wbuf, ws = _guarded_ws(nbytes)
    mqc.conv2d_fwd(xq, wq, cv, out=out, workspace=ws)
    _check(f"fwd {case}", buf, out, ref, wbuf, nbytes)


@pytest.mark.parametrize("case", DGRAD)
def test_input_gradient_writes_stay_inside(mqc, case):
    N, C, H, W, K, R, S, st, pad = case
    _, w, g, _, _ = _inputs(case)
    cv = mqc.conv_desc(N, C, H, W, K, R, S, st, pad)
    wq, gq = mqc.quantize_mx(_dev(w), 0, 2, 1), mqc.quantize_mx(_dev(g), 1, 2, 0)
    ref = mqc.conv2d_bwd_data(wq, gq, cv)
    nbytes = mqc.mqc_conv2d_bwd_data_workspace_bytes(cv, wq.mx, gq.mx)
    buf, out = _guarded_out((N, C, H, W))
    wbuf, ws = _guarded_ws(nbytes)
    mqc.conv2d_bwd_data(wq, gq, cv, out=out, workspace=ws)
    _check(f"dgrad {case}", buf, out, ref, wbuf, nbytes)


@pytest.mark.parametrize("case", WGRAD)
def test_weight_gradient_writes_stay_inside(mqc, case):
    N, C, H, W, K, R, S, st, pad = case
    x, _, g, _, _ = _inputs(case)
    cv = mqc.conv_desc(N, C, H, W, K, R, S, st, pad)
    gq, xq = mqc.quantize_mx(_dev(g), 1, 2, 1), mqc.quantize_mx(_dev(x), 0, 2, 1)
    ref = mqc.conv2d_bwd_weight(gq, xq, cv)
    nbytes = mqc.conv2d_bwd_weight_workspace_bytes(cv, gq.mx, xq.mx)
    buf, out = _guarded_out((K, C, R, S))
    wbuf, ws = _guarded_ws(nbytes)
    mqc.conv2d_bwd_weight(gq, xq, cv, out=out, workspace=ws)
    _check(f"wgrad {case}", buf, out, ref, wbuf, nbytes)
