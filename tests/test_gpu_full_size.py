"""Parity at the benchmark's full sizes, in the launch configuration the
benchmark times: every layer of the YOLOv8n-shaped N=16 640x640 training
stack, the N=128, C=128, 80x80 MXFP8 and MXFP4 layers (MXFP4 also at
N=32) and the latent-replay block (E2M1 activations), with the benchmark's own
seeded inputs and the same C-ABI entry points (the library picks the tiling
from the problem shape, so these are the benchmark's kernel launches).

- Quantization (MicroQonv paper, section III-A, Eq. 5-7): the codes of X,
  W and G_Y in both orders and their E8M0 scales are compared with the
  oracle's in full, bit for bit.
- Convolutions (section II-C3, Eq. 1-3): the forward output and the input
  gradient on 65,536 seeded elements plus every border pixel of image 0,
  the weight gradient on 768 seeded elements (each a sum over N x P x Q);
  each computed by the oracle on its own dequantized operands as a sum in
  double, within |err| <= 1e-3 * sum|a*b| + 1e-6.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu
RTOL, ATOL = 1e-3, 1e-6
CASES = [(3, i) for i in range(8)] + [((5, "fp8", 128), 0), (4, 0), ((5, "fp4", 32), 0), ((5, "fp4", 128), 0)]
# mid-sized layers (YOLO-like, N = 16) whose tile count gives units of two
# 128-row sub-tiles rather than four
MID = [synth.Layer(16, 16, 160, 160, 32, 3, 3, 2, 1), synth.Layer(16, 32, 80, 80, 32, 1, 1, 1, 0)]


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


def _sample(shape, n, seed, border=False):
    """Seeded flat indices into an output of `shape`; with border, also every
    border pixel (first/last row and column) of image 0, all channels."""
    rng = np.random.default_rng(seed)
    size = int(np.prod(shape))
    idx = [rng.integers(0, size, size=min(n, size), dtype=np.int64)]
    if border:
        _, ch, hh, ww = shape
        m = np.zeros((hh, ww), dtype=bool)
        m[0, :] = m[-1, :] = m[:, 0] = m[:, -1] = True
        pix = np.flatnonzero(m)
        idx.append((np.arange(ch, dtype=np.int64)[:, None] * (hh * ww) + pix[None, :]).ravel())
    return np.unique(np.concatenate(idx))


def _check(name, got, idx, ref, refabs):
    g = got.reshape(-1)[idx].astype(np.float64)
    err = np.abs(g - ref)
    bad = ~(err <= RTOL * refabs + ATOL)
    if bad.any():
        k = np.nonzero(bad)[0][:6]
        raise AssertionError(f"{name}: {bad.sum()} of {idx.size} sampled outputs outside tolerance; "
                             f"first flat indices {idx[k].tolist()} got {g[k].tolist()} want {ref[k].tolist()}")


@pytest.mark.parametrize("wl_key,layer", CASES, ids=[f"{k}-L{i}" for k, i in CASES])
def test_full_size_layer(mqc, orc, wl_key, layer):
    wl = synth.WORKLOADS[wl_key]
    _layer_parity(mqc, orc, wl, layer)


@pytest.mark.parametrize("k", range(len(MID)))
def test_mid_size_layer(mqc, orc, k):
    base = synth.WORKLOADS[3]
    wl = synth.Workload(f"mid-{k}", 30 + k, (MID[k],), base.fmt_x, base.fmt_w, base.fmt_g, base.block, True,
                        base.dist, base.w_std)
    _layer_parity(mqc, orc, wl, 0)


def _layer_parity(mqc, orc, wl, layer):
    L = wl.layers[layer]
    x, w, g = synth.layer_inputs(wl, layer)
    BA, AB = mqc.ORDER_BA, mqc.ORDER_AB

    # the path: each tensor quantized once, both code orders
    xq = mqc.quantize_mx(_dev(x), wl.fmt_x, wl.block, BA, both_orders=True)
    wq = mqc.quantize_mx(_dev(w), wl.fmt_w, wl.block, BA, both_orders=True)
    gq = mqc.quantize_mx(_dev(g), wl.fmt_g, wl.block, BA, both_orders=True)
    cv = mqc.conv_desc(L.N, L.C, L.H, L.W, L.K, L.R, L.S, L.stride, L.pad)
    y = mqc.conv2d_fwd(xq, wq, cv)
    gx = mqc.conv2d_bwd_data(wq.other_order(), gq, cv)
    gw = mqc.conv2d_bwd_weight(gq.other_order(), xq.other_order(), cv)
    mqc.check(mqc.get_device_status())

    # the oracle's own quantization, compared in full
    deq = {}
    for name, t, q, f in (("X", x, xq, wl.fmt_x), ("W", w, wq, wl.fmt_w), ("G_Y", g, gq, wl.fmt_g)):
        rc, rs = orc.quantize(t, f, wl.block, BA)
        assert np.array_equal(_host(q.scales), rs), f"{name}: scales differ"
        assert np.array_equal(_host(q.codes), rc), f"{name}: codes (order BA) differ"
        rc2, _ = orc.quantize(t, f, wl.block, AB)
        assert np.array_equal(_host(q.codes_alt), rc2), f"{name}: codes (order AB) differ"
        deq[name] = orc.dequantize(rc, rs, t.shape, f, wl.block, BA)

    st, pd = L.stride, L.pad
    yi = _sample(y.shape, 65536, 11 + layer, border=True)
    ref, refabs = orc.conv_fwd_at(deq["X"], deq["W"], yi, st, st, pd, pd)
    _check(f"fwd {wl.name} layer {layer}", _host(y), yi, ref, refabs)

    gi = _sample(gx.shape, 65536, 12 + layer, border=True)
    ref, refabs = orc.conv_dgrad_at(deq["W"], deq["G_Y"], L.H, L.W, gi, st, st, pd, pd)
    _check(f"dgrad {wl.name} layer {layer}", _host(gx), gi, ref, refabs)

    wi = _sample(gw.shape, 768, 13 + layer)
    ref, refabs = orc.conv_wgrad_at(deq["G_Y"], deq["X"], L.R, L.S, wi, st, st, pd, pd)
    _check(f"wgrad {wl.name} layer {layer}", _host(gw), wi, ref, refabs)
