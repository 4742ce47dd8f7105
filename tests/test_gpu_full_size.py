"""Parity at the benchmark's full sizes, in the launch configuration the
benchmark times: every layer of the YOLOv8n-shaped N=16 640x640 training
stack and of its forward-only A32 twin, the 80x80 C=K=128 large-batch layer
at every batch of the sweep (N = 32, 64, 128, 256) in MXFP8 and MXFP4, and
the latent-replay block (E2M1 activations), with the benchmark's own seeded
inputs and the same C-ABI entry points (the library picks the tiling from
the problem shape, so these are the benchmark's kernel launches).

- Quantization (MicroQonv paper, section III-A, Eq. 5-7): the codes of X,
  W and G_Y in both orders and their E8M0 scales are compared with the
  oracle's in full, bit for bit.
- Convolutions (section II-C3, Eq. 1-3), each output computed by the oracle
  on its own dequantized operands as a sum in double, within |err| <= 1e-3 *
  sum|a*b| + 1e-6:
  - forward output and input gradient: one seeded channel at EVERY output
    pixel (n, p, q) (so every 128-row tile of every plan, and with millions
    of pixels every column tile, is compared), plus 65,536 seeded elements
    and every border pixel of image 0 in all channels;
  - weight gradient: every element.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu
RTOL, ATOL = 1e-3, 1e-6
CASES = ([(3, i) for i in range(8)] + [(2, i) for i in range(8)] + [(4, 0)]
         + [((5, "fp8", n), 0) for n in (32, 64, 128, 256)] + [((5, "fp4", n), 0) for n in (32, 64, 128, 256)])
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


def _sample(shape, n, seed):
    """Seeded flat indices into an NCHW output of `shape`: one seeded channel
    at every pixel (n, h, w), n seeded elements anywhere, and every border
    pixel (first/last row and column) of image 0 in all channels."""
    rng = np.random.default_rng(seed)
    nn, ch, hh, ww = shape
    size = int(np.prod(shape))
    idx = [rng.integers(0, size, size=min(n, size), dtype=np.int64)]
    img = np.arange(nn, dtype=np.int64)[:, None]
    pix = np.arange(hh * ww, dtype=np.int64)[None, :]
    c = rng.integers(0, ch, size=(nn, hh * ww), dtype=np.int64)
    idx.append(((img * ch + c) * (hh * ww) + pix).ravel())
    m = np.zeros((hh, ww), dtype=bool)
    m[0, :] = m[-1, :] = m[:, 0] = m[:, -1] = True
    border = np.flatnonzero(m)
    idx.append((np.arange(ch, dtype=np.int64)[:, None] * (hh * ww) + border[None, :]).ravel())
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
    two = wl.backward          # the training step needs both code orders

    # the path: each tensor quantized once (both code orders for training)
    xq = mqc.quantize_mx(_dev(x), wl.fmt_x, wl.block, BA, both_orders=two)
    wq = mqc.quantize_mx(_dev(w), wl.fmt_w, wl.block, BA, both_orders=two)
    cv = mqc.conv_desc(L.N, L.C, L.H, L.W, L.K, L.R, L.S, L.stride, L.pad)
    y = mqc.conv2d_fwd(xq, wq, cv)
    tensors = [("X", x, xq, wl.fmt_x), ("W", w, wq, wl.fmt_w)]
    if two:
        gq = mqc.quantize_mx(_dev(g), wl.fmt_g, wl.block, BA, both_orders=True)
        gx = mqc.conv2d_bwd_data(wq.other_order(), gq, cv)
        gw = mqc.conv2d_bwd_weight(gq.other_order(), xq.other_order(), cv)
        tensors.append(("G_Y", g, gq, wl.fmt_g))
    mqc.check(mqc.get_device_status())

    # the oracle's own quantization, compared in full
    deq = {}
    for name, t, q, f in tensors:
        rc, rs = orc.quantize(t, f, wl.block, BA)
        assert np.array_equal(_host(q.scales), rs), f"{name}: scales differ"
        assert np.array_equal(_host(q.codes), rc), f"{name}: codes (order BA) differ"
        if two:
            rc2, _ = orc.quantize(t, f, wl.block, AB)
            assert np.array_equal(_host(q.codes_alt), rc2), f"{name}: codes (order AB) differ"
        deq[name] = orc.dequantize(rc, rs, t.shape, f, wl.block, BA)

    st, pd = L.stride, L.pad
    yi = _sample(y.shape, 65536, 11 + layer)
    ref, refabs = orc.conv_fwd_at(deq["X"], deq["W"], yi, st, st, pd, pd)
    _check(f"fwd {wl.name} layer {layer}", _host(y), yi, ref, refabs)
    if not two:
        return

    gi = _sample(gx.shape, 65536, 12 + layer)
    ref, refabs = orc.conv_dgrad_at(deq["W"], deq["G_Y"], L.H, L.W, gi, st, st, pd, pd)
    _check(f"dgrad {wl.name} layer {layer}", _host(gx), gi, ref, refabs)

    ref, refabs = orc.conv_wgrad(deq["G_Y"], deq["X"], L.R, L.S, st, st, pd, pd)
    wi = np.arange(ref.size, dtype=np.int64)
    _check(f"wgrad {wl.name} layer {layer}", _host(gw), wi, ref.reshape(-1), refabs.reshape(-1))
