"""The algebra the sub-pixel input gradient relies on, checked on the CPU
against the oracle's plain Eq. 2 (MicroQonv paper, section II-C3):

For a convolution with strides (sh, sw), the input pixel (sh*i + ah, sw*j + aw)
receives G_Y[i + dh][j + dw] through kernel tap r = ah + pad_h - sh*dh,
s = aw + pad_w - sw*dw wherever that tap exists.  Over all phases (ah, aw) the
offsets (dh, dw) span a small window, so G_X is one stride-1 correlation of
G_Y with window weights Ws[(dh, dw)][(ah, aw, c)][k] (zero where no tap links
an offset to a phase), stored depth-to-space.  This file rebuilds G_X that
way in numpy, with the window bounds and the weight rearrangement written
out independently of the library, and compares it with the oracle."""
import itertools

import numpy as np
import pytest

import synth


def _window(stride, R, pad):
    d = [(a + pad - r) // stride for a in range(stride) for r in range(R) if (a + pad - r) % stride == 0]
    return min(d), max(d) - min(d) + 1


def _subpixel_dgrad(w, g, H, W, sh, sw, ph, pw):
    K, C, R, S = w.shape
    N, _, P, Q = g.shape
    dh0, Rs = _window(sh, R, ph)
    dw0, Ss = _window(sw, S, pw)
    Cs = sh * sw * C
    ws = np.zeros((Rs * Ss, Cs, K))
    for t, cs in itertools.product(range(Rs * Ss), range(Cs)):
        phase, c = divmod(cs, C)
        ah, aw = divmod(phase, sw)
        r, s = ah + ph - sh * (dh0 + t // Ss), aw + pw - sw * (dw0 + t % Ss)
        if 0 <= r < R and 0 <= s < S:
            ws[t, cs] = w[:, c, r, s]
    gx = np.zeros((N, C, H, W))
    for i, j in itertools.product(range(H // sh), range(W // sw)):
        acc = np.zeros((N, Cs))
        for t in range(Rs * Ss):
            p, q = i + dh0 + t // Ss, j + dw0 + t % Ss
            if 0 <= p < P and 0 <= q < Q:
                acc += g[:, :, p, q] @ ws[t].T
        for cs in range(Cs):
            phase, c = divmod(cs, C)
            ah, aw = divmod(phase, sw)
            gx[:, c, sh * i + ah, sw * j + aw] = acc[:, cs]
    return gx, (Rs, Ss)


# (N, C, H, W, K, R, S, stride, pad, expected window)
CASES = [
    (2, 3, 8, 8, 4, 3, 3, 2, 1, (2, 2)),     # 3x3, stride 2, pad 1: the YOLO layers
    (1, 2, 10, 8, 3, 1, 1, 2, 0, (1, 1)),    # 1x1, stride 2: odd rows and columns get nothing
    (1, 2, 12, 10, 3, 5, 5, 2, 2, (3, 3)),   # 5x5: offsets -1 .. 1
    (1, 2, 8, 8, 3, 4, 4, 2, 1, (3, 3)),     # 4x4 (a transposed-conv upsampler's kernel)
    (1, 2, 8, 8, 3, 3, 3, 2, 0, (2, 2)),     # no padding: offsets -1 .. 0
    (1, 2, 9, 12, 3, 3, 3, 3, 1, (2, 2)),    # stride 3 (9 phases): offsets 0 .. 1, one tap per phase
]


@pytest.mark.parametrize("case", CASES)
def test_subpixel_gemm_equals_eq2(orc, case):
    N, C, H, W, K, R, S, st, pad, window = case
    if H % st or W % st:
        pytest.skip("the sub-pixel plan needs the phases to tile the input")
    P, Q = orc.out_hw(H, W, R, S, st, st, pad, pad)
    w = synth.random_tensor((K, C, R, S), seed=40 + R, scale=0.5)
    g = synth.random_tensor((N, K, P, Q), seed=41 + R)
    got, win = _subpixel_dgrad(w.astype(np.float64), g.astype(np.float64), H, W, st, st, pad, pad)
    assert win == window
    want, _ = orc.conv_dgrad(w, g, H, W, st, st, pad, pad)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
