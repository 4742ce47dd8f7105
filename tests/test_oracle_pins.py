"""Pins of the oracle against things other than itself.

Each test checks a part of the oracle against what the MicroQonv paper
(arXiv:2609.28358) or the mathematics fixes: values the paper prints (Table I,
the format maxima of section III-A), closed forms, invariants, a hand-worked
example of the layout, brute force on tiny inputs, and library routines that
compute a special case (torch float8 casts, torch unfold / conv2d /
conv_transpose2d / autograd in float64).
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")
FMTS = {"e4m3": 0, "e5m2": 1, "e2m1": 2}
BLOCKS = {"A32": 0, "B32": 1, "SQ32": 2}
ORDERS = {"BA": 0, "AB": 1}


def gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- formats
def test_format_maxima_and_tables(orc):
    g = gold("mx_format_maxima.json")
    for name, fmt in FMTS.items():
        assert orc.max_finite(fmt) == g["max_finite"][name]
        assert orc.emax_elem(fmt) == g["emax_elem"][name]
        tab = orc.decode_table(fmt)
        assert int(np.isfinite(tab).sum()) == g["finite_code_count"][name]
    e2 = orc.decode_table(2)
    assert list(e2[:8]) == g["e2m1_nonnegative_values"]
    assert list(e2[8:]) == [-v for v in g["e2m1_nonnegative_values"]]
    # emax_elem is the exponent of the largest normal: max in [2^emax, 2^(emax+1))
    for fmt in FMTS.values():
        m = orc.max_finite(fmt)
        assert 2.0 ** orc.emax_elem(fmt) <= m < 2.0 ** (orc.emax_elem(fmt) + 1)


@pytest.mark.parametrize("name,tdt", [("e4m3", torch.float8_e4m3fn), ("e5m2", torch.float8_e5m2)])
def test_fp8_decode_matches_torch(orc, name, tdt):
    fmt = FMTS[name]
    ours = orc.decode_table(fmt)
    ref = torch.arange(256, dtype=torch.uint8).view(tdt).to(torch.float64).numpy()
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(ours), fin)
    assert np.array_equal(ours[fin], ref[fin])


def _brute_encode(tab_vals, nbits, v):
    """Nearest finite code by exhaustive search, ties to the even code."""
    best, bestd = None, None
    half = 1 << (nbits - 1)
    a = abs(v)
    for c in range(half):
        t = tab_vals[c]
        if not np.isfinite(t):
            continue
        d = abs(t - a)
        if bestd is None or d < bestd or (d == bestd and c % 2 == 0):
            best, bestd = c, d
    sign = 1 if np.signbit(v) else 0
    return (sign << (nbits - 1)) | best


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_encode_brute_force(orc, fmt):
    tab = orc.decode_table(fmt)
    nb = orc.fmt_bits(fmt)
    fin = tab[np.isfinite(tab)]
    pos = np.unique(fin[fin >= 0])
    mids = (pos[1:] + pos[:-1]) / 2          # exact ties
    rng = np.random.default_rng(7)
    vals = list(pos) + list(mids) + list(-mids) + [0.0, -0.0]
    vals += list(mids * (1 + 1e-9)) + list(mids * (1 - 1e-9))
    vals += list(rng.uniform(-2 * pos[-1], 2 * pos[-1], 400))
    vals += list(pos[-1] * np.array([1.01, 1.5, 3.0, 1e6]))   # saturation band
    vals += list(rng.uniform(0, pos[1] * 2, 100))             # subnormal band
    for v in vals:
        assert orc.encode(fmt, v) == _brute_encode(tab, nb, v), (fmt, v)


@pytest.mark.parametrize("name,tdt", [("e4m3", torch.float8_e4m3fn), ("e5m2", torch.float8_e5m2)])
def test_encode_matches_torch_cast(orc, name, tdt):
    """Within range, RNE to FP8 is the torch fp32->float8 cast; beyond it the
    oracle saturates, which is the cast of the value clamped to +-max."""
    fmt = FMTS[name]
    m = orc.max_finite(fmt)
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.uniform(-1, 1, 3000) * m * 1.3,
        np.exp2(rng.uniform(-24, 17, 3000)) * np.where(rng.random(3000) < .5, -1, 1),
        orc.decode_table(fmt)[np.isfinite(orc.decode_table(fmt))],
    ]).astype(np.float32)
    ref = torch.from_numpy(np.clip(x, -m, m)).to(tdt).view(torch.uint8).numpy()
    ours = np.array([orc.encode(fmt, float(v)) for v in x], dtype=np.uint8)
    assert np.array_equal(ours, ref)


def test_scale_rule_examples_and_top_binade(orc):
    # E4M3: amax 448 -> e = 8 - 8 = 0; amax 1 -> e = -8; E2M1 amax 6 -> e = 0
    assert orc.scale_code(0, 448.0) == 127
    assert orc.scale_code(0, 1.0) == 119
    assert orc.scale_code(2, 6.0) == 127
    assert orc.scale_code(1, 57344.0) == 127
    assert orc.scale_code(0, 0.0) == 0
    assert orc.scale_code(0, 1e-45) == 0           # clamped at 2^-127
    assert orc.scale_code(2, 3.0e38) == 127 + 127 - 2
    rng = np.random.default_rng(3)
    for fmt in (0, 1, 2):
        for amax in np.exp2(rng.uniform(-100, 100, 500)):
            e = orc.scale_code(fmt, amax) - 127
            if e in (-127, 127):
                continue
            # the scaled block maximum lands in the element format's top binade
            scaled = amax * 2.0 ** (-e)
            assert 2.0 ** orc.emax_elem(fmt) <= scaled < 2.0 ** (orc.emax_elem(fmt) + 1)


# ---------------------------------------------------------------- layout
def test_layout_hand_worked_example(orc):
    g = gold("layout_example.json")
    x = np.zeros(g["shape"], dtype=np.float32)
    for n, c, h, w, v in g["x_nonzero"]:
        x[n, c, h, w] = v
    for case in g["cases"]:
        codes, scales = orc.quantize(x, FMTS[case["fmt"]], BLOCKS[case["block"]], ORDERS[case["order"]])
        assert codes.size == case["codes_len"]
        exp = np.zeros(case["codes_len"], dtype=np.uint8)
        for k, v in case["codes_nonzero"].items():
            exp[int(k)] = v
        assert np.array_equal(codes, exp), case["why"]
        if "scales" in case:
            assert list(scales) == case["scales"]
        else:
            exp_s = np.zeros(case["scales_len"], dtype=np.uint8)
            for k, v in case["scales_nonzero"].items():
                exp_s[int(k)] = v
            assert np.array_equal(scales, exp_s)


def test_block_modes_hand_worked_example(orc):
    """B32 and SQ32 (and A32) on tensors with more than 32 elements along both
    blocked axes and a short block of 16, both code orders, E4M3 / E5M2 /
    E2M1: every code and scale byte worked out by hand (golden file)."""
    g = gold("layout_blocks_example.json")
    tensors = {}
    for name, t in g["tensors"].items():
        x = np.zeros(t["shape"], dtype=np.float32)
        for b, a, v in t["x_nonzero"]:
            x[b, a, 0, 0] = v
        tensors[name] = x
    for case in g["cases"]:
        x = tensors[case["tensor"]]
        codes, scales = orc.quantize(x, FMTS[case["fmt"]], BLOCKS[case["block"]], ORDERS[case["order"]])
        assert codes.size == case["codes_len"], case["why"]
        exp = np.zeros(case["codes_len"], dtype=np.uint8)
        for k, v in case["codes_nonzero"].items():
            exp[int(k)] = v
        assert np.array_equal(codes, exp), case["why"]
        if "scales" in case:
            assert list(scales) == case["scales"], case["why"]
        else:
            exp_s = np.zeros(case["scales_len"], dtype=np.uint8)
            for k, v in case["scales_nonzero"].items():
                exp_s[int(k)] = v
            assert np.array_equal(scales, exp_s), case["why"]


def _numpy_blocks_reference(x, fmt, block, order):
    """Codes and scales of the block modes built another way than the oracle:
    blocks are numpy reshapes of the zero-padded tensor, the exponent comes
    from np.frexp of each block's maximum, the codes from torch's saturating
    float8 cast of x / 2^e, and the layout from transposes (no index formula).
    Section IV-B directions: A32 blocks run along d1, B32 along d0, SQ32 are
    32 x 32 squares over (d0, d1)."""
    tdt = {0: torch.float8_e4m3fn, 1: torch.float8_e5m2}[fmt]
    emax = {0: 8, 1: 15}[fmt]
    vmax = {0: 448.0, 1: 57344.0}[fmt]
    B, A, H, W = x.shape
    Bq, Aq = -(-B // 32) * 32, -(-A // 32) * 32
    xp = np.zeros((Bq, Aq, H, W), dtype=np.float64)
    xp[:B, :A] = x
    if block == 2:
        amax = np.abs(xp.reshape(Bq // 32, 32, Aq // 32, 32, H, W)).max(axis=(1, 3))   # [bb][ab][h][w]
        per_elem = lambda e: np.repeat(np.repeat(e, 32, axis=0), 32, axis=1)
    elif block == 1:
        amax = np.abs(xp.reshape(Bq // 32, 32, Aq, H, W)).max(axis=1)                  # [bb][a][h][w]
        per_elem = lambda e: np.repeat(e, 32, axis=0)
    else:
        amax = np.abs(xp.reshape(Bq, Aq // 32, 32, H, W)).max(axis=2)                  # [b][ab][h][w]
        per_elem = lambda e: np.repeat(e, 32, axis=1)
    _, ex = np.frexp(amax)                                  # amax = f * 2^ex, f in [0.5, 1)
    e = np.clip(ex - 1 - emax, -127, 127)
    sc = np.where(amax == 0, 0, e + 127).astype(np.uint8)
    ee = per_elem(np.where(amax == 0, -127, e))[:B, :A]
    v = np.clip(x.astype(np.float64) * np.exp2(-ee), -vmax, vmax).astype(np.float32)
    codes8 = torch.from_numpy(v).to(tdt).view(torch.uint8).numpy()                   # [B][A][H][W]
    row = 16
    if order == 0:
        Ap = -(-A // row) * row
        lay = np.zeros((H, W, B, Ap), dtype=np.uint8)
        lay[..., :A] = codes8.transpose(2, 3, 0, 1)
    else:
        Bp = -(-B // row) * row
        lay = np.zeros((H, W, A, Bp), dtype=np.uint8)
        lay[..., :B] = codes8.transpose(2, 3, 1, 0)
    # scales over the layout's extents (the padded innermost extent is at most
    # the 32-padded one, so slicing keeps exactly the blocks the layout has)
    if block == 2:
        s = sc.transpose(2, 3, 0, 1)                                               # [h][w][bb][ab]
    elif block == 1:
        Ap = -(-A // row) * row if order == 0 else A
        s = sc[:, :Ap].transpose(2, 3, 0, 1)                                       # [h][w][bb][a]
    else:
        Bp = -(-B // row) * row if order == 1 else B
        s = sc[:Bp].transpose(2, 3, 0, 1)                                          # [h][w][b][ab]
    return lay.reshape(-1), s.reshape(-1)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("block", [0, 1, 2])
@pytest.mark.parametrize("order", [0, 1])
@pytest.mark.parametrize("shape", [(40, 72, 2, 3), (16, 40, 3, 2), (70, 33, 1, 2)])
def test_block_modes_match_numpy_blocks_and_torch_cast(orc, fmt, block, order, shape):
    x = synth.random_tensor(shape, seed=31 + 7 * block + order, dist="student_t")
    # give each 32 x 32 square its own magnitude so that mixing blocks changes scales
    B, A = shape[0], shape[1]
    for bb in range(-(-B // 32)):
        for ab in range(-(-A // 32)):
            x[32 * bb:32 * bb + 32, 32 * ab:32 * ab + 32] *= np.float32(2.0 ** (3 * bb - 5 * ab))
    codes, scales = orc.quantize(x, fmt, block, order)
    ref_codes, ref_scales = _numpy_blocks_reference(x, fmt, block, order)
    assert np.array_equal(scales, ref_scales)
    assert np.array_equal(codes, ref_codes)


def _quant_error_bound(orc, fmt, x, xq, e_of_elem):
    """|x - dequant| <= half an ulp of the top binade at the block scale, or the
    saturation gap for elements beyond the largest finite value."""
    mb = {0: 3, 1: 2, 2: 1}[fmt]
    em = orc.emax_elem(fmt)
    half_ulp = np.exp2(e_of_elem + em - mb - 1)
    sat_gap = np.exp2(e_of_elem) * (2.0 ** (em + 1) - orc.max_finite(fmt))
    return np.abs(x - xq) <= np.maximum(half_ulp, sat_gap) * (1 + 1e-12)


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("block", [0, 1, 2])
@pytest.mark.parametrize("order", [0, 1])
def test_roundtrip_error_bound_and_idempotence(orc, fmt, block, order):
    x = synth.random_tensor((37, 45, 3, 2), seed=100 + 10 * fmt + 3 * block + order, dist="uniform_exp")
    codes, scales = orc.quantize(x, fmt, block, order)
    xq = orc.dequantize(codes, scales, x.shape, fmt, block, order)
    # per-element scale exponent, recovered from the block layout definition
    Ap, Bp = orc.padded_extents(fmt, order, 45, 37)
    nba, nbb = -(-Ap // 32), -(-Bp // 32)
    e = np.empty(x.shape)
    for b, a, h, w in itertools.product(range(37), range(45), range(3), range(2)):
        pix = h * 2 + w
        if block == 0:
            si = (pix * Bp + b) * nba + a // 32
        elif block == 1:
            si = (pix * nbb + b // 32) * Ap + a
        else:
            si = (pix * nbb + b // 32) * nba + a // 32
        e[b, a, h, w] = int(scales[si]) - 127
    assert _quant_error_bound(orc, fmt, x.astype(np.float64), xq, e).all()
    # re-quantizing the dequantized tensor reproduces codes and scales exactly
    codes2, scales2 = orc.quantize(xq.astype(np.float32), fmt, block, order)
    assert np.array_equal(codes, codes2) and np.array_equal(scales, scales2)


def test_strided_source_equals_contiguous(orc):
    x = synth.random_tensor((40, 70, 5, 6), seed=5)
    xt = np.ascontiguousarray(x.transpose(2, 3, 0, 1)).transpose(2, 3, 0, 1)  # non-NCHW strides
    for block in (0, 1, 2):
        a = orc.quantize(x, 0, block, 0)
        b = orc.quantize(xt, 0, block, 0)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_codes_match_torch_cast_at_block_scale(orc):
    """A32 along C with E4M3: the codes are the saturating FP8 cast of x / 2^e
    where 2^e is the block scale (torch computes the cast)."""
    x = synth.random_tensor((3, 64, 4, 5), seed=21, dist="student_t")
    codes, scales = orc.quantize(x, 0, 0, 0)
    cod = codes.reshape(4, 5, 3, 64)
    sc = scales.reshape(4, 5, 3, 2).astype(np.int32) - 127
    xs = x.transpose(2, 3, 0, 1).astype(np.float64) * np.exp2(-np.repeat(sc, 32, axis=3))
    ref = torch.from_numpy(np.clip(xs, -448, 448).astype(np.float32)).to(torch.float8_e4m3fn)
    assert np.array_equal(cod, ref.view(torch.uint8).numpy())


# ---------------------------------------------------------------- im2col
@pytest.mark.parametrize("R,S,st,pad", [(3, 3, 1, 1), (3, 3, 2, 1), (1, 1, 1, 0), (2, 3, 2, 0), (3, 3, 1, 0)])
def test_im2col_fp32_matches_unfold(orc, R, S, st, pad):
    x = synth.random_tensor((2, 5, 9, 7), seed=31)
    xe = orc.im2col_fp32(x, R, S, st, st, pad, pad)
    N, C, H, W = x.shape
    P, Q = orc.out_hw(H, W, R, S, st, st, pad, pad)
    u = F.unfold(torch.from_numpy(x), (R, S), padding=pad, stride=st).numpy()   # [N][C*R*S][P*Q], (c, r, s)
    u = u.reshape(N, C, R, S, P, Q).transpose(0, 2, 3, 1, 4, 5).reshape(N, R * S * C, P, Q)
    assert np.array_equal(xe, u)


@pytest.mark.parametrize("block", [0, 1, 2])
@pytest.mark.parametrize("order", [0, 1])
@pytest.mark.parametrize("geom", [(3, 3, 1, 1), (3, 3, 2, 1), (1, 1, 1, 0), (3, 3, 2, 0), (2, 2, 1, 1)])
@pytest.mark.parametrize("fmt", [0, 2])
def test_invariant_quantize_then_im2col(orc, block, order, geom, fmt):
    """Quantize-then-channel-batch-first-im2col is bit-identical to
    im2col-then-quantize when the blocked axes are multiples of 32 (paper,
    sections IV-A and IV-C: the reordered X is quantized before its expansion)."""
    R, S, st, pad = geom
    N = 40 if block != 0 else 3      # short B-blocks are the same on both sides
    x = synth.random_tensor((N, 64, 7, 6), seed=41 + block, dist="student_t")
    codes, scales = orc.quantize(x, fmt, block, order)
    c1, s1 = orc.im2col_cbf(codes, scales, N, 64, 7, 6, R, S, st, st, pad, pad, fmt, block, order)
    xe = orc.im2col_fp32(x, R, S, st, st, pad, pad)
    c2, s2 = orc.quantize(xe, fmt, block, order)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)


# ---------------------------------------------------------------- convolutions
def _tiny(seed, shape):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("R,S,st,pad", [(3, 3, 1, 1), (3, 3, 2, 1), (1, 1, 1, 0), (2, 3, 2, 1), (3, 2, 1, 0)])
def test_convs_match_torch_float64(orc, R, S, st, pad):
    N, C, H, W, K = 2, 3, 7, 6, 4
    x, w = _tiny(1, (N, C, H, W)), _tiny(2, (K, C, R, S))
    y, ya = orc.conv_fwd(x, w, st, st, pad, pad)
    xt = torch.from_numpy(x).requires_grad_(True)
    wt = torch.from_numpy(w).requires_grad_(True)
    yt = F.conv2d(xt, wt, stride=st, padding=pad)
    assert np.allclose(y, yt.detach().numpy(), rtol=1e-12, atol=1e-12)
    # sum |a*b| is the convolution of |x| with |w|
    ya_t = F.conv2d(torch.from_numpy(np.abs(x)), torch.from_numpy(np.abs(w)), stride=st, padding=pad)
    assert np.allclose(ya, ya_t.numpy(), rtol=1e-12, atol=1e-12)
    gy = _tiny(3, y.shape)
    yt.backward(torch.from_numpy(gy))
    gx, gxa = orc.conv_dgrad(w, gy, H, W, st, st, pad, pad)
    gw, gwa = orc.conv_wgrad(gy, x, R, S, st, st, pad, pad)
    assert np.allclose(gx, xt.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(gw, wt.grad.numpy(), rtol=1e-12, atol=1e-12)
    # G_X through the transposed convolution routine as well
    op = (H + 2 * pad - R) % st, (W + 2 * pad - S) % st
    gx2 = F.conv_transpose2d(torch.from_numpy(gy), torch.from_numpy(w), stride=st, padding=pad, output_padding=op)
    assert np.allclose(gx, gx2.numpy(), rtol=1e-12, atol=1e-12)
    assert (gxa >= np.abs(gx) - 1e-12).all() and (gwa >= np.abs(gw) - 1e-12).all()


def test_conv_brute_force_tiny(orc):
    """Eq. 1-3 by direct summation in Python on a tiny problem."""
    N, C, H, W, K, R, S, st, pad = 1, 2, 4, 3, 2, 3, 2, 2, 1
    x, w = _tiny(4, (N, C, H, W)), _tiny(5, (K, C, R, S))
    P, Q = orc.out_hw(H, W, R, S, st, st, pad, pad)
    y = np.zeros((N, K, P, Q))
    for n, k, p, q, c, r, s in itertools.product(range(N), range(K), range(P), range(Q), range(C), range(R), range(S)):
        h, ww = p * st + r - pad, q * st + s - pad
        if 0 <= h < H and 0 <= ww < W:
            y[n, k, p, q] += w[k, c, r, s] * x[n, c, h, ww]
    assert np.allclose(orc.conv_fwd(x, w, st, st, pad, pad)[0], y, rtol=1e-13, atol=1e-13)
    gy = _tiny(6, (N, K, P, Q))
    gx = np.zeros_like(x)
    gw = np.zeros_like(w)
    for n, k, p, q, c, r, s in itertools.product(range(N), range(K), range(P), range(Q), range(C), range(R), range(S)):
        h, ww = p * st + r - pad, q * st + s - pad
        if 0 <= h < H and 0 <= ww < W:
            gx[n, c, h, ww] += w[k, c, r, s] * gy[n, k, p, q]
            gw[k, c, r, s] += gy[n, k, p, q] * x[n, c, h, ww]
    assert np.allclose(orc.conv_dgrad(w, gy, H, W, st, st, pad, pad)[0], gx, rtol=1e-13, atol=1e-13)
    assert np.allclose(orc.conv_wgrad(gy, x, R, S, st, st, pad, pad)[0], gw, rtol=1e-13, atol=1e-13)


def test_sampled_outputs_equal_full(orc):
    N, C, H, W, K, R, S, st, pad = 2, 3, 6, 5, 4, 3, 3, 2, 1
    x, w = _tiny(7, (N, C, H, W)), _tiny(8, (K, C, R, S))
    y, ya = orc.conv_fwd(x, w, st, st, pad, pad)
    gy = _tiny(9, y.shape)
    gx, gxa = orc.conv_dgrad(w, gy, H, W, st, st, pad, pad)
    gw, gwa = orc.conv_wgrad(gy, x, R, S, st, st, pad, pad)
    for full, fa, fn, args in [(y, ya, orc.conv_fwd_at, (x, w)), (gx, gxa, orc.conv_dgrad_at, (w, gy, H, W)),
                               (gw, gwa, orc.conv_wgrad_at, (gy, x, R, S))]:
        idx = np.arange(full.size)
        v, va = fn(*args, idx, st, st, pad, pad)
        assert np.array_equal(v, full.ravel()) and np.array_equal(va, fa.ravel())


def test_block_scaled_dot_product_identity(orc):
    """Eq. 7: when both operands are blocked along the reduction, the dot
    product is the sum over blocks of (scale_r * scale_t * integer-grid dot of
    the element values); it equals the dot product of the dequantized tensors."""
    x = synth.random_tensor((1, 96, 1, 1), seed=51, dist="student_t")
    w = synth.random_tensor((1, 96, 1, 1), seed=52, dist="student_t")
    cx, sx = orc.quantize(x, 0, 0, 0)
    cw, sw = orc.quantize(w, 1, 0, 0)
    tx, tw = orc.decode_table(0), orc.decode_table(1)
    blocks = 0.0
    for j in range(3):
        ex, ew = int(sx[j]) - 127, int(sw[j]) - 127
        inner = sum(tx[cx[32 * j + i]] * tw[cw[32 * j + i]] for i in range(32))
        blocks += 2.0 ** (ex + ew) * inner
    xd = orc.dequantize(cx, sx, x.shape, 0, 0, 0)
    wd = orc.dequantize(cw, sw, w.shape, 1, 0, 0)
    y, _ = orc.conv_fwd(xd, wd)
    assert y.item() == pytest.approx(blocks, rel=1e-14, abs=1e-300)


# ---------------------------------------------------------------- Table I
def test_table1_quantization_counts(orc):
    g = gold("table1_counts.json")
    t = g["per_element_quantization"]
    N, C, H, W = 2, 3, 12, 11
    counts, entries = orc.im2col_counts(N, C, H, W, 3, 3, 1, 1, 1, 1)
    interior = counts[:, :, 1:-1, 1:-1]
    # an interior element appears once per kernel tap: quantizing the expanded
    # tensor once (Cuyckens et al.) quantizes it 9 times, DaCapo twice that
    assert (interior == t["Cuyckens"]["A"]).all()
    assert (2 * interior == t["DaCapo"]["A"]).all()
    # X' has Kh*Kw*Hout*Wout/(Hin*Win) entries per element of X
    P, Q = orc.out_hw(H, W, 3, 3, 1, 1, 1, 1)
    assert entries == 9 * P * Q * N * C and entries / (N * C * H * W) == t["Cuyckens"]["A"]
    assert counts.max() == 9 and counts.min() == 4     # corners see 4 windows
    # W and G_Y are GEMM operands as they are: once per direction (DaCapo) or once
    assert t["MicroQonv"] == {"A": 1, "W": 1, "G": 1}
    # stride 2: the expansion is Kh*Kw*Hout*Wout/(Hin*Win), about 9/4
    counts2, entries2 = orc.im2col_counts(1, 1, 16, 16, 3, 3, 2, 2, 1, 1)
    assert entries2 == 9 * 8 * 8


def test_table1_memory_movement(orc):
    """Backward memory movement: FP32 activations vs MX (4-bit elements,
    one 8-bit scale per 32) is 32/4.25 = 7.53; storing the quantized im2col
    expansion instead of the quantized X costs the 9x expansion (3x3, s1, p1)."""
    g = gold("table1_counts.json")["backward_memory_movement_vs_MicroQonv"]
    N, C, H, W = 32, 64, 10, 10
    fp32 = 4 * N * C * H * W
    # one E8M0 scale per 32-element line (A32): 4 + 8/32 bits per element
    mx4 = orc.codes_bytes(2, 0, N, C, H, W) + orc.scales_bytes(2, 0, 0, N, C, H, W)
    assert round(fp32 / mx4, 2) == g["DaCapo"]["A"]
    # a 32x32 square sharing one scale stores 4 + 8/1024 bits per element
    sq = orc.codes_bytes(2, 0, N, C, H, W) + orc.scales_bytes(2, 2, 0, N, C, H, W)
    assert abs(fp32 / sq - 32 / (4 + 8 / 1024)) < 1e-12
    x = synth.random_tensor((N, C, H, W), seed=61)
    codes, scales = orc.quantize(x, 2, 2, 0)
    ce, se = orc.im2col_cbf(codes, scales, N, C, H, W, 3, 3, 1, 1, 1, 1, 2, 2, 0)
    assert (ce.size + se.size) / (codes.size + scales.size) == g["Cuyckens"]["A"]
    # MXFP8 with B=32: 32 / 8.25 = 3.879 (the paper's "closer to x3.93" is the B=64 figure 32/8.125)
    mx8 = orc.codes_bytes(0, 0, N, C, H, W) + orc.scales_bytes(0, 0, 0, N, C, H, W)
    assert abs(fp32 / mx8 - 32 / 8.25) < 1e-12


# ---------------------------------------------------------------- activation
def test_activation_matches_torch(orc):
    """The activations of the quantized forward output: torch's relu and silu
    in float64, and the closed forms silu(0) = 0, silu(x) -> x and -> 0."""
    y = synth.random_tensor((3, 5, 7, 11), seed=8, dist="student_t").astype(np.float64) * 4
    t = torch.from_numpy(y)
    assert np.array_equal(orc.activation(y, orc.ACT_NONE), y)
    assert np.array_equal(orc.activation(y, orc.ACT_RELU), F.relu(t).numpy())
    assert np.allclose(orc.activation(y, orc.ACT_SILU), F.silu(t).numpy(), rtol=1e-15, atol=1e-300)
    big = np.array([0.0, 60.0, -60.0])
    s = orc.activation(big, orc.ACT_SILU)
    assert s[0] == 0.0 and abs(s[1] - 60.0) < 1e-20 and abs(s[2]) < 1e-20
