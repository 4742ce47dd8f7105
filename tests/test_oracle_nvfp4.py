"""Pins of the oracle's NVFP4 quantization (MicroQonv paper, section III-A,
Eq. 4-6: per-tensor FP32 scale T = max|X| / (448 * 6), an E4M3 scale per
block of 16, E2M1 elements), evaluated step by step in fp32.

- A hand-worked example (golden file), values away from rounding ties.
- The tensor maximum lands on the top of both formats: its block scale is
  448 (0x7E) and its code is +-6.
- Exact invariance under power-of-two scaling: every step is a product or
  quotient, so scaling X by 2^k scales T by 2^k and leaves codes and block
  scales unchanged.
- The block scale is torch's float8_e4m3fn cast of max|X_i| / (T * 6).
- The dequantized tensor is within half an E2M1 step of X at the block's
  scale (or the saturation gap).
"""
import json
import os

import numpy as np
import pytest
import torch

import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")
E2M1_VALS = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)


def test_nvfp4_hand_worked_example(orc):
    g = json.load(open(os.path.join(GOLD, "nvfp4_example.json")))
    x = np.zeros(g["shape"], dtype=np.float32)
    for a, v in enumerate(g["x_nonzero_along_a"]):
        x[0, a, 0, 0] = v
    codes, scales, t = orc.quantize_nvfp4(x, orc.NV_A16, 0)
    assert list(codes) == g["codes"], g["why"]
    assert list(scales) == g["scales"], g["why"]
    assert t == np.float32(g["tscale_times_2688"]) / np.float32(2688.0)


@pytest.mark.parametrize("block", [0, 1, 2])
@pytest.mark.parametrize("order", [0, 1])
def test_nvfp4_tensor_max_and_power_of_two_invariance(orc, block, order):
    x = synth.random_tensor((20, 40, 3, 2), seed=60 + block, dist="student_t")
    codes, scales, t = orc.quantize_nvfp4(x, block, order)
    # the element of largest magnitude: code +-6, its block scale 448
    b, a, h, w = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    d = orc.dequantize_nvfp4(codes, scales, t, x.shape, block, order)
    assert abs(d[b, a, h, w]) == pytest.approx(6 * 448 * t, rel=1e-12)
    assert 0x7E in set(scales.tolist())
    for k in (-9, -1, 3, 14):
        c2, s2, t2 = orc.quantize_nvfp4((x * np.float32(2.0 ** k)).astype(np.float32), block, order)
        assert np.array_equal(c2, codes) and np.array_equal(s2, scales)
        assert t2 == np.float32(t * 2.0 ** k)


def test_nvfp4_block_scales_are_torch_e4m3_casts(orc):
    """A16 blocks, order BA, scales [pix][B][A/16]: the byte equals torch's
    RNE float8_e4m3fn cast of max|X_i| / (T * 6) computed in float32."""
    B, A, H, W = 7, 48, 2, 3
    x = synth.random_tensor((B, A, H, W), seed=70, dist="student_t")
    x[:, :16] *= np.float32(1e-3)                       # small blocks: scales far below 448
    _, scales, t = orc.quantize_nvfp4(x, orc.NV_A16, 0)
    t32 = np.float32(np.abs(x).max()) / np.float32(2688.0)
    assert t == t32
    bmax = np.abs(x).reshape(B, A // 16, 16, H, W).max(axis=2)          # [b][block][h][w]
    q = (bmax.astype(np.float32) / (t32 * np.float32(6.0))).astype(np.float32)
    ref = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # the FP4 row is padded to 64 codes: a fourth block of padding with scale 0
    lay = scales.reshape(H, W, B, 4)
    assert (lay[..., 3] == 0).all()
    ours = lay[..., :3].transpose(2, 3, 0, 1)
    assert np.array_equal(ours, ref)


@pytest.mark.parametrize("block", [0, 1, 2])
def test_nvfp4_error_bound(orc, block):
    x = synth.random_tensor((33, 70, 2, 2), seed=80 + block, dist="student_t")
    codes, scales, t = orc.quantize_nvfp4(x, block, 0)
    d = orc.dequantize_nvfp4(codes, scales, t, x.shape, block, 0)
    # the block scale B * T of every element: dequantize a tensor of ones'
    # codes is not available, so recover it from the nonzero dequantized
    # values' own codes: |d| / value(code); elements with a zero code are
    # bounded by half the first step of any scale up to the tensor's
    ones = orc.dequantize_nvfp4(np.full_like(codes, 0x22), scales, t, x.shape, block, 0)   # code 2 = 1.0
    s = np.abs(ones)                                       # B * T per element
    v = np.abs(x.astype(np.float64)) / np.where(s > 0, s, 1)
    half = np.where(v < 2, 0.25, np.where(v < 4, 0.5, 1.0))
    bound = s * np.maximum(half, v - 6) * (1 + 1e-6) + 1e-30
    assert (np.abs(d - x) <= bound).all()
