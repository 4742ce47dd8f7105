"""Pins of the oracle's stochastic rounding (MicroQonv paper, section III-A,
Eq. 6 and the text after it: gradients are rounded stochastically) and of
its random bits.

- Philox4x64-10 against numpy's independent implementation of the same
  published generator (numpy.random.Philox; its first block for a counter c
  is the block of c + 1).
- The rounding rule against closed forms: representable values never move,
  every result is one of the two neighbours, r = 0 gives the upper
  neighbour and r = 2^16 - 1 the lower one (unless f > 1 - 2^-16), and the
  average over all 2^16 random values equals the value itself to within
  ulp * 2^-16 (the rule's only bias).
- Whole tensors: the block scales are those of round-to-nearest, every code
  is one of the two neighbours of the exact scaled value, and the mean over
  many seeds converges to the input (unbiasedness).
"""
import numpy as np
import pytest

import synth

U64 = (1 << 64) - 1


def numpy_philox_block(ctr, key):
    """numpy's Philox4x64-10 block for counter `ctr`: numpy increments its
    256-bit counter (with carry) before each block, so start one below."""
    c = [int(v) for v in ctr]
    i = 0
    while i < 4:
        c[i] = (c[i] - 1) & U64
        if c[i] != U64:
            break
        i += 1
    return np.random.Philox(counter=np.array(c, dtype=np.uint64), key=np.array(key, dtype=np.uint64)).random_raw(4)


@pytest.mark.parametrize("ctr,key", [((0, 0, 0, 0), (0, 0)), ((1, 0, 0, 0), (0, 0)), ((6, 7, 0, 0), (123, 0)),
                                     ((2 ** 40 + 3, 99, 5, 1), (2 ** 63 + 11, 77)),
                                     ((U64, 0, 0, 0), (1, 2))])
def test_philox4x64_matches_numpy(orc, ctr, key):
    ours = orc.philox4x64(np.array(ctr, dtype=np.uint64), np.array(key, dtype=np.uint64))
    ref = numpy_philox_block(ctr, key)
    assert [int(v) for v in ours] == [int(v) for v in ref]


def test_sr_bits_are_philox_lanes(orc):
    """Element (pix, b, a) of a tensor with extents (B, A) takes 16-bit lane
    j = i % 16 of block i / 16, i = (pix*B + b)*A16 + a, A16 = A rounded to 16."""
    seed, offset, B, A = 1234567, 42, 5, 37
    A16 = 48
    rng = np.random.default_rng(0)
    for _ in range(40):
        pix, b, a = int(rng.integers(0, 9)), int(rng.integers(0, B)), int(rng.integers(0, A))
        i = (pix * B + b) * A16 + a
        blk = numpy_philox_block((i // 16, offset, 0, 0), (seed, 0))
        j = i % 16
        want = (int(blk[j // 4]) >> (16 * (j % 4))) & 0xFFFF
        assert orc.sr_bits(seed, offset, B, A, pix, b, a) == want


def _neighbours(tab, a):
    """Largest finite magnitude <= a and the next one (brute force)."""
    fin = np.unique(tab[np.isfinite(tab) & (tab >= 0)])
    lo = fin[fin <= a].max()
    hi = fin[fin > a].min() if (fin > a).any() else lo
    return lo, hi


@pytest.mark.parametrize("fmt", [0, 1, 2])
def test_encode_sr_closed_forms(orc, fmt):
    tab = orc.decode_table(fmt)
    nb = orc.fmt_bits(fmt)
    vmax = orc.max_finite(fmt)
    rng = np.random.default_rng(7 + fmt)
    # representable values: unchanged for any r (RNE gives the same code)
    for v in tab[np.isfinite(tab)][::3]:
        for r in (0, 1, 32768, 65535):
            assert orc.encode_sr(fmt, v, r) == orc.encode(fmt, v)
    # beyond the largest finite value: saturation
    for v in (vmax * 1.01, vmax * 7.0, -vmax * 1.5):
        assert orc.encode_sr(fmt, v, 0) == orc.encode(fmt, v)
    vals = rng.uniform(0, vmax, size=300) * np.where(rng.random(300) < 0.5, -1, 1)
    vals = np.concatenate([vals, rng.uniform(0, tab[np.isfinite(tab) & (tab > 0)].min() * 3, size=50)])
    for v in vals:
        lo, hi = _neighbours(tab, abs(v))
        sgn = -1.0 if v < 0 else 1.0
        dec = lambda c: tab[c]
        up = orc.encode_sr(fmt, v, 0)
        dn = orc.encode_sr(fmt, v, 65535)
        if lo == abs(v):
            continue
        assert dec(up) == sgn * hi, (v, dec(up), hi)
        f = (abs(v) - lo) / (hi - lo)
        assert dec(dn) == sgn * (hi if f * 65536 > 65535 else lo)
        # mean over every r: lo + (hi - lo) * ceil(f * 2^16) / 2^16 (here
        # f * 2^16 is never an integer by construction of the values)
        n_up = int(np.ceil(f * 65536))
        r_all = np.arange(65536)
        codes = np.array([orc.encode_sr(fmt, v, int(r)) for r in r_all[::97]])
        got = tab[codes]
        assert set(np.abs(got)) <= {lo, hi}
        assert ((np.abs(got) == hi) == (r_all[::97] < f * 65536)).all()
        mean = lo + (hi - lo) * n_up / 65536
        assert abs(mean - abs(v)) <= (hi - lo) / 65536
        assert (code_bits := up >> (nb - 1)) == (1 if v < 0 else 0), code_bits


@pytest.mark.parametrize("fmt", [0, 1, 2])
@pytest.mark.parametrize("block", [0, 1, 2])
def test_quantize_sr_scales_and_neighbours(orc, fmt, block):
    x = synth.random_tensor((20, 40, 3, 2), seed=50 + fmt, dist="student_t")
    c_rn, s_rn = orc.quantize(x, fmt, block, 0)
    c_sr, s_sr = orc.quantize_sr(x, fmt, block, 0, seed=99, offset=3)
    assert np.array_equal(s_sr, s_rn)
    d_rn = orc.dequantize(c_rn, s_rn, x.shape, fmt, block, 0)
    d_sr = orc.dequantize(c_sr, s_sr, x.shape, fmt, block, 0)
    # both are neighbours of x: at most one step apart, the exact value between
    # them or at a saturated end
    tab = orc.decode_table(fmt)
    step = np.diff(np.unique(tab[np.isfinite(tab) & (tab >= 0)])).max()
    sc = np.abs(d_rn - x)
    assert (np.abs(d_sr - x) <= np.abs(d_sr - d_rn) + sc + 1e-300).all()
    # the second order holds the same decisions
    c_sr_ab, s_sr_ab = orc.quantize_sr(x, fmt, block, 1, seed=99, offset=3)
    d_ab = orc.dequantize(c_sr_ab, s_sr_ab, x.shape, fmt, block, 1)
    assert np.array_equal(d_ab, d_sr)
    # another seed or offset changes some codes; the same one repeats exactly
    assert np.array_equal(orc.quantize_sr(x, fmt, block, 0, seed=99, offset=3)[0], c_sr)
    assert not np.array_equal(orc.quantize_sr(x, fmt, block, 0, seed=99, offset=4)[0], c_sr)
    assert step > 0


@pytest.mark.parametrize("fmt", [1, 2])
def test_quantize_sr_is_unbiased(orc, fmt):
    """Mean over 400 seeds of the dequantized tensor approaches the input.
    For an element between neighbours lo < |x| / 2^e < hi with fraction f,
    the mean of n draws has standard deviation sqrt(f (1 - f) / n) (hi - lo)
    2^e and the rule's bias is below (hi - lo) 2^e / 2^16; every element is
    within 6 standard deviations plus that bias, and the signed error
    averaged over all elements is near zero."""
    B, A, H, W = 8, 64, 2, 2
    x = synth.random_tensor((B, A, H, W), seed=77, scale=1e-3)
    n = 400
    acc = np.zeros(x.shape)
    for k in range(n):
        c, s = orc.quantize_sr(x, fmt, 2, 0, seed=1000 + k, offset=0)
        acc += orc.dequantize(c, s, x.shape, fmt, 2, 0)
    mean = acc / n
    # the block exponent of every element (SQ32 scales [pix][b/32][a/32])
    _, sc = orc.quantize(x, fmt, 2, 0)
    e = (sc.reshape(H, W, 1, A // 32).astype(np.float64) - 127)
    e = np.repeat(e, 32, axis=3).transpose(2, 3, 0, 1)                 # [1][A][H][W], broadcast over b
    v = np.abs(x.astype(np.float64)) * np.exp2(-e)
    tab = orc.decode_table(fmt)
    mags = np.unique(tab[np.isfinite(tab) & (tab >= 0)])
    k = np.searchsorted(mags, v, side="right") - 1
    lo = mags[k]
    hi = mags[np.minimum(k + 1, mags.size - 1)]
    gap = (hi - lo) * np.exp2(e)
    f = np.where(hi > lo, (v - lo) / np.maximum(hi - lo, 1e-300), 0.0)
    std = np.sqrt(f * (1 - f) / n) * gap
    err = np.abs(mean - x.astype(np.float64))
    sel = v < mags[-1]                      # saturated elements have no upper neighbour
    assert (err <= 6 * std + gap / 65536 + 1e-300)[sel].all()
    rel = ((mean - x.astype(np.float64))[sel] / gap[sel]).mean()
    assert abs(rel) < 0.01
