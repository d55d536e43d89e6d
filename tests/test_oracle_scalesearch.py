"""Pins for the oracle's ScaleSearch ["Search Your Block Floating Point
Scales!", ScaleSearch: offsets f in [-2, 6] on the bit pattern of the default
scale, the least squared error kept], applied to the fp16 scales of the
int4 / int2 (asymmetric) and int8 (symmetric) codecs.  Checked against a
brute force in fp64 over every candidate, the codec without the search, a
group that sits on the default grid, and constant groups.  No GPU."""
import numpy as np
import pytest

import oracle as O

CASES = [(O.INT4_ASYM, 32, 1.0), (O.INT2_ASYM, 128, 0.9), (O.INT2_ASYM, 64, 1.0), (O.INT8_SYM, 128, 1.0),
         (O.INT8_SYM, 64, 1.0)]


def _rows(n, d, seed, heavy=False):
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((n, d)) if not heavy else rng.laplace(size=(n, d)) * (1 + 9 * (rng.random((n, d)) < 0.02))
    return y.astype(np.float32)


def _h2f(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def _sq_err64(y, codes, scale, zero):
    return float(np.sum((y.astype(np.float64) - (codes.astype(np.float64) * scale + zero)) ** 2))


def _candidate(y, fmt, bits, zero_f32):
    """codes of one group with scale bits `bits`, the codec's fp32 steps"""
    sf = np.float32(_h2f(bits))
    inv = np.float32(1.0) / sf if sf != 0 else np.float32(0.0)
    if fmt == O.INT8_SYM:
        c = np.clip(np.rint(y * inv), -127, 127)
    else:
        qmax = 15 if fmt == O.INT4_ASYM else 3
        c = np.clip(np.rint((y - zero_f32) * inv), 0, qmax)
    return c, float(sf)


@pytest.mark.parametrize("fmt,group,clip", CASES)
@pytest.mark.parametrize("heavy", [False, True])
def test_search_keeps_the_best_candidate_by_brute_force(fmt, group, clip, heavy):
    d = group if fmt != O.INT4_ASYM else 128
    y = _rows(300, d, 7 + fmt + group, heavy)
    c0, s0, z0, _, _ = O.quantize_rows(fmt, group, clip, y, search=0)
    c1, s1, z1, _, _ = O.quantize_rows(fmt, group, clip, y, search=1)
    assert np.array_equal(z0, z1)  # the zero never moves
    off = s1.astype(np.int64) - s0.astype(np.int64)
    assert np.all((off >= -2) & (off <= 6))
    g = d if fmt == O.INT8_SYM else group
    ng = d // g
    improved = 0
    for r in range(y.shape[0]):
        for k in range(ng):
            yg = y[r, k * g:(k + 1) * g]
            zf = np.float32(_h2f(z1[r, k])) if fmt != O.INT8_SYM else np.float32(0)
            # the stored codes are the codec's codes for the stored scale
            cc, sf = _candidate(yg, fmt, s1[r, k], zf)
            assert np.array_equal(cc, c1[r, k * g:(k + 1) * g]), (r, k)
            chosen = _sq_err64(yg, cc, sf, float(zf))
            errs = []
            for f in range(-2, 7):
                b = int(s0[r, k]) + f
                if 0 < b < 0x7C00:
                    cf, sff = _candidate(yg, fmt, b, zf)
                    errs.append(_sq_err64(yg, cf, sff, float(zf)))
            assert chosen <= min(errs) * (1 + 1e-5) + 1e-12, (r, k, chosen, min(errs))
            default = _sq_err64(yg, *_candidate(yg, fmt, s0[r, k], zf), float(zf))
            assert chosen <= default * (1 + 1e-5) + 1e-12
            improved += chosen < default * (1 - 1e-6)
    assert improved > 0  # the search does move some scales


def test_a_group_on_the_default_grid_keeps_its_scale():
    """Values zero + code * scale with every code 0..15 present: the default
    scale reproduces them exactly (error 0); ties keep the default."""
    rng = np.random.default_rng(3)
    sf, zf = np.float32(0.1875), np.float32(-1.25)  # exact in fp16
    codes = np.concatenate([np.arange(16), rng.integers(0, 16, 16)])
    y = (zf + codes.astype(np.float32) * sf).astype(np.float32)[None, :]
    y = np.concatenate([y, y], axis=1)  # a 64-wide row of two such groups
    for search in (0, 1):
        c, s, z, e, _ = O.quantize_rows(O.INT4_ASYM, 32, 1.0, y, search=search)
        assert np.all(_h2f(s) == 0.1875) and np.all(_h2f(z) == -1.25) and e[0] == 0.0
        assert np.array_equal(c[0, :32], codes)


def test_constant_groups_are_left_alone():
    y = np.full((2, 64), 0.7, np.float32)
    for fmt, group in ((O.INT4_ASYM, 32), (O.INT2_ASYM, 64)):
        a = O.quantize_rows(fmt, group, 1.0, y, search=0)
        b = O.quantize_rows(fmt, group, 1.0, y, search=1)
        for u, v in zip(a, b):
            assert np.array_equal(u, v)
    z = np.zeros((1, 64), np.float32)
    a, b = O.quantize_rows(O.INT8_SYM, 64, 1.0, z, search=0), O.quantize_rows(O.INT8_SYM, 64, 1.0, z, search=1)
    assert all(np.array_equal(u, v) for u, v in zip(a, b))


def test_mean_squared_error_falls_on_gaussian_groups():
    """The page reports ~27% less error for NVFP4, whose fp8 scale has 3
    mantissa bits; an fp16 scale's neighbours are 0.1% apart, and the same
    search lowers int4 error by about 2% (the figure is recorded, the pin is
    only that it falls)."""
    y = _rows(2000, 128, 11)
    out = []
    for search in (0, 1):
        c, s, z, _, _ = O.quantize_rows(O.INT4_ASYM, 32, 1.0, y, search=search)
        yh = c.reshape(2000, 4, 32) * _h2f(s)[:, :, None] + _h2f(z)[:, :, None]
        out.append(float(np.mean((y.reshape(2000, 4, 32) - yh) ** 2)))
    assert out[1] < out[0] * 0.995, out


def tie_row():
    """A 64-wide row of two int4 groups: 31 values at -0.9375 and one at
    15 * 2^-15.  (max - min) / 15 = 2^-4 + 2^-15 lies halfway between the fp16
    scales 2^-4 (bits 0x2C00, the default: ties to even) and 2^-4 + 2^-14
    (0x2C01); with either scale the one large value is off by exactly
    15 * 2^-15 and every other value is exact, so the two candidates tie in
    fp32.  Values are fp16-exact (usable with the rotation off)."""
    g = np.full(32, -0.9375, np.float32)
    g[5] = 15 * 2.0 ** -15
    return np.concatenate([g, g])[None, :].astype(np.float32)


def test_an_exact_tie_keeps_the_candidate_tried_first():
    y = tie_row()
    _, s0, _, _, _ = O.quantize_rows(O.INT4_ASYM, 32, 1.0, y, search=0)
    _, s1, _, _, _ = O.quantize_rows(O.INT4_ASYM, 32, 1.0, y, search=1)
    assert np.all(s0 == 0x2C00) and np.all(s1 == 0x2C00)
    for bits in (0x2C00, 0x2C01):  # the tie itself, in fp32 as the codec computes it
        c, sf = _candidate(y[0, :32], O.INT4_ASYM, bits, np.float32(-0.9375))
        e = y[0, :32] - (c.astype(np.float32) * np.float32(sf) + np.float32(-0.9375))
        assert float(np.sum(e.astype(np.float64) ** 2)) == 225.0 * 2.0 ** -30
