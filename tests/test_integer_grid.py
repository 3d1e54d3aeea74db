"""Bounds the few-token integer gate/up path relies on (host-side arithmetic, no GPU).

The path puts each 64-group of a token on a 12-bit grid, q = rint(x 2^e) with
e = 11 - floor(log2 max|x|), stores B = 4q or q as two signed bytes lo + 256 hi, and
sums 64 products A B per group in an int32 accumulator that starts at the bit pattern
of 1.5 * 2^23, reading the result back as fp32.  These tests check, from those
definitions alone, that the digits fit their bytes, that the worst-case group sum
stays inside the window where the fp32 reinterpretation is exact, and how far the grid
moves bf16 tokens.
"""
import numpy as np

import synth


def _grid(x):
    """q and e of one group, as the path defines them (x: float64 array of one group)."""
    m = np.max(np.abs(x))
    e = 11 - int(np.floor(np.log2(m))) if m > 0 else 0
    return np.rint(np.ldexp(x, e)).astype(np.int64), e


def _bf16(a):
    return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(np.asarray(a, np.float32))).astype(np.float64)


def test_digits_fit_signed_bytes_for_extreme_groups():
    # the largest |q| comes from a group whose maximum is just below a power of two
    for m in (1.0, 1.9921875, 2.0, 3.99, 0.015625, 1e-30, 3e38):
        x = _bf16([m, -m, m / 3, 0.0] + [m / 7] * 60)
        q, _ = _grid(x)
        assert np.abs(q).max() <= 4096
        for bv in (4 * q, q):
            lo = ((bv & 0xFF) ^ 0x80) - 0x80
            hi = (bv - lo) >> 8
            assert np.all((lo >= -128) & (lo <= 127)) and np.all((hi >= -128) & (hi <= 127))
            assert np.array_equal(lo + 256 * hi, bv)


def test_group_sum_stays_inside_the_magic_window():
    # worst case per digit column: 64 products of the largest A byte (4 x code 3 = 12)
    # with the largest digit magnitude (128); the fp32 value 1.5 * 2^23 + D is exact
    # and recovers D by one subtraction while |D| < 2^22
    d_max = 64 * 12 * 128
    assert d_max < 2 ** 22
    for d in (-d_max, -1, 0, 1, d_max):
        bits = np.int64(0x4B400000) + d
        f = np.array([bits], np.uint32).view(np.float32)[0]
        assert float(f) - 12582912.0 == d


def test_grid_moves_bf16_tokens_by_about_1e_4_rms():
    rng = np.random.default_rng(0)
    x = _bf16(rng.standard_normal(64 * 4096)).reshape(-1, 64)
    err = []
    for g in x:
        q, e = _grid(g)
        xt = np.ldexp(q.astype(np.float64), -e)
        big = np.abs(g) >= np.max(np.abs(g)) / 16
        assert np.array_equal(xt[big], g[big])            # exact above 1/16 of the group maximum
        assert np.max(np.abs(xt - g)) <= np.max(np.abs(g)) / 4096
        err.append(xt - g)
    rel = np.sqrt(np.mean(np.square(err))) / np.sqrt(np.mean(np.square(x)))
    assert 5e-5 < rel < 2e-4
