"""Bounds the integer MMA path of the decode kernels relies on (the fused kernel; the
separate gate/up and down launches up to four tokens; host-side arithmetic, no GPU).

The path puts each 64-group of a row (a token, or an h row) on a 12-bit grid,
q = rint(v 2^e) with e = 11 - floor(log2 max|v|), stores B = 4q or q as two signed
bytes lo + 256 hi, and sums 64 products A B per group and digit in int32 (the low
digit's accumulator starting at the bit pattern of 1.5 * 2^23); the two digit sums are
joined as d0 + 256 d1, the code offset is removed exactly as D - 4 o sum q, and the
result is read back as fp32.  These tests check, from those definitions alone, that the
digits fit their bytes, that the joined and corrected group sum stays inside the window
where the fp32 reinterpretation is exact, that the steps give exactly
sum 4 (c - o) q, and how far the grid moves bf16 values.
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


def test_joined_and_corrected_sum_is_exact_and_inside_the_window():
    rng = np.random.default_rng(1)
    magic = 0x4B400000
    for o4, cmax in ((4, 2), (6, 3)):                        # ternary (o = 1), 2-bit (o = 1.5)
        for trial in range(200):
            c = rng.integers(0, cmax + 1, 64)
            if trial == 0:
                q = np.full(64, 4096)                         # the extreme group
                c = np.full(64, cmax if o4 == 6 else 2)
            else:
                q = rng.integers(-4096, 4097, 64)
            # class of element k: c = (k mod 8) / 2; odd classes hold 4 c with B = q,
            # even classes hold c with B = 4 q: every product is 4 c q
            cls = (np.arange(64) % 8) // 2
            a = np.where(cls % 2 == 1, 4 * c, c)
            b = np.where(cls % 2 == 1, q, 4 * q)
            lo = ((b & 0xFF) ^ 0x80) - 0x80
            hi = (b - lo) >> 8
            d0 = magic + int(np.sum(a * lo))
            d1 = int(np.sum(a * hi))
            joined = d0 + 256 * d1 - o4 * int(np.sum(q))
            D = joined - magic
            assert D == int(np.sum(4 * c * q)) - o4 * int(np.sum(q))
            assert abs(D) < 2 ** 22
            f = np.array([joined], np.uint32).view(np.float32)[0]
            assert float(f) - 12582912.0 == D
