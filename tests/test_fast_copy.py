"""The fast mode's 2-bit copy of 3-bit experts (host side, no GPU): the requantiser
against the nearest-level property, fp16 scale doubling at the format's edges, argument
errors, and a whole layer's copy read back through the oracle's own unpacker."""
import numpy as np
import pytest

import bit_routed_expert_fp32_b200 as moe
import oracle
import synth
from tests.dense_ref import codes_int


def _f16(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def _q3_matrix(rows, K, seed):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, (rows, K // 4), dtype=np.uint8)
    hi = rng.integers(0, 256, (rows, K // 8), dtype=np.uint8)
    scales = np.float16(rng.uniform(0.01, 0.05, (rows, K // 64))).view(np.uint16)
    return codes, hi, scales


def test_each_weight_moves_to_the_nearest_2bit_level():
    codes, hi, scales = _q3_matrix(24, 192, 1)
    oc, oh, osc = moe.moe_requantize_q3_to_q2(codes, hi, scales)
    assert oh is None
    c3 = codes_int(codes, hi)                       # 0..7
    c2 = codes_int(oc, None)                        # 0..3
    s3 = np.repeat(_f16(scales), 64, axis=1)
    s2 = np.repeat(_f16(osc), 64, axis=1)
    w3 = (c3 - 3.5) * s3
    w2 = (c2 - 1.5) * s2
    assert np.array_equal(np.abs(w2 - w3), s3 / 2)              # exactly half the old scale
    # brute force: the chosen level is the nearest of the four the new scale allows
    levels = (np.arange(4)[None, None, :] - 1.5) * s2[:, :, None]
    dist = np.abs(levels - w3[:, :, None])
    assert np.array_equal(np.argmin(dist, axis=2), c2)
    assert np.all(np.sort(dist, axis=2)[:, :, 1] > np.sort(dist, axis=2)[:, :, 0])   # no ties


@pytest.mark.parametrize("bits,doubled", [
    (0x0001, 0x0002),       # smallest subnormal
    (0x03FF, 0x07FE),       # largest subnormal -> normal
    (0x0400, 0x0800),       # smallest normal
    (0x3C00, 0x4000),       # 1.0
    (0x77FF, 0x7BFF),       # largest value whose double is finite
    (0x0000, 0x0000),       # zero
    (0xBC00, 0xC000),       # -1.0
])
def test_scale_doubling_is_exact(bits, doubled):
    codes, hi, _ = _q3_matrix(1, 64, 2)
    _, _, osc = moe.moe_requantize_q3_to_q2(codes, hi, np.array([[bits]], np.uint16))
    assert osc[0, 0] == doubled
    assert _f16(doubled) == 2 * _f16(bits)


@pytest.mark.parametrize("bits", [0x7800, 0x7BFF, 0x7C00, 0x7E00, 0xFC00])
def test_scales_without_a_finite_double_are_refused(bits):
    codes, hi, _ = _q3_matrix(1, 64, 3)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_requantize_q3_to_q2(codes, hi, np.array([[bits]], np.uint16))
    assert ei.value.status == 1


def test_shape_errors():
    codes, hi, scales = _q3_matrix(2, 128, 4)
    with pytest.raises(ValueError):
        moe.moe_requantize_q3_to_q2(codes, hi[:, :8], scales)
    with pytest.raises(ValueError):
        moe.moe_requantize_q3_to_q2(codes, hi, scales[:, :1])


def test_layer_copy_reads_back_through_the_oracle_unpacker():
    cfg = synth.micro(T=1, H=192, E=10, k=2, I=128, S=1, formats="mixed", seed=5)
    layer = synth.Layer(cfg)
    assert (layer.fmt == synth.FMT_Q3).any() and (layer.fmt != synth.FMT_Q3).any()
    fmt2, fn2 = moe.fast_copy(layer.fmt, layer.expert)
    assert not (fmt2 == synth.FMT_Q3).any()
    buf = moe.pack_layer(cfg, fmt2, fn2)
    assert buf.size == moe.moe_packed_size(cfg, fmt2) < moe.moe_packed_size(cfg, layer.fmt)
    for e in range(cfg.E + cfg.S):
        mats = layer.expert(e)
        for which, name, rows, K in ((0, "gate", cfg.I, cfg.H), (1, "up", cfg.I, cfg.H), (2, "down", cfg.H, cfg.I)):
            f, codes, scales = oracle.unpack(buf, e, which, rows, K)
            c, h, s = mats[name]
            if layer.fmt[e] == synth.FMT_Q3:
                assert f == synth.FMT_Q2
                np.testing.assert_array_equal(codes, codes_int(c, h) >> 1)
                np.testing.assert_array_equal(_f16(scales), 2 * _f16(s))
            else:
                assert f == layer.fmt[e]
                np.testing.assert_array_equal(codes, codes_int(c, h))
                np.testing.assert_array_equal(scales, s)
