"""Host-side checks of the C ABI library (no GPU): exported symbols, argument
validation, and the packer checked against the oracle's independent reader of the
packed format."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import bit_routed_expert_fp32_b200 as moe
import oracle
import synth
from tests.dense_ref import codes_int

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_header_declarations_match_binding():
    assert declared_functions() == sorted(moe.EXPORTS)


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    syms = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in syms, name
        assert getattr(moe.lib(), name) is not None
    assert moe.lib().moe_abi_version() == 1
    assert moe.moe_status_string(0) == "ok"


def _shape(H=128, I=64, E=4, k=2, S=1):
    return moe.Shape(H, I, E, k, S)


def test_argument_errors_are_synchronous():
    L = moe.lib()
    sz = ctypes.c_size_t(0)
    fmt = np.ones(5, np.uint8)
    assert L.moe_packed_size(None, fmt.ctypes.data, ctypes.byref(sz)) == 1
    assert L.moe_event_record(None, None) == 1          # null event: rejected before any CUDA call
    bad = _shape(H=100)
    assert L.moe_packed_size(ctypes.byref(bad), fmt.ctypes.data, ctypes.byref(sz)) == 1
    assert L.moe_workspace_size(ctypes.byref(_shape(k=5)), 4, ctypes.byref(sz)) == 1       # k > E
    assert L.moe_workspace_size(ctypes.byref(_shape()), -1, ctypes.byref(sz)) == 1
    fmt_bad = np.array([1, 1, 4, 1, 1], np.uint8)                 # 3 is the dense ternary storage form
    assert L.moe_packed_size(ctypes.byref(_shape()), fmt_bad.ctypes.data, ctypes.byref(sz)) == 1
    sh = _shape()
    fake = ctypes.c_void_p(0x1000)
    r = moe.Routing(*([0x1000] * 6))
    assert L.moe_workspace_size(ctypes.byref(sh), 8, ctypes.byref(sz)) == 0
    need = sz.value
    # workspace too small, negative T, null x, null routing member: rejected before any launch
    assert L.moe_route(ctypes.byref(sh), 8, fake, fake, None, ctypes.byref(r), fake, need - 1, None) == 3
    assert L.moe_route(ctypes.byref(sh), -1, fake, fake, None, ctypes.byref(r), fake, need, None) == 1
    assert L.moe_route(ctypes.byref(sh), 8, None, fake, None, ctypes.byref(r), fake, need, None) == 1
    r0 = moe.Routing(0x1000, 0x1000, 0, 0x1000, 0x1000, 0x1000)
    assert L.moe_route(ctypes.byref(sh), 8, fake, fake, None, ctypes.byref(r0), fake, need, None) == 1
    assert L.moe_forward(ctypes.byref(sh), 8, fake, fake, ctypes.byref(r), fake, 7, fake, need, None) == 1
    # T = 0 is a no-op
    assert L.moe_route(ctypes.byref(sh), 0, fake, fake, None, ctypes.byref(r), fake, need, None) == 0
    assert L.moe_forward(ctypes.byref(sh), 0, fake, fake, ctypes.byref(r), fake, 0, fake, need, None) == 0


def test_static_entry_point_checks_everything_before_any_cuda_call():
    """moe_decode_static runs every argument check of moe_route and moe_forward before
    it touches the device (no GPU here: any CUDA call would fail with MOE_ERR_CUDA)."""
    L = moe.lib()
    fake = ctypes.c_void_p(0x1000)
    r = moe.Routing(*([0x1000] * 6))
    r0 = moe.Routing(0x1000, 0x1000, 0, 0x1000, 0x1000, 0x1000)
    sh = _shape()
    assert L.moe_decode_static(None, 4, fake, fake, None, fake, ctypes.byref(r), fake, None) == 1
    assert L.moe_decode_static(ctypes.byref(_shape(k=5)), 4, fake, fake, None, fake, ctypes.byref(r), fake,
                               None) == 1                                  # k > E
    bad_s = moe.Shape(128, 64, 4, 2, -1)                                      # negative n_shared
    assert L.moe_decode_static(ctypes.byref(bad_s), 4, fake, fake, None, fake, ctypes.byref(r), fake, None) == 1
    assert L.moe_decode_static(ctypes.byref(sh), -1, fake, fake, None, fake, ctypes.byref(r), fake, None) == 1
    assert L.moe_decode_static(ctypes.byref(sh), 4, None, fake, None, fake, ctypes.byref(r), fake, None) == 1
    assert L.moe_decode_static(ctypes.byref(sh), 4, fake, None, None, fake, ctypes.byref(r), fake, None) == 1
    assert L.moe_decode_static(ctypes.byref(sh), 4, fake, fake, None, None, ctypes.byref(r), fake, None) == 1
    assert L.moe_decode_static(ctypes.byref(sh), 4, fake, fake, None, fake, ctypes.byref(r0), fake, None) == 1
    assert L.moe_decode_static(ctypes.byref(sh), 4, fake, fake, None, fake, ctypes.byref(r), None, None) == 1
    big = moe.Shape(7168, 2048, 256, 8, 1)                                   # 64 tokens need ~19 MB
    assert L.moe_decode_static(ctypes.byref(big), 64, fake, fake, None, fake, ctypes.byref(r), fake, None) == 3
    assert L.moe_decode_static(ctypes.byref(sh), 0, fake, fake, None, fake, ctypes.byref(r), fake, None) == 0
    assert L.moe_workspace_set_test_stall(None, 1 << 20, 100, None) == 1


def test_forward_plan_names_the_kernels_and_launches():
    """moe_forward_plan (host-only): the path choice, the launch count of moe_route +
    moe_forward and the K parts, with moe_forward's argument errors."""
    import dataclasses
    L = moe.lib()
    plan = np.zeros(4, np.int32)
    sh = _shape(H=256, I=128, E=8, k=2, S=1)
    assert L.moe_forward_plan(ctypes.byref(sh), 4, 0, None) == 1
    assert L.moe_forward_plan(None, 4, 0, plan.ctypes.data) == 1
    assert L.moe_forward_plan(ctypes.byref(sh), -1, 0, plan.ctypes.data) == 1
    assert L.moe_forward_plan(ctypes.byref(sh), 4, 7, plan.ctypes.data) == 1                 # no such path
    assert L.moe_forward_plan(ctypes.byref(sh), 17, moe.PATH_DECODE_FUSED, plan.ctypes.data) == 2
    odd = _shape(H=192, I=128, E=8, k=2, S=1)                                               # H not a multiple of 128
    assert L.moe_forward_plan(ctypes.byref(odd), 100, moe.PATH_PREFILL, plan.ctypes.data) == 2
    cfg = synth.micro(T=1, H=256, E=8, k=2, I=128, S=1)
    assert moe.moe_forward_plan(cfg, 0) == {"path": "decode", "launches": 0, "kparts_gu": 1, "kparts_dn": 1}
    # decode above 64 tokens when the tcgen05 kernels cannot run: the router's three
    # kernels, the decode operands, gate/up, down, combine
    cfg_odd = synth.micro(T=100, H=192, E=8, k=2, I=128, S=1)
    assert moe.moe_forward_plan(cfg_odd, 100) == {"path": "decode", "launches": 3 + 1 + 3, "kparts_gu": 1,
                                                  "kparts_dn": 1}
    assert moe.moe_forward_plan(cfg, 4, moe.PATH_PREFILL)["launches"] == 1 + 4
    assert moe.moe_forward_plan(cfg, 1, moe.PATH_DECODE_FUSED) == {"path": "fused", "launches": 2, "kparts_gu": 1,
                                                                     "kparts_dn": 1}
    assert moe.moe_forward_plan(cfg, 1, moe.PATH_AUTO | moe.OUT_F32) == moe.moe_forward_plan(cfg, 1)   # fp32 y: same kernels
    # the full-size layer: one token splits K (gate/up in 7 parts, which adds the
    # reduction launch), 5-8 tokens take the fused kernel, above 64 the tcgen05 kernels
    full = synth.CONFIGS[2]
    assert moe.moe_forward_plan(full, 1) == {"path": "decode", "launches": 5, "kparts_gu": 7, "kparts_dn": 4}
    for T in range(1, 97):
        p = moe.moe_forward_plan(dataclasses.replace(full, T=T), T)
        want = "prefill" if T > 64 else "fused" if 5 <= T <= 8 else "decode"
        assert p["path"] == want, (T, p)
        if want == "decode":
            assert p["launches"] == 1 + 3 + (p["kparts_gu"] > 1)


def test_workspace_size_never_shrinks_as_tokens_grow():
    # A workspace sized for max_tokens must serve every smaller T: the K-part split
    # of the decode passes and the few-token integer operands must not make a smaller
    # T need more bytes than a larger one.
    for cfg in (synth.CONFIGS[2], synth.micro(T=8, H=256, E=8, k=2, I=128, S=0)):
        sizes = [moe.moe_workspace_size(cfg, T) for T in range(0, 97)]
        assert all(b >= a for a, b in zip(sizes, sizes[1:]))
    # the full-size layer: the library's static scratch holds 21 tokens, not 22
    cfg = synth.CONFIGS[2]
    assert moe.moe_workspace_size(cfg, 21) <= moe.STATIC_WS_BYTES < moe.moe_workspace_size(cfg, 22)


@pytest.mark.parametrize("H,I,formats", [(128, 64, "mixed"), (192, 128, "q3"), (256, 64, "ternary"),
                                         (64, 192, "q2"), (384, 256, "mixed")])
def test_pack_roundtrip_through_oracle_reader(H, I, formats):
    cfg = synth.micro(T=1, H=H, E=6, k=2, I=I, S=1, formats=formats, seed=H + I)
    layer = synth.Layer(cfg)
    buf = moe.pack_layer(cfg, layer.fmt, layer.expert)
    assert buf.size == moe.moe_packed_size(cfg, layer.fmt)
    for e in range(cfg.E + cfg.S):
        mats = layer.expert(e)
        for which, name, rows, K in ((0, "gate", I, H), (1, "up", I, H), (2, "down", H, I)):
            f, codes, scales = oracle.unpack(buf, e, which, rows, K)
            c, h, s = mats[name]
            assert f == layer.fmt[e]
            np.testing.assert_array_equal(codes, codes_int(c, h))
            np.testing.assert_array_equal(scales, s)


def test_pack_edge_codes():
    """All-minimum and all-maximum codes survive the round trip."""
    cfg = synth.micro(T=1, H=128, E=2, k=1, I=64, S=0, formats="q3", seed=1)
    fmt = np.array([2, 2], np.uint8)

    def mats(e):
        byte = 0x00 if e == 0 else 0xFF
        out = {}
        for name, rows, K in (("gate", 64, 128), ("up", 64, 128), ("down", 128, 64)):
            out[name] = (np.full((rows, K // 4), byte, np.uint8), np.full((rows, K // 8), byte, np.uint8),
                         np.full((rows, K // 64), 0x3C00, np.uint16))
        return out

    buf = moe.pack_layer(cfg, fmt, mats)
    for e, v in ((0, 0), (1, 7)):
        for which, rows, K in ((0, 64, 128), (1, 64, 128), (2, 128, 64)):
            f, codes, scales = oracle.unpack(buf, e, which, rows, K)
            assert np.all(codes == v) and np.all(scales == 0x3C00)


def test_pack_rejects_ternary_code_three_and_small_buffer():
    cfg = synth.micro(T=1, H=64, E=1, k=1, I=64, S=0, formats="ternary", seed=2)
    layer = synth.Layer(cfg)
    m = layer.expert(0)
    size = moe.moe_packed_size(cfg, layer.fmt)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_pack_experts(cfg, layer.fmt, 0, [m], np.zeros(size - 1, np.uint8))
    assert ei.value.status == 3
    c, h, s = m["down"]
    c = c.copy()
    c[5, 3] |= 0x0C          # one 2-bit field = 3
    m["down"] = (c, h, s)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_pack_experts(cfg, layer.fmt, 0, [m], np.zeros(size, np.uint8))
    assert ei.value.status == 1


def test_pack_roundtrip_random_shapes_and_formats():
    """Property check of the packer against the oracle's independent reader: random
    shapes (H, I multiples of 64, partial chunks included), expert counts and a random
    format per expert, shared expert in any format."""
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=25, deadline=None, derandomize=True)
    @given(st.integers(1, 9), st.integers(1, 6), st.integers(1, 6), st.integers(0, 1), st.data())
    def check(hg, ig, E, S, data):
        H, I = 64 * hg, 64 * ig
        fmts = np.array(data.draw(st.lists(st.integers(0, 2), min_size=E + S, max_size=E + S)), np.uint8)
        cfg = synth.micro(T=1, H=H, E=E, k=1, I=I, S=S, formats="mixed", seed=hg * 100 + ig * 10 + E)
        rng = np.random.default_rng(int(fmts.sum()) + H + I)

        def mats(e):
            out = {}
            for name, rows, K in (("gate", I, H), ("up", I, H), ("down", H, I)):
                codes = rng.integers(0, 256, (rows, K // 4), dtype=np.uint8)
                if fmts[e] == synth.FMT_TERNARY:          # fields 0..2 only
                    f = np.stack([(codes >> (2 * i)) & 3 for i in range(4)])
                    f = np.where(f == 3, 2, f)
                    codes = (f[0] | (f[1] << 2) | (f[2] << 4) | (f[3] << 6)).astype(np.uint8)
                hi = rng.integers(0, 256, (rows, K // 8), dtype=np.uint8) if fmts[e] == synth.FMT_Q3 else None
                sc = np.float16(rng.uniform(-0.05, 0.05, (rows, K // 64))).view(np.uint16)
                out[name] = (codes, hi, sc)
            return out

        cache = {e: mats(e) for e in range(E + S)}
        buf = moe.pack_layer(cfg, fmts, lambda e: cache[e])
        assert buf.size == moe.moe_packed_size(cfg, fmts)
        for e in range(E + S):
            for which, name, rows, K in ((0, "gate", I, H), (1, "up", I, H), (2, "down", H, I)):
                f, codes, scales = oracle.unpack(buf, e, which, rows, K)
                c, h, s = cache[e][name]
                assert f == fmts[e]
                np.testing.assert_array_equal(codes, codes_int(c, h))
                np.testing.assert_array_equal(scales, s)

    check()
