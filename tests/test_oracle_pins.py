"""Pins of the CPU oracle against facts fixed outside it (no GPU).

Each test checks the oracle against something it does not compute itself: IEEE
bit patterns, closed forms, brute-force enumeration, or a dense numpy evaluation of
the same layer from the generator's interchange form.  The pages print no worked
example or numeric result for this layer, so no pin comes from them.
"""
import itertools
import math

import numpy as np
import pytest

import oracle
import synth
from synth import FMT_Q2, FMT_Q3, FMT_TERNARY
from tests.dense_ref import dequant, expert_dense, silu


# ---- scalar decoders: IEEE binary16 / bfloat16 bit patterns ----------------

@pytest.mark.parametrize("bits,val", [
    (0x3C00, 1.0), (0xC000, -2.0), (0x7BFF, 65504.0), (0x0001, 2.0 ** -24),
    (0x0400, 2.0 ** -14), (0x3555, 1365 * 2.0 ** -12), (0x211F, 1311 * 2.0 ** -17),
    (0x2A66, 1638 * 2.0 ** -15), (0x8000, -0.0), (0x03FF, 1023 * 2.0 ** -24),
])
def test_f16_decode(bits, val):
    assert oracle.lib().oracle_f16_to_f64(bits) == val


@pytest.mark.parametrize("bits,val", [
    (0x3F80, 1.0), (0xBF80, -1.0), (0x4049, 3.140625), (0x0001, 2.0 ** -133),
    (0x7F7F, 255 * 2.0 ** 120), (0x3C23, 163 * 2.0 ** -14),
])
def test_bf16_decode(bits, val):
    assert oracle.lib().oracle_bf16_to_f64(bits) == val


# ---- routing: logits, top-k, gates -------------------------------------------

def test_route_closed_form():
    """x = e_0 makes the logits the first column of Wr; gates by hand."""
    H, E, k = 64, 6, 3
    col = np.array([0.5, -1.0, 2.0, 0.25, 1.5, -0.75], dtype=np.float32)
    Wr = np.zeros((E, H), np.float32)
    Wr[:, 0] = col
    Wr[:, 1] = 7.0          # multiplies x[1] = 0: must not matter
    x = np.zeros((1, H), np.uint16)
    x[0, 0] = 0x3F80        # 1.0
    L, ids, g = oracle.route(x, Wr, None, k)
    assert L[0].tolist() == col.astype(np.float64).tolist()
    assert ids[0].tolist() == [2, 4, 0]
    ex = [math.exp(v) for v in (2.0, 1.5, 0.5)]
    np.testing.assert_allclose(g[0], [v / sum(ex) for v in ex], rtol=1e-15)


def test_route_ties_prefer_lower_id():
    H, E, k = 64, 5, 3
    Wr = np.zeros((E, H), np.float32)
    Wr[:, 0] = [1.0, 3.0, 3.0, 2.0, 3.0]
    x = np.zeros((1, H), np.uint16)
    x[0, 0] = 0x3F80
    _, ids, g = oracle.route(x, Wr, None, k)
    assert ids[0].tolist() == [1, 2, 4]
    np.testing.assert_allclose(g[0], [1 / 3] * 3, rtol=1e-15)


def test_route_bias_shifts_selection():
    H, E, k = 64, 4, 1
    Wr = np.zeros((E, H), np.float32)
    Wr[:, 0] = [1.0, 0.0, 0.5, 0.9]
    x = np.zeros((1, H), np.uint16)
    x[0, 0] = 0x3F80
    b = np.array([0.0, 2.0, 0.0, 0.0], np.float32)
    L = oracle.logits(x, Wr)
    assert oracle.select(L, None, k)[0][0, 0] == 0
    assert oracle.select(L, b, k)[0][0, 0] == 1


@pytest.mark.parametrize("seed,use_bias", [(0, False), (1, True), (2, False)])
def test_route_brute_force(seed, use_bias):
    """E=8, k=2: the chosen pair maximises the summed biased logit over all pairs,
    in p-descending order, and the gates are the softmax over the chosen logits."""
    cfg = synth.micro(T=64, H=256, E=8, k=2, I=64, S=0, seed=seed)
    x = synth.tokens(cfg)
    Wr = synth.router_weight(cfg)
    b = np.random.default_rng(seed).normal(0, 0.3, cfg.E).astype(np.float32) if use_bias else None
    L, ids, g = oracle.route(x, Wr, b, cfg.k)
    z = L + (0 if b is None else b.astype(np.float64))
    for t in range(cfg.T):
        best = max(itertools.combinations(range(cfg.E), cfg.k), key=lambda c: sum(z[t, list(c)]))
        assert set(ids[t].tolist()) == set(best)
        assert z[t, ids[t, 0]] >= z[t, ids[t, 1]]
        sel = z[t, ids[t]]
        ex = np.exp(sel - sel.max())
        np.testing.assert_allclose(g[t], ex / ex.sum(), rtol=1e-13)
        assert abs(g[t].sum() - 1.0) < 1e-12


def test_logits_match_exact_dot():
    """fp64 logits equal a dot product of the exactly decoded inputs (bf16 -> fp32)."""
    cfg = synth.micro(T=5, H=192, E=7, k=2, I=64, S=0, seed=3)
    x = synth.tokens(cfg)
    Wr = synth.router_weight(cfg)
    L = oracle.logits(x, Wr)
    ref = synth.bf16_bits_to_f32(x).astype(np.float64) @ Wr.astype(np.float64).T
    np.testing.assert_allclose(L, ref, rtol=1e-12, atol=1e-13)


# ---- histogram / scan / permutation -----------------------------------------

@pytest.mark.parametrize("T,E,k,seed", [(1, 8, 2, 0), (37, 16, 4, 1), (200, 256, 8, 2)])
def test_permute_invariants(T, E, k, seed):
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, inv = oracle.permute(ids, E)
    assert counts.sum() == T * k
    np.testing.assert_array_equal(counts, np.bincount(ids.ravel(), minlength=E))
    assert offsets[0] == 0 and offsets[-1] == T * k and np.all(np.diff(offsets) == counts)
    assert sorted(perm.tolist()) == list(range(T * k))                  # bijection
    np.testing.assert_array_equal(inv[perm], np.arange(T * k))
    flat = ids.ravel()
    for e in range(E):
        rows = perm[offsets[e]:offsets[e + 1]]
        assert np.all(flat[rows] == e)                                   # grouped by expert
        assert np.all(np.diff(rows // k) > 0)                            # tokens ascending
    # gather by perm then scatter by inv_perm is the identity (bit-exact)
    x = rng.integers(0, 65535, size=(T * k, 33), dtype=np.uint16)
    xp = x[perm]
    np.testing.assert_array_equal(xp[inv], x)


# ---- expert math and combine ------------------------------------------------

def _layer(cfg):
    return synth.Layer(cfg)


@pytest.mark.parametrize("fmt", [FMT_TERNARY, FMT_Q2, FMT_Q3])
def test_single_expert_is_dense_swiglu(fmt):
    """E = k = 1, S = 0: the layer is a dense SwiGLU MLP (numpy fp64 matmuls)."""
    formats = {FMT_TERNARY: "ternary", FMT_Q2: "q2", FMT_Q3: "q3"}[fmt]
    cfg = synth.micro(T=6, H=192, E=1, k=1, I=128, S=0, formats=formats, seed=4)
    layer = _layer(cfg)
    x = synth.tokens(cfg)
    _, ids, g = oracle.route(x, layer.router_w, None, 1)
    assert np.all(ids == 0) and np.all(g == 1.0)
    y = oracle.forward_tokens(layer, x, ids, g, range(cfg.T), threads=2)
    ref = expert_dense(fmt, layer.expert(0), synth.bf16_bits_to_f32(x).astype(np.float64))
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-11 * np.abs(ref).max())


@pytest.mark.parametrize("cfgkw", [
    dict(T=12, H=128, E=8, k=2, I=64, S=1, formats="mixed", seed=5),
    dict(T=9, H=256, E=8, k=2, I=128, S=0, formats="q2", seed=0),
    dict(T=7, H=192, E=6, k=3, I=64, S=1, formats="mixed", seed=6),
])
def test_brute_force_all_experts_masked(cfgkw):
    """Run every expert on every token densely, keep the brute-force top-k set,
    weight by the softmax over its logits, add the shared expert."""
    cfg = synth.micro(**cfgkw)
    layer = _layer(cfg)
    x = synth.tokens(cfg)
    L, ids, g = oracle.route(x, layer.router_w, None, cfg.k)
    y = oracle.forward_tokens(layer, x, ids, g, range(cfg.T), threads=2)
    x64 = synth.bf16_bits_to_f32(x).astype(np.float64)
    all_y = np.stack([expert_dense(int(layer.fmt[e]), layer.expert(e), x64)
                      for e in range(cfg.E + cfg.S)])            # [E+S][T][H]
    for t in range(cfg.T):
        best = max(itertools.combinations(range(cfg.E), cfg.k), key=lambda c: sum(L[t, list(c)]))
        z = L[t, list(best)]
        w = np.exp(z - z.max())
        w /= w.sum()
        ref = sum(w[i] * all_y[e, t] for i, e in enumerate(best))
        ref = ref + sum(all_y[cfg.E + s, t] for s in range(cfg.S))
        np.testing.assert_allclose(y[t], ref, rtol=1e-10, atol=1e-11 * np.abs(ref).max())


def _const_mats(rows_gu, H, c_gu, s_gu, rows_d, I, c_d, s_d, fmt):
    def mat(rows, K, c, s):
        byte = (c & 3) * 0x55                                  # same 2-bit code in all fields
        codes = np.full((rows, K // 4), byte, np.uint8)
        hi = np.full((rows, K // 8), 0xFF if c >= 4 else 0, np.uint8) if fmt == FMT_Q3 else None
        scales = np.full((rows, K // 64), np.float16(s).view(np.uint16), np.uint16)
        return codes, hi, scales
    return {"gate": mat(rows_gu, H, c_gu, s_gu), "up": mat(rows_gu, H, c_gu, s_gu),
            "down": mat(rows_d, I, c_d, s_d)}


@pytest.mark.parametrize("fmt,c_gu,c_d,o", [(FMT_Q2, 3, 0, 1.5), (FMT_Q3, 6, 1, 3.5),
                                            (FMT_TERNARY, 2, 0, 1.0)])
def test_constant_codes_closed_form(fmt, c_gu, c_d, o):
    """All gate/up codes c, scale s: a = b = (c - o) s sum(x); h = silu(a) a;
    y_m = (c_d - o) s_d * I * h for every output m."""
    H, I = 128, 64
    s_gu, s_d = 0.03125, 0.046875            # exact in fp16
    mats = _const_mats(I, H, c_gu, s_gu, H, I, c_d, s_d, fmt)
    rng = np.random.default_rng(7)
    x = synth.f32_to_bf16_bits(rng.standard_normal((3, H)).astype(np.float32))
    y = oracle.expert_ffn(H, I, fmt, mats, x)
    xs = synth.bf16_bits_to_f32(x).astype(np.float64).sum(axis=1)
    a = (c_gu - o) * s_gu * xs
    expect = (c_d - o) * s_d * I * (a / (1 + np.exp(-a)) * a)
    np.testing.assert_allclose(y, np.repeat(expect[:, None], H, axis=1), rtol=1e-12)


def test_zero_input_gives_zero():
    cfg = synth.micro(T=4, H=128, E=8, k=2, I=64, S=1, seed=8)
    layer = _layer(cfg)
    x = np.zeros((cfg.T, cfg.H), np.uint16)
    L, ids, g = oracle.route(x, layer.router_w, None, cfg.k)
    assert np.all(L == 0)
    assert ids[0].tolist() == [0, 1]                       # all tied: lowest ids
    y = oracle.forward_tokens(layer, x, ids, g, range(cfg.T), threads=2)
    assert np.all(y == 0)


def test_shared_expert_added_unweighted():
    """With routed experts whose down matrix is all zero-value codes, the output is
    exactly the shared expert's dense output."""
    cfg = synth.micro(T=5, H=128, E=4, k=2, I=64, S=1, formats="ternary", seed=9)
    layer = _layer(cfg)

    class ZeroRouted:
        def __init__(self, base):
            self.cfg, self.fmt, self.base = base.cfg, base.fmt, base

        def expert(self, e):
            m = self.base.expert(e)
            if e < self.cfg.E:
                c, h, s = m["down"]
                m["down"] = (np.full_like(c, 0x55), h, s)       # ternary code 1 = value 0
            return m

    x = synth.tokens(cfg)
    _, ids, g = oracle.route(x, layer.router_w, None, cfg.k)
    y = oracle.forward_tokens(ZeroRouted(layer), x, ids, g, range(cfg.T), threads=2)
    ref = expert_dense(int(layer.fmt[cfg.E]), layer.expert(cfg.E),
                       synth.bf16_bits_to_f32(x).astype(np.float64))
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-12)


def test_ternary_code_three_rejected():
    H, I = 64, 64
    mats = _const_mats(I, H, 1, 0.03125, H, I, 1, 0.03125, FMT_TERNARY)
    c, h, s = mats["gate"]
    c = c.copy()
    c[3, 2] = 0xFF
    mats["gate"] = (c, h, s)
    with pytest.raises(ValueError):
        oracle.expert_ffn(H, I, FMT_TERNARY, mats, np.zeros((1, H), np.uint16))


def test_dequant_scale_index_is_per_row_group():
    """A single nonzero scale at (row 3, group 1) yields nonzero weights exactly in
    row 3, columns 64..127 (catches a transposed scale index)."""
    H, I = 256, 64
    mats = _const_mats(I, H, 3, 0.0, H, I, 0, 0.0, FMT_Q2)
    c, h, s = mats["gate"]
    s = s.copy()
    s[3, 1] = np.float16(0.5).view(np.uint16)
    x = np.zeros((1, H), np.uint16)
    x[0, 100] = 0x3F80
    mats["gate"] = (c, h, s)
    W = dequant(FMT_Q2, mats["gate"])
    assert np.count_nonzero(W) == 64 and np.all(W[3, 64:128] == 0.75)
    # through the oracle: only h[3] can be nonzero, and a = 0.75 * x[100]
    mats["up"] = (c, h, s)
    mats["down"] = _const_mats(I, H, 3, 0.5, H, I, 3, 0.5, FMT_Q2)["down"]
    y = oracle.expert_ffn(H, I, FMT_Q2, mats, x)
    a = 0.75
    np.testing.assert_allclose(y[0], np.full(H, 0.75 * silu(a) * a), rtol=1e-14)


# ---- the oracle's reader of the packed format -------------------------------

def _hand_packed(fmt, H, I, gu_codes, gu_hi, dn_codes, dn_hi, scale_bits):
    """Packed buffer (format version 2) for E=1, S=0 built directly from the format's
    definition, element by element (tests only)."""
    def blocks(rows, K, code_of):
        G = K // 64
        NC = (G + 7) // 8
        codes = np.zeros(rows * K // 16, np.uint32)
        hi = np.zeros(rows * K // 32, np.uint32)
        scales = np.zeros((rows // 16) * NC * 128, np.uint16)
        for pr in range(rows):
            j, r = divmod(pr, 16)
            for k in range(K):
                g, kk = divmod(k, 64)
                c, gl = divmod(g, 8)
                ng = min(8, G - 8 * c)
                wl = 4 * gl + kk // 16
                pos = r * 32 + (wl ^ (4 * (r % 8))) if ng == 8 else r * 4 * ng + wl
                idx = (4 * K * j + 2048 * c) // 4 + pos
                p_, h_ = divmod(k % 16, 2)
                cv = code_of(pr, k)
                codes[idx] |= np.uint32((cv & 3) << (16 * h_ + 2 * p_))
                vl = 2 * gl + kk // 32
                hpos = r * 16 + (vl ^ (2 * ((r % 8) // 2))) if ng == 8 else r * 2 * ng + vl
                hidx = (128 * G * j + 1024 * c) // 4 + hpos
                q_, rest = divmod(k % 32, 16)
                p1, h1 = divmod(rest, 2)
                hi[hidx] |= np.uint32(((cv >> 2) & 1) << (16 * h1 + 8 * q_ + p1))
            for g in range(G):
                c, gl = divmod(g, 8)
                scales[(256 * NC * j + 256 * c) // 2 + 8 * r + gl] = scale_bits
        return scales, codes, hi

    def gu_src(r):                   # packed GU row -> (gate?, source row)
        b, jj = divmod(r, 16)
        return (jj < 8), 8 * b + (jj % 8)

    gu_full = lambda r, k: (gu_codes[0] if gu_src(r)[0] else gu_codes[1])[gu_src(r)[1], k]
    gs, gc, gh = blocks(2 * I, H, gu_full)
    ds, dc, dh = blocks(H, I, lambda r, k: dn_codes[r, k])
    arrays = [gs, gc, gh if fmt == FMT_Q3 else None, ds, dc, dh if fmt == FMT_Q3 else None]
    off = 256 + 64
    offs = []
    blobs = []
    for a in arrays:
        if a is None:
            offs.append(0)
            continue
        off = (off + 255) // 256 * 256
        offs.append(off)
        blobs.append((off, a.tobytes()))
        off += a.nbytes
    total = off
    buf = bytearray(total)
    hdr = np.array([0x50454F4D, 2, H, I, 1, 0, 64, 8], np.uint32).tobytes()
    buf[0:32] = hdr
    buf[32:40] = np.uint64(total).tobytes()
    ent = np.zeros(8, np.uint64)
    ent[0] = fmt
    ent[1:7] = offs
    buf[256:320] = ent.tobytes()
    for o, b in blobs:
        buf[o:o + len(b)] = b
    return np.frombuffer(bytes(buf), np.uint8)


@pytest.mark.parametrize("fmt,H,I", [(FMT_Q2, 128, 64), (FMT_Q3, 128, 64), (FMT_Q3, 576, 64),
                                    (FMT_Q2, 64, 1024)])
def test_oracle_unpack_reads_hand_built_buffer(fmt, H, I):
    """Covers full 8-group chunks (swizzled) and tail chunks of 1, 2 and 1 groups."""
    rng = np.random.default_rng(10)
    top = 8 if fmt == FMT_Q3 else 4
    g = rng.integers(0, top, size=(I, H))
    u = rng.integers(0, top, size=(I, H))
    d = rng.integers(0, top, size=(H, I))
    buf = _hand_packed(fmt, H, I, (g, u), None, d, None, np.float16(0.03).view(np.uint16))
    for which, ref, rows, K in ((0, g, I, H), (1, u, I, H), (2, d, H, I)):
        f, codes, scales = oracle.unpack(buf, 0, which, rows, K)
        assert f == fmt
        np.testing.assert_array_equal(codes, ref)
        assert np.all(scales == np.float16(0.03).view(np.uint16))
