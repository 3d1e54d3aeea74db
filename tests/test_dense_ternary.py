"""Dense ternary storage form (MOE_FMT_TERNARY_DENSE in include/moe.h).

Ternary experts are in the pages' mix (ossradar.top, Xolotl README, "Get a model") and
the bytes moved per token set the speed (the same README, "Fast mode (DeepSeek-V4.1)");
five base-3 codes fit a byte (3^5 = 243 <= 256), 1.6 bits per weight against the 2 of
the kernels' ternary layout.  The form is a storage one: the packer writes it, the
expert cache moves it from host memory and expands it on the GPU, no expert kernel
reads it.

CPU: the oracle's reader against a buffer whose bytes are placed by hand from the
format's definition; the packer's dense output read back by the oracle; sizes; a byte
above 242 is rejected.  GPU: a cache loaded from a dense host buffer holds, for every
expert, exactly the bytes the packer writes for the same expert in the 2-bit ternary
layout (the expansion is bit-exact), the layer run from it equals the oracle, and
moe_forward on a dense device buffer reports MOE_DETAIL_FORMAT on every path and
computes nothing, leaving the workspace usable.
"""
import numpy as np
import pytest

import oracle
import synth
from tests import harness as H
from tests.dense_ref import codes_int

DENSE = 3


def _dense_row(codes_row):
    """Bytes of one dense row: byte i = sum_j c[5i + j] 3^j (codes past K are 0)."""
    K = codes_row.size
    out = np.zeros((K + 4) // 5, np.uint8)
    for i in range(out.size):
        v = 0
        for j in range(5):
            k = 5 * i + j
            v += (int(codes_row[k]) if k < K else 0) * 3 ** j
        out[i] = v
    return out


def _hand_dense(H_, I, g, u, d, scale_bits):
    """A packed buffer (E = 1, S = 0) holding one dense ternary expert, written from the
    format text: blocked scales, then ceil(K/5) bytes per packed row."""
    def scales(rows, K):
        G = K // 64
        NC = (G + 7) // 8
        s = np.zeros((rows // 16) * NC * 128, np.uint16)
        for pr in range(rows):
            j, r = divmod(pr, 16)
            for grp in range(G):
                c, gl = divmod(grp, 8)
                s[(256 * NC * j + 256 * c) // 2 + 8 * r + gl] = scale_bits
        return s

    def gu_row(pr):                  # packed GU row -> gate or up source row
        b, jj = divmod(pr, 16)
        return (g if jj < 8 else u)[8 * b + jj % 8]

    gc = np.concatenate([_dense_row(gu_row(pr)) for pr in range(2 * I)])
    dc = np.concatenate([_dense_row(d[pr]) for pr in range(H_)])
    arrays = [scales(2 * I, H_), gc, None, scales(H_, I), dc, None]
    off, offs, blobs = 256 + 64, [], []
    for a in arrays:
        if a is None:
            offs.append(0)
            continue
        off = (off + 255) // 256 * 256
        offs.append(off)
        blobs.append((off, a.tobytes()))
        off += a.nbytes
    buf = bytearray(off)
    buf[0:32] = np.array([0x50454F4D, 2, H_, I, 1, 0, 64, 8], np.uint32).tobytes()
    buf[32:40] = np.uint64(off).tobytes()
    ent = np.zeros(8, np.uint64)
    ent[0] = DENSE
    ent[1:7] = offs
    buf[256:320] = ent.tobytes()
    for o, b in blobs:
        buf[o:o + len(b)] = b
    return np.frombuffer(bytes(buf), np.uint8)


@pytest.mark.parametrize("H_,I", [(128, 64), (576, 64), (64, 1024)])
def test_oracle_reads_hand_built_dense_buffer(H_, I):
    rng = np.random.default_rng(5)
    g, u = rng.integers(0, 3, size=(I, H_)), rng.integers(0, 3, size=(I, H_))
    d = rng.integers(0, 3, size=(H_, I))
    buf = _hand_dense(H_, I, g, u, d, np.float16(0.02).view(np.uint16))
    for which, ref, rows, K in ((0, g, I, H_), (1, u, I, H_), (2, d, H_, I)):
        f, codes, scales = oracle.unpack(buf, 0, which, rows, K)
        assert f == DENSE
        np.testing.assert_array_equal(codes, ref)
        assert np.all(scales == np.float16(0.02).view(np.uint16))


def test_oracle_rejects_a_dense_byte_above_242():
    H_, I = 64, 64
    z = np.zeros((I, H_), np.int64)
    buf = _hand_dense(H_, I, z, z, np.zeros((H_, I), np.int64), np.float16(0.02).view(np.uint16)).copy()
    gc = int(np.frombuffer(buf[256 + 16:256 + 24].tobytes(), np.uint64)[0])
    buf[gc + 3] = 243
    with pytest.raises(ValueError):
        oracle.unpack(buf, 0, 0, I, H_)


def _dense_fmt(layer):
    return np.where(layer.fmt == synth.FMT_TERNARY, DENSE, layer.fmt).astype(np.uint8)


@pytest.mark.parametrize("H_,I", [(128, 64), (320, 192), (1024, 128)])
def test_packer_dense_output_reads_back_and_is_smaller(H_, I):
    import bit_routed_expert_fp32_b200 as moe
    cfg = synth.micro(T=1, H=H_, E=6, k=2, I=I, S=1, formats="mixed", seed=H_ + I)
    layer = synth.Layer(cfg)
    fmt = _dense_fmt(layer)
    assert (fmt == DENSE).any()
    buf = moe.pack_layer(cfg, fmt, layer.expert)
    for e in range(cfg.E + cfg.S):
        mats = layer.expert(e)
        for which, name, rows, K in ((0, "gate", I, H_), (1, "up", I, H_), (2, "down", H_, I)):
            f, codes, scales = oracle.unpack(buf, e, which, rows, K)
            c, h, s = mats[name]
            assert f == fmt[e]
            np.testing.assert_array_equal(codes, codes_int(c, h))
            np.testing.assert_array_equal(scales, s)
    # code bytes of a dense expert: ceil(K/5) per row against K/4
    only_t = np.zeros(cfg.E + cfg.S, np.uint8)
    only_d = np.full(cfg.E + cfg.S, DENSE, np.uint8)
    saved = moe.moe_packed_size(cfg, only_t) - moe.moe_packed_size(cfg, only_d)
    per_expert = 2 * I * (H_ // 4 - (H_ + 4) // 5) + H_ * (I // 4 - (I + 4) // 5)
    assert abs(saved - (cfg.E + cfg.S) * per_expert) <= 2 * 256 * (cfg.E + cfg.S)    # alignment padding


@pytest.mark.gpu
def test_cache_expands_dense_experts_bit_exactly_and_the_layer_matches_the_oracle():
    import torch
    import bit_routed_expert_fp32_b200 as moe
    from bit_routed_expert_fp32_b200.cache import ExpertCache
    import dataclasses
    cfg = synth.micro(T=4, H=576, E=8, k=2, I=192, S=1, formats="ternary", seed=91)
    cfg = dataclasses.replace(cfg, shared_format=synth.FMT_TERNARY)       # every expert dense
    case = H.make_case(cfg)
    fmt_d = _dense_fmt(case.layer)
    dense = moe.pack_layer(cfg, fmt_d, case.layer.expert)
    plain = H.pack(case)                                        # the same experts, 2-bit ternary
    cache = ExpertCache(cfg, dense, n_slots=cfg.E + cfg.S)
    cache.ensure(range(cfg.E + cfg.S))
    torch.cuda.synchronize()
    dev = cache.buf.cpu().numpy()

    def entry(buf, e):
        return np.frombuffer(buf[256 + 64 * e:256 + 64 * e + 64].tobytes(), np.uint64)

    G_h, G_i = cfg.H // 64, cfg.I // 64
    sizes = [(2 * cfg.I // 16) * 256 * ((G_h + 7) // 8), 2 * cfg.I * cfg.H // 4,
             (cfg.H // 16) * 256 * ((G_i + 7) // 8), cfg.H * cfg.I // 4]
    assert (fmt_d == DENSE).all()
    for e in range(cfg.E + cfg.S):
        de, pe = entry(dev, e), entry(plain, e)
        assert int(de[0]) == synth.FMT_TERNARY and de[3] == 0 and de[6] == 0
        for slot, n in zip((1, 2, 4, 5), sizes):                 # gate/up scales, codes; down scales, codes
            np.testing.assert_array_equal(dev[int(de[slot]):int(de[slot]) + n], plain[int(pe[slot]):int(pe[slot]) + n])
    layer = moe.MoeLayer(cfg, plain, case.layer.router_w, case.layer.router_b, cfg.T)
    layer.packed = cache.buf
    rt, y = H.run_gpu(case, None, path=1, gpu_layer=layer)
    H.check_routing(case, rt)
    H.check_outputs(y, H.oracle_outputs(case, list(range(cfg.T))))


@pytest.mark.gpu
@pytest.mark.parametrize("T,path", [(1, 1), (1, 3), (4, 1), (6, 1), (24, 1), (96, 2)])
def test_forward_on_a_dense_buffer_is_reported(T, path):
    """The separate decode launches (1, 4 and 24 tokens), the fused decode kernel (1 token
    when asked for, 6 tokens by default) and prefill (96): MOE_DETAIL_FORMAT, nothing
    computed, the workspace still usable."""
    import torch
    import bit_routed_expert_fp32_b200 as moe
    cfg = synth.micro(T=T, H=256, E=8, k=2, I=128, S=1, formats="ternary", seed=92)   # every routed expert dense
    case = H.make_case(cfg)
    dense = moe.pack_layer(cfg, _dense_fmt(case.layer), case.layer.expert)
    layer = moe.MoeLayer(cfg, dense, case.layer.router_w, case.layer.router_b, T)
    x = moe.bf16_to_device(case.x)
    y = torch.zeros((T, cfg.H), dtype=torch.bfloat16, device="cuda")
    layer.route(x)
    layer.forward(x, y, path=path)
    st, det = moe.moe_get_error(layer.ws)
    assert moe.STATUS[st] == "MOE_ERR_DEVICE_CHECK" and det & 0xF00 == moe.DETAIL["FORMAT"], (st, hex(det))
    plain = moe.MoeLayer(cfg, H.pack(case), case.layer.router_w, case.layer.router_b, T)
    plain.ws = layer.ws                                          # the same workspace
    rt, y2 = H.run_gpu(case, None, path=path, gpu_layer=plain)
    H.check_outputs(y2, H.oracle_outputs(case, list(range(T))))
