"""Host-tiered experts (bit_routed_expert_fp32_b200/cache.py, moe_cache_* in moe.h).

CPU: the slot plan (free slots first, then the least recently used expert that is
neither needed now nor pinned; the needed experts become the most recent) and the
library's host-side checks of the cache calls.  GPU: a layer run from a cache smaller
than the layer, step after step with evictions, gives bit for bit the output of the
same layer resident in HBM (the same kernels read the same bytes), with loads on the
compute stream and with loads prefetched on a copy stream."""
import ctypes
from collections import OrderedDict

import numpy as np
import pytest

import synth
from bit_routed_expert_fp32_b200.cache import slot_plan
from tests import harness as H


def test_slot_plan_free_slots_then_lru():
    res = OrderedDict()
    assert slot_plan(res, 4, [5, 6]) == [(5, 0), (6, 1)]
    assert slot_plan(res, 4, [6, 7], pinned=[9]) == [(7, 2)]
    assert list(res) == [5, 6, 7]                      # 6 used again, 7 new: most recent
    assert slot_plan(res, 4, [8, 9]) == [(8, 3), (9, 0)]   # 5 is the least recently used
    assert list(res) == [6, 7, 8, 9]
    # pinned experts are never evicted: with 6, 7, 8 pinned, 9 (slot 0) makes room
    assert slot_plan(res, 4, [1], pinned=[6, 7, 8]) == [(1, 0)]
    res2 = OrderedDict([(10, 0), (11, 1)])
    assert slot_plan(res2, 2, [12], pinned=[10]) == [(12, 1)]
    with pytest.raises(ValueError):
        slot_plan(OrderedDict(), 2, [1, 2, 3])


def test_cache_calls_check_their_arguments_without_a_gpu():
    import bit_routed_expert_fp32_b200 as moe
    cfg = synth.micro(T=4, H=128, E=8, k=2, I=64, S=1, formats="mixed", seed=3)
    layer = synth.Layer(cfg)
    buf = moe.pack_layer(cfg, layer.fmt, layer.expert)
    L = moe.lib()
    sh = moe.Shape(cfg.H, cfg.I, cfg.E, cfg.k, cfg.S)
    sz = ctypes.c_size_t(0)
    assert L.moe_cache_size(ctypes.byref(sh), buf.ctypes.data, 4, ctypes.byref(sz)) == 0
    # table + 4 slots, each at least the largest expert's bytes
    per_expert = (buf.nbytes - 1024) / (cfg.E + cfg.S)
    assert sz.value >= 4 * per_expert
    assert L.moe_cache_size(ctypes.byref(sh), buf.ctypes.data, 0, ctypes.byref(sz)) == 1
    bad = moe.Shape(cfg.H, cfg.I, cfg.E + 1, cfg.k, cfg.S)            # header does not match
    assert L.moe_cache_size(ctypes.byref(bad), buf.ctypes.data, 4, ctypes.byref(sz)) == 1
    fake = ctypes.c_void_p(0x1000)
    ex = np.array([cfg.E + cfg.S], np.int32)                            # expert index out of range
    sl = np.array([0], np.int32)
    assert L.moe_cache_load(ctypes.byref(sh), buf.ctypes.data, 4, fake, 1 << 30, ex.ctypes.data, sl.ctypes.data,
                            1, None) == 1


@pytest.mark.gpu
@pytest.mark.parametrize("prefetch", [False, True])
def test_layer_runs_from_a_cache_smaller_than_the_layer(prefetch):
    import torch
    import bit_routed_expert_fp32_b200 as moe
    from bit_routed_expert_fp32_b200.cache import ExpertCache
    cfg = synth.micro(T=4, H=256, E=16, k=2, I=128, S=1, formats="mixed", seed=61)
    case = H.make_case(cfg)
    packed = H.pack(case)
    resident = moe.MoeLayer(cfg, packed, case.layer.router_w, case.layer.router_b, cfg.T)
    cached = moe.MoeLayer(cfg, packed, case.layer.router_w, case.layer.router_b, cfg.T)
    cache = ExpertCache(cfg, packed, n_slots=10)               # 10 slots for 17 experts (a step needs <= 9)
    cached.packed = cache.buf                                   # the forward reads the cache
    copy = torch.cuda.Stream()
    for step in range(12):
        x = moe.bf16_to_device(synth.tokens(cfg, 0, 50 + step))
        y_ref = resident(x)
        cached.route(x)
        ids = np.unique(cached.rt["topk_ids"][:cfg.T].cpu().numpy())      # the step's experts
        if prefetch:
            ev = cache.prefetch(ids, copy)
            torch.cuda.current_stream().wait_event(ev)
        else:
            cache.ensure(ids)
        y = torch.empty_like(y_ref)
        cached.forward(x, y)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(moe.bf16_to_host(y), moe.bf16_to_host(y_ref))
    assert cache.loads > cache.n_slots                          # slots were reused
    assert moe.moe_get_error(cached.ws)[0] == 0
