"""The no-allocation decode entry point (moe_decode_static), checked against the
regular moe_route + moe_forward path on two calls in a row.

Some callers cannot allocate device memory (a plugin whose host framework's pool
allocator owns the GPU's memory, a serving loop that cannot afford a synchronising
cudaMalloc, code recording a CUDA graph); moe_decode_static serves them with a
scratch array the library holds itself.  This file is collected last on purpose.
"""
import numpy as np
import pytest

import synth
from tests import harness as H

pytestmark = pytest.mark.gpu


def test_static_scratch_matches_workspace_path_twice():
    import torch
    import bit_routed_expert_fp32_b200 as moe
    cfg = synth.micro(T=12, H=512, E=16, k=4, I=256, S=1, formats="mixed", seed=21)
    case = H.make_case(cfg)
    packed = H.pack(case)
    layer = moe.MoeLayer(cfg, packed, case.layer.router_w, case.layer.router_b, cfg.T)
    assert moe.moe_workspace_size(cfg, cfg.T) <= moe.STATIC_WS_BYTES
    for step in range(2):                      # two calls in a row, different tokens
        x_np = synth.tokens(cfg, 0, 100 + step)
        x = moe.bf16_to_device(x_np)
        y_ref = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
        layer.route(x)
        layer.forward(x, y_ref, path=moe.PATH_DECODE)
        rt = moe.alloc_routing(cfg, cfg.T)
        y = torch.full((cfg.T, cfg.H), float("nan"), dtype=torch.bfloat16, device="cuda")
        moe.moe_decode_static(cfg, cfg.T, x, layer.router_w, layer.router_b, layer.packed, rt, y)
        torch.cuda.synchronize()
        for name in ("topk_ids", "counts", "offsets", "perm", "inv_perm"):
            np.testing.assert_array_equal(rt[name].cpu().numpy(), layer.rt[name].cpu().numpy())
        # the same kernels on the same routing, every sum in a fixed order: bit for bit
        np.testing.assert_array_equal(moe.bf16_to_host(y), moe.bf16_to_host(y_ref))
        assert moe.moe_decode_static_get_error() == (0, 0)


def test_static_scratch_reports_a_device_check_and_recovers():
    """A packed buffer whose header does not describe the shape: the kernels record
    MOE_ERR_DEVICE_CHECK (detail HEADER) in the library's array, the error reader returns
    it once and clears it, and the next call with the right buffer is correct."""
    import torch
    import bit_routed_expert_fp32_b200 as moe
    cfg = synth.micro(T=4, H=256, E=8, k=2, I=128, S=1, formats="mixed", seed=22)
    case = H.make_case(cfg)
    packed = H.pack(case)
    layer = moe.MoeLayer(cfg, packed, case.layer.router_w, case.layer.router_b, cfg.T)
    bad = layer.packed.clone()
    bad[8:12] = 0                              # the header's H field
    x = moe.bf16_to_device(case.x)
    rt = moe.alloc_routing(cfg, cfg.T)
    y = torch.zeros((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
    moe.moe_decode_static(cfg, cfg.T, x, layer.router_w, layer.router_b, bad, rt, y)
    st, det = moe.moe_decode_static_get_error()
    assert moe.STATUS[st] == "MOE_ERR_DEVICE_CHECK" and det & 0xF00 == moe.DETAIL["HEADER"], (st, hex(det))
    assert moe.moe_decode_static_get_error() == (0, 0)           # read once, then cleared
    moe.moe_decode_static(cfg, cfg.T, x, layer.router_w, layer.router_b, layer.packed, rt, y)
    assert moe.moe_decode_static_get_error() == (0, 0)
    H.check_outputs(moe.bf16_to_host(y), H.oracle_outputs(case, list(range(cfg.T))))


def test_static_scratch_rejects_too_many_tokens():
    import torch
    import bit_routed_expert_fp32_b200 as moe
    cfg = synth.CONFIGS[2]
    T = 64                                     # needs about 19 MB of scratch
    assert moe.moe_workspace_size(cfg, T) > moe.STATIC_WS_BYTES
    dummy = torch.zeros(16, dtype=torch.uint8, device="cuda")
    rt = {n: dummy for n in ("topk_ids", "topk_w", "counts", "offsets", "perm", "inv_perm")}
    y = torch.full((T, cfg.H), float("nan"), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_decode_static(cfg, T, dummy, dummy, None, dummy, rt, y)
    assert ei.value.status == 3
    torch.cuda.synchronize()
    assert torch.isnan(y).all()                # rejected before anything was enqueued
