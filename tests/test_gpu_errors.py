"""Device-side error reporting, without any GPU fault: a packed buffer whose header
does not match the layer is detected by the FFN kernels, which return early and
record MOE_ERR_DEVICE_CHECK (detail: header) in the workspace's error word; the host
reads it with moe_get_error and the context stays usable."""
import numpy as np
import pytest

import harness as H
import synth

pytestmark = pytest.mark.gpu

DET_HEADER = 0x400


@pytest.mark.parametrize("path", [1, 2])          # decode, prefill
def test_corrupt_header_is_reported(path):
    import torch
    import bit_routed_expert_fp32_b200 as moe
    cfg = synth.micro(T=8, H=256, E=8, k=2, I=128, S=1, seed=21)
    case = H.make_case(cfg)
    packed = H.pack(case)
    lay = moe.MoeLayer(cfg, packed, case.layer.router_w, case.layer.router_b, cfg.T)
    lay.packed[0:4] = 0                            # magic word gone (device copy only)
    x = moe.bf16_to_device(case.x)
    y = torch.zeros((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
    lay.route(x)
    lay.forward(x, y, path=path)                   # launches succeed; the kernels detect it
    torch.cuda.synchronize()
    st, det = moe.moe_get_error(lay.ws)
    assert moe.STATUS[st] == "MOE_ERR_DEVICE_CHECK" and det == DET_HEADER
    # the context is still usable: the intact buffer runs cleanly on a fresh layer
    rt, y2 = H.run_gpu(case, packed, path=path)
    H.check_routing(case, rt)
    H.check_outputs(y2, H.oracle_outputs(case, list(range(cfg.T))))
