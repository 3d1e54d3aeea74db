"""Parity of the CUDA path with the CPU oracle (needs a B200).

Routing (ids, counts, offsets, perm, inv_perm) must match bit-exactly and the gates
to 1e-5 relative; layer outputs must satisfy max |gpu - oracle| <= 2e-2 rms(oracle)
and relative Frobenius error <= 5e-3.  Inputs are regenerated token by token until
every adjacent gap among a token's k+1 largest logits is >= 1e-4 (fp64).
"""
import numpy as np
import pytest

import synth
from tests import harness as H

pytestmark = pytest.mark.gpu

PATHS = {"decode": 1, "prefill": 2, "fused": 3}


def _full_check(cfg, path, bias=None, router_w=None, T=None):
    case = H.make_case(cfg, bias=bias, router_w=router_w, T=T)
    packed = H.pack(case)
    rt, y = H.run_gpu(case, packed, path=path)
    H.check_routing(case, rt)
    ref = H.oracle_outputs(case, range(case.x.shape[0]))
    return H.check_outputs(y, ref), case, rt


@pytest.mark.parametrize("path", ["decode", "prefill"])
def test_tiny_layer_both_paths(path):
    """The 4-token tiny layer (hidden 256, 8 experts, top-2, all 2-bit)."""
    _full_check(synth.CONFIGS[1], PATHS[path])


@pytest.mark.parametrize("T", [1, 7, 63, 64, 65, 130])
def test_token_counts_around_the_path_switch(T):
    cfg = synth.micro(T=T, H=128, E=16, k=4, I=64, S=1, formats="mixed", seed=100 + T)
    _full_check(cfg, 0)


@pytest.mark.parametrize("kw", [
    dict(T=9, H=64, E=8, k=2, I=64, S=0, formats="q2"),            # K = 64: one group
    dict(T=33, H=192, E=32, k=8, I=128, S=1, formats="mixed"),     # odd group counts
    dict(T=20, H=256, E=256, k=8, I=64, S=1, formats="mixed"),     # full expert count
    dict(T=5, H=320, E=8, k=1, I=192, S=0, formats="q3"),          # k = 1, 3-bit only
    dict(T=17, H=128, E=12, k=12, I=64, S=1, formats="ternary"),   # k = E: every expert
    dict(T=3, H=128, E=40, k=16, I=64, S=0, formats="mixed"),      # k = 16
    dict(T=2, H=192, E=8, k=2, I=64, S=1, formats="mixed"),        # integer gate/up, partial chunk only
    dict(T=2, H=576, E=8, k=4, I=128, S=1, formats="ternary"),     # integer gate/up, full + partial chunk
])
def test_micro_shapes(kw):
    import bit_routed_expert_fp32_b200 as moe
    cfg = synth.micro(**kw, seed=sum(kw[k] for k in ("T", "H", "E", "k", "I")))
    _full_check(cfg, 1)
    if cfg.H % 128 == 0:                  # the prefill kernels tile hidden rows by 128
        _full_check(cfg, 2)
    else:
        with pytest.raises(moe.MoeError) as ei:
            _full_check(cfg, 2)
        assert ei.value.status == 2


def test_one_expert_takes_every_token_and_empty_experts():
    """A large bias on expert 3 makes every token pick it first; most experts stay
    empty (k = 2 of 64)."""
    cfg = synth.micro(T=96, H=128, E=64, k=2, I=64, S=1, formats="mixed", seed=7)
    bias = np.zeros(cfg.E, np.float32)
    bias[3] = 30.0
    bias[40:] = -30.0
    (_, _), case, rt = _full_check(cfg, 0, bias=bias)
    assert rt["counts"][3] == cfg.T
    assert (rt["counts"] == 0).sum() >= 1


def test_zero_tokens_is_a_no_op():
    import torch
    import bit_routed_expert_fp32_b200 as moe
    cfg = synth.micro(T=4, H=128, E=8, k=2, I=64, S=1)
    case = H.make_case(cfg)
    layer = moe.MoeLayer(cfg, H.pack(case), case.layer.router_w, None, 4)
    x = moe.bf16_to_device(case.x)
    y = torch.zeros((4, cfg.H), dtype=torch.bfloat16, device="cuda")
    layer.route(x, T=0)
    layer.forward(x, y, T=0)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y.view(torch.int16)) == 0


def test_repeated_calls_are_deterministic():
    """Counters are self-resetting: the same call twice gives identical bits."""
    import torch
    import bit_routed_expert_fp32_b200 as moe
    cfg = synth.micro(T=70, H=256, E=32, k=4, I=128, S=1, formats="mixed", seed=3)
    case = H.make_case(cfg)
    layer = moe.MoeLayer(cfg, H.pack(case), case.layer.router_w, None, cfg.T)
    x = moe.bf16_to_device(case.x)
    outs = []
    for path in (1, 1, 2, 2):
        y = layer(x, path=path)
        torch.cuda.synchronize()
        outs.append(moe.bf16_to_host(y))
    np.testing.assert_array_equal(outs[0], outs[1])
    np.testing.assert_array_equal(outs[2], outs[3])
    assert moe.moe_get_error(layer.ws)[0] == 0


# ---- full-size workloads (sampled outputs) -------------------------------------

@pytest.mark.parametrize("n", [2, 3, 4, 5])
def test_full_size_workloads(n):
    """The four full-size workloads in the launch configuration the benchmark times:
    routing checked for every token, outputs for a sample the oracle can afford."""
    import torch
    cfg = synth.CONFIGS[n]
    case = H.make_case(cfg)
    packed = H.pack(case)
    rt, y = H.run_gpu(case, packed, path=0)
    H.check_routing(case, rt)
    toks = list(range(cfg.T)) if cfg.T <= 16 else H.sample_tokens(case, 64, seed=n)
    ref = H.oracle_outputs(case, toks)
    H.check_outputs(y[toks], ref)
    if n == 5:
        assert case.counts.max() >= 8 * case.counts.mean() and (case.counts == 0).sum() >= 1
    del packed
    torch.cuda.empty_cache()


@pytest.mark.parametrize("n,layer_idx", [(3, 1), (3, 2), (3, 3), (5, 1), (5, 2), (5, 3)])
def test_full_size_cycled_layers(n, layer_idx):
    """The benchmark cycles four distinct layers for these two workloads (their own
    format shuffles, router weights and Zipf biases); layers 1-3 are checked like layer
    0 above."""
    import torch
    cfg = synth.CONFIGS[n]
    case = H.make_case(cfg, layer_idx=layer_idx)
    packed = H.pack(case)
    rt, y = H.run_gpu(case, packed, path=0)
    H.check_routing(case, rt)
    toks = list(range(cfg.T)) if cfg.T <= 16 else H.sample_tokens(case, 64, seed=10 * n + layer_idx)
    H.check_outputs(y[toks], H.oracle_outputs(case, toks))
    del packed
    torch.cuda.empty_cache()


def test_full_size_few_tokens_and_determinism():
    """The full-size decode layer at 1-4 and 16 tokens on one workspace (the fused decode
    kernel: one launch whose warps take work units at run time and wait on each other
    through counters): outputs of every token against the oracle, and two calls of one
    batch bit-identical (every sum is formed in a fixed order whichever warp ran it)."""
    import torch
    import bit_routed_expert_fp32_b200 as moe
    base = synth.CONFIGS[2]
    case1 = H.make_case(base, T=1)
    packed = H.pack(case1)
    layer = moe.MoeLayer(base, packed, case1.layer.router_w, case1.layer.router_b, 16)
    for T in (1, 2, 3, 4, 16):
        case = case1 if T == 1 else H.make_case(base, step=T, T=T)
        ref = H.oracle_outputs(case, list(range(T)))
        for path in (1, 3):              # the decode choice for T, and the fused decode kernel
            rt, y = H.run_gpu(case, None, path=path, gpu_layer=layer)
            H.check_routing(case, rt)
            H.check_outputs(y, ref)
            if T in (1, 16):
                _, y_again = H.run_gpu(case, None, path=path, gpu_layer=layer)
                np.testing.assert_array_equal(y, y_again)
    del layer, packed
    torch.cuda.empty_cache()


@pytest.mark.parametrize("T,shared_format,path", [(1, synth.FMT_TERNARY, "fused"), (2, synth.FMT_Q2, "fused"),
                                                  (4, synth.FMT_TERNARY, "fused"), (1, synth.FMT_TERNARY, "decode"),
                                                  (2, synth.FMT_Q2, "decode"), (1, synth.FMT_Q2, "decode")])
def test_few_token_integer_gate_up_full_chunks(T, shared_format, path):
    """The fused decode kernel runs gate/up and down of ternary and 2-bit experts on
    integer MMAs, the separate gate/up launch (one and two tokens) gate/up: hidden 1024
    gives whole 8-group chunks (the micro shapes above only reach the partial-chunk
    code), all routed experts ternary exercises the o = 1 offset, and a ternary or 2-bit
    shared expert takes the integer path's shared-expert rows (every other workload's
    shared expert is 3-bit, which stays on the bf16 path)."""
    import dataclasses
    cfg = synth.micro(T=T, H=1024, E=16, k=8, I=128, S=1, formats="ternary", seed=40 + T)
    cfg = dataclasses.replace(cfg, shared_format=shared_format)
    _full_check(cfg, PATHS[path])


@pytest.mark.parametrize("T,shared_format,path", [(1, synth.FMT_Q2, "fused"), (2, synth.FMT_TERNARY, "fused"),
                                                  (2, synth.FMT_Q2, "fused"), (2, synth.FMT_Q3, "fused"),
                                                  (5, synth.FMT_Q2, "fused"), (1, synth.FMT_Q2, "decode"),
                                                  (2, synth.FMT_TERNARY, "decode")])
def test_shared_gate_up_and_down_in_k_parts(T, shared_format, path):
    """Inter 2048 with eight experts a token: at one or two tokens the fused kernel
    splits every gate/up tile into K parts (their sums added in part order by the last
    part, which forms h in fp32 for the integer down pass or fp16 for the bf16 one) and
    every down tile into two; at five tokens the gate/up tiles of all experts exceed
    one wave of warps and only the shared expert's are split.  Shared expert in each
    format.  The separate launches at one and two tokens split gate/up in K parts too
    (the integer path's partial sums, added in part order by the K-part reduction)."""
    import dataclasses
    cfg = synth.micro(T=T, H=1024, E=16, k=8, I=2048, S=1, formats="mixed", seed=80 + T)
    cfg = dataclasses.replace(cfg, shared_format=shared_format)
    _full_check(cfg, PATHS[path])


@pytest.mark.parametrize("formats,T,path", [("q2", 1, "decode"), ("mixed", 12, "decode"), ("mixed", 96, "prefill")])
def test_fast_mode_copy(formats, T, path):
    """The fast mode's second buffer (every 3-bit expert replaced by its 2-bit copy)
    through both paths: the GPU reads the library's requantised and packed copy, the
    oracle the test harness's own numpy requantisation of the same layer."""
    import oracle
    import bit_routed_expert_fp32_b200 as moe
    cfg = synth.micro(T=T, H=256, E=16, k=4, I=128, S=1, formats=formats, seed=60 + T)
    case = H.make_case(cfg)
    fmt2, fn2 = moe.fast_copy(case.layer.fmt, case.layer.expert)
    packed = moe.pack_layer(cfg, fmt2, fn2)
    rt, y = H.run_gpu(case, packed, path=PATHS[path])
    H.check_routing(case, rt)
    ref = oracle.forward_tokens(H.FastLayer(case.layer), case.x, case.ids, case.gates, range(T))
    H.check_outputs(y, ref)
