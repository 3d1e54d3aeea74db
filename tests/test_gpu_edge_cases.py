"""Edge cases of the CUDA path against the oracle and the device-side checks (needs a B200).

* Tokens with large outliers (one element per 64-wide group at 100x or 1000x the group's
  rms): the activation shape of DeepSeek-class models, and the case the integer path's
  per-group 12-bit grids and the prefill path's fp16 tokens are most exposed to.  Checked element by element against the oracle at the parity tolerances, on the
  full-size layer, at 1-4 tokens (integer gate/up), 16 tokens (decode) and 96 tokens
  (prefill).
* The range contract of moe_forward: a token element above the fp16 range, and tokens
  whose expert activations h overflow fp16, are reported as MOE_ERR_DEVICE_CHECK
  (detail RANGE) by both paths, without a fault; the context stays usable.
* moe_forward with a T other than the routed T is reported (detail ROUTED_T).
* The failure path of every expert kernel: a test-only wait on a barrier that nothing
  completes runs out (MOE_ERR_TIMEOUT, detail TEST_STALL); the kernels give up, drain
  their copies, free tensor memory and return; the next call on the same workspace is
  correct.
* Two host threads driving one device concurrently with separate workspaces.
"""
import threading

import numpy as np
import pytest

import synth
from tests import harness as H

pytestmark = pytest.mark.gpu

PATHS = {"decode": 1, "prefill": 2, "fused": 3}


def plant_outliers(factor, seed, every=1, base=1.0):
    """A transform for harness.make_case: every listed token is scaled by `base`, then in
    every `every`-th 64-wide group (from a seeded offset) one element (chosen by a seeded
    draw) becomes +-factor x the group's rms; rounded to bf16."""
    def fn(x, rows):
        for t in np.asarray(rows, dtype=np.int64):
            rng = np.random.default_rng([seed, int(t)])
            v = base * synth.bf16_bits_to_f32(x[t]).astype(np.float64).reshape(-1, 64)
            rms = np.sqrt(np.mean(v ** 2, axis=1))
            groups = np.arange(int(rng.integers(0, every)), v.shape[0], every)
            pos = rng.integers(0, 64, size=groups.size)
            sign = rng.choice([-1.0, 1.0], size=groups.size)
            v[groups, pos] = sign * factor * rms[groups]
            x[t] = synth.f32_to_bf16_bits(v.reshape(-1).astype(np.float32))
    return fn


@pytest.fixture(scope="module")
def mixed_layer():
    """The full-size mixed-format layer (77 ternary / 128 2-bit / 51 3-bit routed experts,
    3-bit shared), packed once for the outlier cases."""
    import torch
    import bit_routed_expert_fp32_b200 as moe
    cfg = synth.CONFIGS[3]
    case0 = H.make_case(cfg, T=1)
    packed = H.pack(case0)
    layer = moe.MoeLayer(cfg, packed, case0.layer.router_w, case0.layer.router_b, 96)
    yield cfg, layer
    del layer, packed
    torch.cuda.empty_cache()


# One element per group at 100x or 1000x the group's rms (in every group, or in every
# 16th group: a few massive channels, as in DeepSeek-class activations).  What matters to
# the per-group grids and the fp16 tokens is the outlier's size relative to its group, so
# the rest of the token is scaled down (rms 0.1, 0.02) to keep the expert activations h
# of these random weights inside the fp16 range the layer is defined for; with N(0,1)
# tokens, 1000x outliers push h past 65504, which moe_forward reports (tested below).
OUTLIERS = {"100x_every_group": (100.0, 1, 0.1), "1000x_every_group": (1000.0, 1, 0.02),
            "1000x_every_16th_group": (1000.0, 16, 0.1)}


@pytest.mark.parametrize("kind", sorted(OUTLIERS))
@pytest.mark.parametrize("T,path", [(1, "decode"), (1, "fused"), (2, "fused"), (4, "decode"), (16, "decode"),
                                    (16, "fused"), (96, "prefill")])
def test_outlier_tokens_full_size(mixed_layer, kind, T, path):
    cfg, layer = mixed_layer
    factor, every, base = OUTLIERS[kind]
    case = H.make_case(cfg, step=1000 + T, T=T, transform=plant_outliers(factor, seed=T, every=every, base=base))
    rt, y = H.run_gpu(case, None, path=PATHS[path], gpu_layer=layer)
    H.check_routing(case, rt)
    H.check_outputs(y, H.oracle_outputs(case, list(range(T))))


def test_outlier_tokens_all_q2_integer_path():
    """The default decode layer (every routed expert 2-bit): all eight routed experts of
    a one-token step on the integer paths, with a 1000x outlier in every group."""
    import torch
    cfg = synth.CONFIGS[2]
    case = H.make_case(cfg, T=1, transform=plant_outliers(1000.0, seed=7, every=1, base=0.02))
    packed = H.pack(case)
    for path in ("decode", "fused"):
        rt, y = H.run_gpu(case, packed, path=PATHS[path])
        H.check_routing(case, rt)
        H.check_outputs(y, H.oracle_outputs(case, [0]))
    del packed
    torch.cuda.empty_cache()


def _small_layer(T=8, seed=31, hidden=256):
    import bit_routed_expert_fp32_b200 as moe
    cfg = synth.micro(T=T, H=hidden, E=8, k=2, I=128, S=1, formats="mixed", seed=seed)
    case = H.make_case(cfg)
    packed = H.pack(case)
    return cfg, case, packed, moe.MoeLayer(cfg, packed, case.layer.router_w, case.layer.router_b, 96)


def _status(moe, ws):
    st, det = moe.moe_get_error(ws)
    return moe.STATUS[st], det


@pytest.mark.parametrize("path", ["decode", "prefill"])
def test_token_outside_fp16_range_is_reported(path):
    import torch
    import bit_routed_expert_fp32_b200 as moe
    cfg, case, packed, layer = _small_layer()
    x_np = case.x.copy()
    x_np[3, 10] = synth.f32_to_bf16_bits(np.array([1.0e5], np.float32))[0]
    x = moe.bf16_to_device(x_np)
    y = torch.zeros((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
    layer.route(x)
    layer.forward(x, y, path=PATHS[path])
    st, det = _status(moe, layer.ws)
    assert st == "MOE_ERR_DEVICE_CHECK" and det & 0xF00 == moe.DETAIL["RANGE"], (st, hex(det))
    # the context and the workspace stay usable
    rt, y2 = H.run_gpu(case, None, path=PATHS[path], gpu_layer=layer)
    H.check_routing(case, rt)
    H.check_outputs(y2, H.oracle_outputs(case, list(range(cfg.T))))


@pytest.mark.parametrize("path,T,hidden", [("decode", 8, 256), ("decode", 1, 256), ("decode", 1, 1024),
                                          ("decode", 2, 1024), ("decode", 24, 256), ("decode", 24, 1024),
                                          ("prefill", 8, 256)])
def test_activation_outside_fp16_range_is_reported(path, T, hidden):
    """Tokens inside the fp16 range whose activations h are not: every element 3000.  The
    decode cases reach every place h is formed: the fused kernel (8 tokens), the separate
    gate/up epilogue on the integer path (1 token, hidden 256: K in one part) and on the
    bf16 path (24 tokens), and the K-part reductions (hidden 1024: K in two parts; at one
    and two tokens the one that also forms the integer down pass's operands)."""
    import torch
    import bit_routed_expert_fp32_b200 as moe
    cfg, case, packed, layer = _small_layer(T=T, hidden=hidden)
    x_np = np.full((cfg.T, cfg.H), synth.f32_to_bf16_bits(np.array([3000.0], np.float32))[0], np.uint16)
    x = moe.bf16_to_device(x_np)
    y = torch.zeros((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
    layer.route(x)
    layer.forward(x, y, path=PATHS[path])
    st, det = _status(moe, layer.ws)
    assert st == "MOE_ERR_DEVICE_CHECK" and det & 0xF00 == moe.DETAIL["RANGE"] and det & 0xFF != 1, (st, hex(det))
    rt, y2 = H.run_gpu(case, None, path=PATHS[path], gpu_layer=layer)
    H.check_outputs(y2, H.oracle_outputs(case, list(range(cfg.T))))


@pytest.mark.parametrize("t_route,t_fwd,path", [(8, 5, "decode"), (40, 30, "decode"), (8, 5, "prefill")])
def test_forward_with_another_T_than_routed_is_reported(t_route, t_fwd, path):
    """Fused decode kernel (5 tokens), the decode kernels for more tokens (30), prefill."""
    import torch
    import bit_routed_expert_fp32_b200 as moe
    cfg, case, packed, layer = _small_layer()
    xr = moe.bf16_to_device(synth.tokens(cfg, 0, 900, t_route))
    y = torch.zeros((t_route, cfg.H), dtype=torch.bfloat16, device="cuda")
    layer.route(xr)
    layer.forward(xr, y, T=t_fwd, path=PATHS[path])
    st, det = _status(moe, layer.ws)
    assert st == "MOE_ERR_DEVICE_CHECK" and det & 0xF00 == moe.DETAIL["ROUTED_T"], (st, hex(det))
    rt, y2 = H.run_gpu(case, None, path=PATHS[path], gpu_layer=layer)
    H.check_outputs(y2, H.oracle_outputs(case, list(range(cfg.T))))


@pytest.mark.parametrize("T,path", [(1, "decode"), (1, "fused"), (8, "decode"), (24, "decode"), (96, "prefill")])
def test_wait_that_runs_out_is_reported_and_the_next_call_is_correct(T, path):
    """Each expert kernel waits (test-only, 20,000 SM cycles at most) on a barrier that
    nothing completes; the wait runs out, the kernel takes its give-up path and returns.
    Then the stall is switched off and the same workspace computes the layer correctly."""
    import torch
    import bit_routed_expert_fp32_b200 as moe
    cfg = synth.micro(T=T, H=256, E=16, k=4, I=128, S=1, formats="mixed", seed=50 + T)
    case = H.make_case(cfg)
    packed = H.pack(case)
    layer = moe.MoeLayer(cfg, packed, case.layer.router_w, case.layer.router_b, T)
    x = moe.bf16_to_device(case.x)
    y = torch.zeros((T, cfg.H), dtype=torch.bfloat16, device="cuda")
    moe.moe_workspace_set_test_stall(layer.ws, 20000)
    layer.route(x)
    layer.forward(x, y, path=PATHS[path])
    st, det = _status(moe, layer.ws)
    assert st == "MOE_ERR_TIMEOUT" and det & 0xF00 == moe.DETAIL["TEST_STALL"], (st, hex(det))
    moe.moe_workspace_set_test_stall(layer.ws, 0)
    moe.moe_workspace_init(layer.ws)
    for _ in range(2):
        rt, y2 = H.run_gpu(case, None, path=PATHS[path], gpu_layer=layer)
        H.check_routing(case, rt)
        H.check_outputs(y2, H.oracle_outputs(case, list(range(T))))


@pytest.mark.parametrize("kind,T", [("repeated", 1), ("repeated", 2), ("repeated", 24), ("outside", 2)])
def test_caller_routing_with_a_repeated_or_invalid_id_is_reported(kind, T):
    """moe_route_fixed with token 0's ids [1, 1, 3, 5] (the second 1 repeats the first
    slot's expert) or [1, 9, 3, 5] (9 >= E): MOE_DETAIL_RANGE with low byte 5 or 2, the
    pair counted nowhere (no expert gets more rows than tokens, which the decode kernels'
    integer path relies on), the forward runs, and the workspace then serves a normal
    call that matches the oracle."""
    import torch
    import bit_routed_expert_fp32_b200 as moe
    cfg, case, packed, layer = _small_layer(T=T, hidden=1024)
    ids = np.array([[(3 * t + j) % cfg.E for j in range(cfg.k)] for t in range(T)], np.int32)
    ids[0] = [1, 1] if kind == "repeated" else [1, 9]
    if cfg.k != 2:
        raise AssertionError("the case is written for top-2")
    x = moe.bf16_to_device(case.x)
    d_ids = torch.from_numpy(ids).cuda()
    gates = torch.full((T, cfg.k), 0.5, dtype=torch.float32, device="cuda")
    y = torch.zeros((T, cfg.H), dtype=torch.bfloat16, device="cuda")
    moe.moe_route_fixed(cfg, T, x, d_ids, gates, layer.rt, layer.ws)
    layer.forward(x, y, T=T, path=PATHS["decode"])
    st, det = _status(moe, layer.ws)
    assert st == "MOE_ERR_DEVICE_CHECK" and det == moe.DETAIL["RANGE"] | (5 if kind == "repeated" else 2), (st, hex(det))
    counts = layer.rt["counts"].cpu().numpy()
    want = np.bincount(ids[1:].ravel(), minlength=cfg.E)
    want[1] += 1                                     # token 0's first slot only
    np.testing.assert_array_equal(counts, want)
    assert counts.max() <= T
    rt, y2 = H.run_gpu(case, None, path=PATHS["decode"], gpu_layer=layer)
    H.check_routing(case, rt)
    H.check_outputs(y2, H.oracle_outputs(case, list(range(T))))


def test_two_host_threads_on_one_device():
    """Two host threads, each with its own workspace, routing buffers and stream, run the
    layer concurrently; every output equals the single-threaded result bit for bit."""
    import torch
    import bit_routed_expert_fp32_b200 as moe
    cfg = synth.micro(T=4, H=512, E=32, k=4, I=256, S=1, formats="mixed", seed=77)
    case = H.make_case(cfg)
    packed = H.pack(case)
    xs = [moe.bf16_to_device(synth.tokens(cfg, 0, 300 + i)) for i in range(2)]
    ref = []
    for i in range(2):
        lay = moe.MoeLayer(cfg, packed, case.layer.router_w, case.layer.router_b, cfg.T)
        ref.append(moe.bf16_to_host(lay(xs[i])))
    torch.cuda.synchronize()
    errors, outs = [], [[], []]

    def worker(i):
        try:
            torch.cuda.set_device(0)
            lay = moe.MoeLayer(cfg, packed, case.layer.router_w, case.layer.router_b, cfg.T)
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                for _ in range(20):
                    y = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
                    lay.route(xs[i], stream=s)
                    lay.forward(xs[i], y, path=moe.PATH_DECODE, stream=s)
                    outs[i].append(y)
            s.synchronize()
            st, det = moe.moe_get_error(lay.ws, s)
            assert st == 0, (st, det)
        except Exception as exc:          # noqa: BLE001 - reported below
            errors.append(exc)

    th = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not errors, errors
    for i in range(2):
        for y in outs[i]:
            np.testing.assert_array_equal(moe.bf16_to_host(y), ref[i])
