"""Test harness: builds a case (seeded inputs, oracle routing, packed layer) and
compares the CUDA path with the oracle.  Tests only."""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

import oracle
import synth

GAP = 1e-4          # minimum gap between adjacent top-(k+1) logits (fp64)
ATOL_RMS = 2e-2     # max |gpu - oracle| <= ATOL_RMS * rms(oracle)
FROB = 5e-3         # ||gpu - oracle||_F / ||oracle||_F <= FROB
GATE_RTOL = 1e-5


@dataclass
class Case:
    cfg: synth.LayerConfig
    layer: synth.Layer
    x: np.ndarray                    # uint16 bf16 bits [T][H]
    L: np.ndarray                    # fp64 logits without bias
    ids: np.ndarray
    gates: np.ndarray
    counts: np.ndarray
    offsets: np.ndarray
    perm: np.ndarray
    inv_perm: np.ndarray
    redrawn: int = 0
    extra: dict = field(default_factory=dict)


def make_case(cfg, layer_idx=0, step=0, T=None, bias=None, router_w=None, threads=None,
              transform=None) -> Case:
    """transform(x, rows) (optional) rewrites the listed token rows of x in place after
    they are drawn or redrawn (e.g. to plant outliers); the near-tie guard then runs on
    the rewritten tokens."""
    layer = synth.Layer(cfg, layer_idx)
    if router_w is not None:
        layer.router_w = router_w
    if bias is not None:
        layer.router_b = bias
    x = synth.tokens(cfg, layer_idx, step, T)
    if transform is not None:
        transform(x, np.arange(x.shape[0]))
    redrawn = 0
    for rnd in range(20):
        L = oracle.logits(x, layer.router_w, threads)
        bad = np.nonzero(oracle.topk_gaps(L, layer.router_b, cfg.k) < GAP)[0]
        if bad.size == 0:
            break
        redrawn += bad.size
        synth.redraw_tokens(cfg, x, bad, layer_idx, step, rnd)
        if transform is not None:
            transform(x, bad)
    else:
        raise RuntimeError("could not remove near-ties")
    ids, gates = oracle.select(L, layer.router_b, cfg.k)
    counts, offsets, perm, inv = oracle.permute(ids, cfg.E)
    return Case(cfg, layer, x, L, ids, gates, counts, offsets, perm, inv, redrawn)


class FastLayer:
    """The fast-mode copy of a synthetic layer for the oracle, requantised here in
    numpy (not by the library): every 3-bit expert's code c becomes c >> 1 (2-bit
    field = the old field's high bit, then the third bit) and its fp16 scales double;
    other experts are unchanged.  Same interface as synth.Layer for the oracle."""

    def __init__(self, layer):
        self.base = layer
        self.cfg = layer.cfg
        self.router_w, self.router_b = layer.router_w, layer.router_b
        self.fmt = np.where(layer.fmt == synth.FMT_Q3, synth.FMT_Q2, layer.fmt).astype(np.uint8)

    def expert(self, e):
        m = self.base.expert(e)
        if self.base.fmt[e] != synth.FMT_Q3:
            return m
        out = {}
        for name, (c, h, s) in m.items():
            bits = np.unpackbits(h, axis=1, bitorder="little")           # third bit of element k
            f = np.zeros_like(c)
            for i in range(4):
                lo = (c >> (2 * i)) & 3
                third = bits[:, i::4]
                f |= (((lo >> 1) | (third << 1)) << (2 * i)).astype(np.uint8)
            s2 = (s.view(np.float16).astype(np.float32) * 2).astype(np.float16).view(np.uint16)
            out[name] = (f, None, s2)
        return out


def pack(case: Case, threads=None) -> np.ndarray:
    import bit_routed_expert_fp32_b200 as moe
    cfg, layer = case.cfg, case.layer
    buf = np.zeros(moe.moe_packed_size(cfg, layer.fmt), dtype=np.uint8)

    def job(e):
        moe.moe_pack_experts(cfg, layer.fmt, e, [layer.expert(e)], buf)

    with ThreadPoolExecutor(threads or os.cpu_count() or 1) as ex:
        list(ex.map(job, range(cfg.E + cfg.S)))
    return buf


def run_gpu(case: Case, packed_host=None, path=0, gpu_layer=None, check_error=True):
    """Route + forward on the GPU; returns (routing dict of numpy arrays, y uint16)."""
    import torch
    import bit_routed_expert_fp32_b200 as moe
    cfg = case.cfg
    T = case.x.shape[0]
    if gpu_layer is None:
        gpu_layer = moe.MoeLayer(cfg, packed_host, case.layer.router_w, case.layer.router_b, T)
    x = moe.bf16_to_device(case.x)
    y = torch.full((T, cfg.H), float("nan"), dtype=torch.bfloat16, device="cuda")
    gpu_layer.route(x)
    gpu_layer.forward(x, y, path=path)
    torch.cuda.synchronize()
    if check_error:
        st, det = moe.moe_get_error(gpu_layer.ws)
        assert st == 0, f"device error {moe.STATUS[st]} detail {det:#x}"
    rt = {n: t.cpu().numpy() for n, t in gpu_layer.rt.items()}
    return rt, moe.bf16_to_host(y)


def check_routing(case: Case, rt: dict):
    cfg = case.cfg
    T = case.x.shape[0]
    np.testing.assert_array_equal(rt["topk_ids"][:T], case.ids)
    np.testing.assert_array_equal(rt["counts"], case.counts)
    np.testing.assert_array_equal(rt["offsets"], case.offsets)
    np.testing.assert_array_equal(rt["perm"][:T * cfg.k], case.perm)
    np.testing.assert_array_equal(rt["inv_perm"][:T * cfg.k], case.inv_perm)
    # The router's logits are fp32 values (the layer's router is fp32), so a gate
    # g_j = exp(L_j - L_max) / sum is exact only up to the rounding of L_j and L_max to
    # fp32: |dg / g| <= ulp(max |L|) beyond the fixed 1e-5.  For N(0,1) tokens max |L| is
    # a few units (ulp ~ 5e-7); tokens with 1000x outliers reach hundreds (ulp ~ 6e-5).
    Lb = case.L + (0.0 if case.layer.router_b is None else case.layer.router_b.astype(np.float64))
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(Lb).max(axis=1), 1e-30))) - 23)
    rtol = GATE_RTOL + ulp[:, None]
    g = rt["topk_w"][:T].astype(np.float64)
    bad = np.abs(g - case.gates) > rtol * np.abs(case.gates)
    assert not bad.any(), (f"gates differ beyond 1e-5 + ulp(max |L|) at {np.argwhere(bad)[:5].tolist()}: "
                           f"{g[bad][:5]} vs {case.gates[bad][:5]}")


def oracle_outputs(case: Case, tokens, threads=None) -> np.ndarray:
    return oracle.forward_tokens(case.layer, case.x, case.ids, case.gates, tokens, threads)


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 values (8 significant bits) at |v|: the error of rounding
    the exact value to the output format."""
    a = np.maximum(np.abs(v), np.finfo(np.float32).tiny)
    return np.exp2(np.floor(np.log2(a)) - 8)


def check_outputs(y_gpu_bits: np.ndarray, y_ref: np.ndarray):
    """The parity bar.  The layer's output is bf16, so the max-abs bound applies to the
    error beyond the rounding of the exact value to bf16 (half an ulp at |y|): an output
    of 8x rms has a rounding error of ~2 % of rms by itself, more than the bound, even
    from exact arithmetic.  The Frobenius bound applies to the whole error."""
    y = synth.bf16_bits_to_f32(y_gpu_bits).astype(np.float64)
    assert np.all(np.isfinite(y))
    diff = y - y_ref
    rms = np.sqrt(np.mean(y_ref ** 2))
    excess = np.maximum(np.abs(diff) - bf16_half_ulp(y_ref), 0.0)
    max_err = excess.max()
    frob = np.linalg.norm(diff) / np.linalg.norm(y_ref)
    assert max_err <= ATOL_RMS * rms, (f"max |err| beyond bf16 rounding {max_err:.3e} > {ATOL_RMS} * rms {rms:.3e} "
                                       f"(raw max |err| {np.abs(diff).max():.3e})")
    assert frob <= FROB, f"relative Frobenius error {frob:.3e} > {FROB}"
    return max_err / rms, frob


def sample_tokens(case: Case, n_random: int, seed: int = 0) -> list:
    """Tokens whose outputs the oracle computes at full size: the first and last token
    of the permuted ranges of 32 experts spread over the ids, tokens at (up to 32)
    64-row tile boundaries of the hottest expert, and n_random uniform draws."""
    cfg = case.cfg
    T = case.x.shape[0]
    pick = set()
    for e in range(0, cfg.E, max(1, cfg.E // 32)):           # 32 experts spread over the ids
        lo, hi = int(case.offsets[e]), int(case.offsets[e + 1])
        if hi > lo:
            pick.add(int(case.perm[lo]) // cfg.k)
            pick.add(int(case.perm[hi - 1]) // cfg.k)
    hot = int(np.argmax(case.counts))
    lo, hi = int(case.offsets[hot]), int(case.offsets[hot + 1])
    step = max(64, ((hi - lo) // 32 + 63) // 64 * 64)         # at most ~32 tile boundaries
    for r in range(lo, hi, step):
        pick.add(int(case.perm[r]) // cfg.k)
    rng = np.random.default_rng(seed)
    pick.update(int(t) for t in rng.choice(T, size=min(n_random, T), replace=False))
    return sorted(pick)
