"""Seeded synthetic inputs for the routed-MoE layer.

This module is shared by the CUDA path (tests, benchmark) and the CPU oracle, and
holds none of the layer's arithmetic: it only draws random numbers and stores
them in the plain interchange form that both sides read.

Interchange form of one expert matrix W[rows][K] (K a multiple of 64):
  codes  uint8  [rows][K/4]  2-bit field of element k at bits 2*(k%4) of byte k/4
                             (for 3-bit experts: the low two bits of the code)
  hi     uint8  [rows][K/8]  3-bit experts only: bit 2 of the code of element k at
                             bit k%8 of byte k/8; None otherwise
  scales uint16 [rows][K/64] fp16 bit patterns, one scale per 64 weights along K
An expert is (gate [I][H], up [I][H], down [H][I]).

Recipe (every stream is numpy PCG64 seeded by SeedSequence(seed, spawn_key)):
  router weight  N(0, 0.02) float32 [E][H]                 key (layer, 1)
  Zipf bias      b_e = -beta * s * ln(rank_e), rank a seeded permutation of 1..E
                                                            key (layer, 2)
  formats        "q2": all routed experts 2-bit; "mixed": round(0.3E) ternary,
                 round(0.2E) 3-bit, the rest 2-bit, placed by a seeded shuffle;
                 shared experts use cfg.shared_format        key (layer, 0)
  expert e       codes uniform over the format's range, ternary with
                 P(code 0) = P(code 2) = 0.3, P(code 1) = 0.4 (value 0);
                 scales U(0.01, 0.05) float32 rounded to fp16 (nearest even)
                                                            key (layer, 3, e)
  tokens         N(0, 1) float32 rounded to bf16 (nearest even)  key (layer, 4, step)
  token redraw   fresh N(0,1) rows for listed tokens         key (layer, 5, step, round)
"""
from __future__ import annotations

import numpy as np

from .configs import (CONFIGS, FMT_Q2, FMT_Q3, FMT_TERNARY, GROUP, ZIPF_BETA,
                      LayerConfig)


def _rng(cfg: LayerConfig, *key: int) -> np.random.Generator:
    ss = np.random.SeedSequence(entropy=cfg.seed, spawn_key=tuple(int(k) for k in key))
    return np.random.Generator(np.random.PCG64(ss))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> 16) & 1
    return ((u + np.uint32(0x7FFF) + lsb) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def expert_formats(cfg: LayerConfig, layer: int = 0) -> np.ndarray:
    """uint8 [E+S] format id per expert table (routed experts first, then shared)."""
    E = cfg.E
    if cfg.formats == "q2":
        routed = np.full(E, FMT_Q2, dtype=np.uint8)
    elif cfg.formats == "mixed":
        n_t = int(round(0.3 * E))
        n_3 = int(round(0.2 * E))
        routed = np.array([FMT_TERNARY] * n_t + [FMT_Q3] * n_3 + [FMT_Q2] * (E - n_t - n_3),
                          dtype=np.uint8)
        _rng(cfg, layer, 0).shuffle(routed)
    elif cfg.formats in ("ternary", "q3"):
        routed = np.full(E, FMT_TERNARY if cfg.formats == "ternary" else FMT_Q3, dtype=np.uint8)
    else:
        raise ValueError(cfg.formats)
    shared = np.full(cfg.S, cfg.shared_format, dtype=np.uint8)
    return np.concatenate([routed, shared])


def router_weight(cfg: LayerConfig, layer: int = 0) -> np.ndarray:
    return _rng(cfg, layer, 1).normal(0.0, 0.02, size=(cfg.E, cfg.H)).astype(np.float32)


def router_bias(cfg: LayerConfig, layer: int = 0, beta: float | None = None):
    """float32 [E] Zipf-shaped logit bias, or None for an unbiased router."""
    if cfg.zipf is None:
        return None
    if beta is None:
        beta = ZIPF_BETA[cfg.zipf]
    rank = _rng(cfg, layer, 2).permutation(cfg.E) + 1
    return (-beta * cfg.zipf * np.log(rank.astype(np.float64))).astype(np.float32)


def _codes(rng: np.random.Generator, fmt: int, rows: int, K: int):
    nbytes = rows * K // 4
    if fmt == FMT_TERNARY:
        u = np.frombuffer(rng.bytes(2 * rows * K), dtype=np.uint16)    # uniform 0..65535
        c = (u >= 19661).view(np.uint8) + (u >= 45875).view(np.uint8)   # P = .3/.4/.3
        c = c.reshape(rows, K // 4, 4)
        codes = c[..., 0] | (c[..., 1] << 2)
        codes |= c[..., 2] << 4
        codes |= c[..., 3] << 6
        return np.ascontiguousarray(codes, dtype=np.uint8), None
    codes = np.frombuffer(rng.bytes(nbytes), dtype=np.uint8).reshape(rows, K // 4).copy()
    hi = None
    if fmt == FMT_Q3:
        hi = np.frombuffer(rng.bytes(rows * K // 8), dtype=np.uint8).reshape(rows, K // 8).copy()
    return codes, hi


def _scales(rng: np.random.Generator, rows: int, K: int) -> np.ndarray:
    s = rng.uniform(0.01, 0.05, size=(rows, K // GROUP)).astype(np.float32)
    return s.astype(np.float16).view(np.uint16)


def expert(cfg: LayerConfig, e: int, fmt: int, layer: int = 0) -> dict:
    """Matrices of expert table e: {'gate','up','down'} -> (codes, hi, scales)."""
    rng = _rng(cfg, layer, 3, e)
    out = {}
    for name, rows, K in (("gate", cfg.I, cfg.H), ("up", cfg.I, cfg.H), ("down", cfg.H, cfg.I)):
        codes, hi = _codes(rng, fmt, rows, K)
        out[name] = (codes, hi, _scales(rng, rows, K))
    return out


def tokens(cfg: LayerConfig, layer: int = 0, step: int = 0, T: int | None = None) -> np.ndarray:
    """bf16 bit patterns uint16 [T][H], N(0,1)."""
    T = cfg.T if T is None else T
    return f32_to_bf16_bits(_rng(cfg, layer, 4, step).standard_normal((T, cfg.H), dtype=np.float32))


def redraw_tokens(cfg: LayerConfig, x: np.ndarray, idx, layer: int = 0, step: int = 0,
                  round_: int = 0) -> np.ndarray:
    """Replace rows idx of x by fresh N(0,1) draws (used to reject near-tie tokens)."""
    idx = np.asarray(idx, dtype=np.int64)
    if idx.size:
        rng = _rng(cfg, layer, 5, step, round_)
        x[idx] = f32_to_bf16_bits(rng.standard_normal((idx.size, cfg.H), dtype=np.float32))
    return x


def calibration_tokens(cfg: LayerConfig, n: int = 4096) -> np.ndarray:
    return f32_to_bf16_bits(_rng(cfg, 0, 6).standard_normal((n, cfg.H), dtype=np.float32))


class Layer:
    """One synthetic layer; experts are drawn on demand (each from its own stream)."""

    def __init__(self, cfg: LayerConfig, layer: int = 0):
        self.cfg = cfg
        self.layer = layer
        self.fmt = expert_formats(cfg, layer)
        self.router_w = router_weight(cfg, layer)
        self.router_b = router_bias(cfg, layer)

    def expert(self, e: int) -> dict:
        return expert(self.cfg, e, int(self.fmt[e]), self.layer)


def config(n: int) -> LayerConfig:
    return CONFIGS[n]
