"""Seeded synthetic inputs shared by the CUDA path and the oracle (no layer arithmetic)."""
from .configs import (CONFIGS, FMT_NAMES, FMT_Q2, FMT_Q3, FMT_TERNARY, GROUP, LayerConfig,
                      micro)
from .gen import (Layer, bf16_bits_to_f32, calibration_tokens, expert, expert_formats,
                  f32_to_bf16_bits, redraw_tokens, router_bias, router_weight, tokens)
