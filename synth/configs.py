"""The five synthetic workloads of the routed-MoE layer, as named presets.

Nothing here computes any part of the layer; it only fixes sizes, formats and
seeds.  The shapes are DeepSeek-style: the pages name the model
("DeepSeek-V4.1-Flash 552B", yoney.dev news item, opening paragraph; shadowgraph.io
README, title line) and the expert mix ("GSQ mixed ternary / 2-bit / 3-bit",
ossradar.top README, "Get a model"), but give no layer sizes, so the sizes are the
plain DeepSeek-V3-class routed layer: hidden 7168, 256 routed experts, top-8,
one shared expert, expert FFN width 2048.

Prefill token counts (8192, 16384) stand in for the pages' fresh 6K-17K-token
prompts processed in sweeps of about 6-9K tokens (shadowgraph.io README, the
paragraph under the model table).
"""
from __future__ import annotations

from dataclasses import dataclass

# format ids: identical numbering to the packed format's per-expert format byte
FMT_TERNARY = 0   # codes {0,1,2} -> {-1,0,+1} x scale
FMT_Q2 = 1        # codes 0..3   -> {-1.5,-0.5,0.5,1.5} x scale
FMT_Q3 = 2        # codes 0..7   -> -3.5..3.5 x scale
FMT_NAMES = {FMT_TERNARY: "ternary", FMT_Q2: "q2", FMT_Q3: "q3"}

GROUP = 64        # one fp16 scale per 64 weights along K


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int              # tokens per step
    H: int              # hidden size
    E: int              # routed experts
    k: int              # experts per token
    I: int              # expert FFN width
    S: int              # shared experts (0 or 1)
    formats: str        # "q2": every routed expert 2-bit; "mixed": 77 ternary / 128 q2 / 51 q3
    shared_format: int  # format of the shared expert (ignored when S == 0)
    zipf: float | None  # expert popularity exponent, None = unbiased router
    seed: int
    layers: int         # distinct layers cycled by the benchmark
    steps: int          # timed steps the workload description asks for

    @property
    def n_tables(self) -> int:
        return self.E + self.S


# Zipf bias strength beta for b_e = -beta * s * ln(rank_e).  Written by
# tests/golden/calibrate_zipf.py, which routes a 4096-token calibration draw with
# the oracle only and fits the log-count / log-rank slope to -s; for s = 1.2 beta is
# then raised until the 16384-token draw has its hottest expert at >= 8x the mean
# count and at least one empty expert.  See tests/golden/zipf_beta.json.
ZIPF_BETA = {1.1: 0.7848, 1.2: 1.2684}


CONFIGS: dict[int, LayerConfig] = {
    1: LayerConfig("tiny_T4_H256_E8_k2_I128", T=4, H=256, E=8, k=2, I=128, S=0,
                   formats="q2", shared_format=FMT_Q3, zipf=None, seed=0, layers=1, steps=1),
    2: LayerConfig("decode_T1_H7168_E256_k8_I2048_S1", T=1, H=7168, E=256, k=8, I=2048, S=1,
                   formats="q2", shared_format=FMT_Q3, zipf=None, seed=2, layers=1, steps=100),
    3: LayerConfig("decode_T16_mixed_zipf1.1", T=16, H=7168, E=256, k=8, I=2048, S=1,
                   formats="mixed", shared_format=FMT_Q3, zipf=1.1, seed=3, layers=4, steps=100),
    4: LayerConfig("prefill_T8192_mixed_uniform", T=8192, H=7168, E=256, k=8, I=2048, S=1,
                   formats="mixed", shared_format=FMT_Q3, zipf=None, seed=4, layers=1, steps=20),
    5: LayerConfig("prefill_T16384_mixed_zipf1.2", T=16384, H=7168, E=256, k=8, I=2048, S=1,
                   formats="mixed", shared_format=FMT_Q3, zipf=1.2, seed=5, layers=4, steps=10),
}


def micro(T=8, H=128, E=8, k=2, I=64, S=1, formats="mixed", zipf=None, seed=11) -> LayerConfig:
    """A small layer for unit tests (any multiple-of-64 H and I)."""
    return LayerConfig(f"micro_T{T}_H{H}_E{E}_k{k}_I{I}_S{S}", T=T, H=H, E=E, k=k, I=I, S=S,
                       formats=formats, shared_format=FMT_Q3, zipf=zipf, seed=seed, layers=1,
                       steps=1)
