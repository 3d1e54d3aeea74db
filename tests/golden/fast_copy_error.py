"""How far the fast-mode copy (every 3-bit expert replaced by its 2-bit copy: codes
c >> 1, fp16 scales doubled) moves the layer's output, by the CPU oracle in fp64.

Writes tests/golden/fast_copy_error.json.  Uses only the oracle, the synthetic input
generators and the test harness's own numpy requantisation (tests/harness.py,
FastLayer); nothing from the library.

Two layer mixes, 64 tokens each, hidden 512, 32 experts, top-8, ffn 256, one 3-bit
shared expert: routed experts all 2-bit (the default decode workload's mix) and the
mixed ternary / 2-bit / 3-bit routed experts.  Reported per mix: relative Frobenius
norm of y_fast - y over the tokens, max |y_fast - y| over rms(y), the share of the
whole layer's packed bytes saved (not the bytes a decode step reads), and the same
change with the shared expert left out (routed experts only).  With one scale
distribution for every format, a 3-bit expert's output is several times a 2-bit
one's (weights up to 3.5 s against 1.5 s, through two matrix products and SwiGLU), so
the 3-bit experts dominate y and the change reflects their 1-bit loss.

Run:  python tests/golden/fast_copy_error.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402
from tests import harness as H  # noqa: E402


def packed_bytes(cfg, fmt):
    """Codes + third bits + scales of all experts (the format's bytes per weight)."""
    per_w = {synth.FMT_TERNARY: 2.25, synth.FMT_Q2: 2.25, synth.FMT_Q3: 3.25}
    return sum(per_w[int(f)] for f in fmt) * 3 * cfg.H * cfg.I / 8


def main():
    out = {}
    for formats in ("q2", "mixed"):
        cfg = synth.micro(T=64, H=512, E=32, k=8, I=256, S=1, formats=formats, seed=77)
        case = H.make_case(cfg)
        fast = H.FastLayer(case.layer)
        toks = range(cfg.T)
        y0 = oracle.forward_tokens(case.layer, case.x, case.ids, case.gates, toks)
        y1 = oracle.forward_tokens(fast, case.x, case.ids, case.gates, toks)
        d = y1 - y0
        rms = float(np.sqrt(np.mean(y0 ** 2)))
        # routed part only: the same layers without a shared expert
        cfg0 = synth.micro(T=64, H=512, E=32, k=8, I=256, S=0, formats=formats, seed=77)
        lay0 = synth.Layer(cfg0)
        r0 = oracle.forward_tokens(lay0, case.x, case.ids, case.gates, toks)
        r1 = oracle.forward_tokens(H.FastLayer(lay0), case.x, case.ids, case.gates, toks)
        out[formats] = {
            "three_bit_experts": int((case.layer.fmt == synth.FMT_Q3).sum()),
            "rel_frobenius": float(np.linalg.norm(d) / np.linalg.norm(y0)),
            "max_over_rms": float(np.abs(d).max() / rms),
            "layer_bytes_saved": 1.0 - packed_bytes(cfg, fast.fmt) / packed_bytes(cfg, case.layer.fmt),
            "routed_only_rel_frobenius": float(np.linalg.norm(r1 - r0) / np.linalg.norm(r0)),
        }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "fast_copy_error.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out, indent=1))


if __name__ == "__main__":
    main()
