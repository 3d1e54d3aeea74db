"""Calibrate the Zipf bias strength beta of the skewed-routing workloads.

Writes tests/golden/zipf_beta.json; the values are copied into synth/configs.py
(ZIPF_BETA).  Uses only the CPU oracle's routing (fp64 logits, softmax top-k).

Procedure, for each exponent s (1.1: the 16-token decode workload, 1.2: the
16384-token prefill workload):
  1. Route the 4096-token calibration draw of layer 0 with bias
     b_e = -beta * s * ln(rank_e) and count tokens per expert.
  2. Least-squares fit of ln(count) against ln(rank) over experts with a nonzero
     count; bisect beta until the slope equals -s.
  3. For s = 1.2 only: route the workload's own 16384 tokens of layer 0 and raise
     beta in steps of 5 % until the hottest expert's count is at least 8x the mean
     and at least one expert receives no token.

Run:  python tests/golden/calibrate_zipf.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402


def counts_for(L, cfg, beta):
    b = synth.router_bias(cfg, 0, beta=beta)
    ids, _ = oracle.select(L, b, cfg.k)
    return np.bincount(ids.ravel(), minlength=cfg.E), b


def slope(cfg, L, beta):
    c, _ = counts_for(L, cfg, beta)
    rank = np.empty(cfg.E, np.int64)
    rank_perm = np.random.Generator(np.random.PCG64(np.random.SeedSequence(
        entropy=cfg.seed, spawn_key=(0, 2)))).permutation(cfg.E) + 1
    rank[:] = rank_perm
    m = c > 0
    A = np.stack([np.log(rank[m]), np.ones(m.sum())], axis=1)
    sl, _ = np.linalg.lstsq(A, np.log(c[m]), rcond=None)[0]
    return sl, c


def main():
    out = {}
    for n in (3, 5):
        cfg = synth.CONFIGS[n]
        xc = synth.calibration_tokens(cfg, 4096)
        Lc = oracle.logits(xc, synth.router_weight(cfg, 0))
        lo, hi = 0.0, 4.0
        for _ in range(40):
            mid = 0.5 * (lo + hi)
            sl, _ = slope(cfg, Lc, mid)
            if sl > -cfg.zipf:
                lo = mid
            else:
                hi = mid
        beta = round(0.5 * (lo + hi), 4)
        sl, c = slope(cfg, Lc, beta)
        rec = {"s": cfg.zipf, "beta_fit": beta, "slope": float(sl),
               "calib_max_over_mean": float(c.max() / c.mean()), "calib_empty": int((c == 0).sum())}
        if n == 5:
            x = synth.tokens(cfg)
            L = oracle.logits(x, synth.router_weight(cfg, 0))
            b = beta
            while True:
                cnt, _ = counts_for(L, cfg, b)
                if cnt.max() >= 8 * cnt.mean() and (cnt == 0).sum() >= 1:
                    break
                b = round(b * 1.05, 4)
            rec.update({"beta": b, "workload_max_over_mean": float(cnt.max() / cnt.mean()),
                        "workload_empty": int((cnt == 0).sum())})
        else:
            rec["beta"] = beta
        out[str(cfg.zipf)] = rec
        print(n, rec, flush=True)
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "zipf_beta.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
