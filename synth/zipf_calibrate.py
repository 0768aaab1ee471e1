"""Freeze the Zipf logit-bias scale beta of the skewed workload.

The skewed workload adds b_e = -beta * 1.2 * ln(rank_e) to the router logits
(rank_e a seeded permutation of 1..E).  With top-8 routing over distinct
experts no expert can receive more than 1/8 of all assignments, so the target
"hottest expert receives ~30%" is read as: about 30% of tokens select the
hottest expert.  This script bisects beta on the oracle's routing of the
seed-0 inputs to hit 0.30 and writes zipf_beta.json.  It calls only the
oracle (for RMSNorm, router logits and softmax top-k) and this package's
generator.

    python -m synth.zipf_calibrate
"""
import json
import os

import numpy as np

import oracle as O
from synth import workloads as W


def hottest_share(logits, bias, k):
    idx, _, _ = O.route_softmax(logits, k, False, 1.0, bias)
    counts = O.expert_histogram(idx, logits.shape[1])
    return counts.max() / logits.shape[0], int(np.argmax(counts))


def main():
    cfg = W.C5
    x = O.bf16_bits_to_f64(W.host_bf16(cfg, "x"))
    xn = O.round_bf16(O.rmsnorm(x, np.ones(cfg.D), cfg.eps))
    logits = O.router_logits(xn, O.bf16_bits_to_f64(W.host_bf16(cfg, "w_router")))
    lo, hi = 0.0, 8.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        share, _ = hottest_share(logits, W.zipf_bias(cfg.E, mid), cfg.k)
        lo, hi = (mid, hi) if share < 0.30 else (lo, mid)
    beta = round(0.5 * (lo + hi), 6)
    share, hot = hottest_share(logits, W.zipf_bias(cfg.E, beta), cfg.k)
    out = {"beta": beta, "zipf_s": W.ZIPF_S, "hottest_share_of_tokens": round(float(share), 5),
           "hottest_expert": hot, "T": cfg.T, "E": cfg.E, "k": cfg.k, "seed": W.SEED,
           "written_by": "synth/zipf_calibrate.py (oracle routing of the seed-0 inputs)"}
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "zipf_beta.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=2)
    print(out)


if __name__ == "__main__":
    main()
