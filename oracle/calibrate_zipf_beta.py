"""Find the Zipf logit-bias strength beta of the skewed decode workload (CPU only).

Runs the oracle router on 64 decode steps (fresh tokens per step) and bisects
beta so that the p95 over steps of max/mean expert load is 4.0.  The printed
value is the constant ``ZIPF_BETA`` in ``routing_dispatch_grouped_top_b200/inputs.py``.
Usage: python -m oracle.calibrate_zipf_beta
"""
import numpy as np

from routing_dispatch_grouped_top_b200 import inputs
from routing_dispatch_grouped_top_b200.config import DEEPSEEK_R1_DECODE
import oracle

STEPS = 64
TARGET = 4.0


def p95_skew(cfg, beta, base_logits):
    bias = inputs.zipf_bias(cfg.E, cfg.zipf_s, beta, seed=cfg.seed).numpy()
    ratios = []
    for l in base_logits:
        ids, _ = oracle.route((l + bias).astype(np.float32), cfg.K, cfg.renormalize)
        ratios.append(oracle.skew_ratio(oracle.count_scan(ids, cfg.E)["counts"]))
    return oracle.p95_nearest_rank(ratios)


def main():
    cfg = DEEPSEEK_R1_DECODE
    w_g, _ = inputs.make_router(cfg.with_(zipf_s=None))
    w_g = w_g.numpy()
    base = [oracle.gating_logits(inputs.to_bits(inputs.make_tokens(cfg, "cpu", s)), w_g)
            for s in range(STEPS)]
    def smallest_beta_reaching(target):
        lo, hi = 0.0, 3.0
        for _ in range(24):
            mid = 0.5 * (lo + hi)
            if p95_skew(cfg, mid, base) < target:
                lo = mid
            else:
                hi = mid
        return hi

    # The p95 of integer loads moves in steps of E/(T*K); take the middle of the
    # beta interval on which it sits inside TARGET +- 0.125.
    b_lo = smallest_beta_reaching(TARGET - 0.125)
    b_hi = smallest_beta_reaching(TARGET + 0.125)
    beta = round(0.5 * (b_lo + b_hi), 4)
    print(f"beta={beta} p95_skew={p95_skew(cfg, beta, base):.4f}")


if __name__ == "__main__":
    main()
