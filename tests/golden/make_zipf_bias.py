"""Writes zipf_bias_g64.txt: the selection bias of the skewed-routing
workload (16384 tokens, full-size layer, seed 3), calibrated with the
oracle so that expert popularity inside every group follows Zipf's law
p(r) ~ r^-1.1 over the within-group popularity rank r = 1..64.

The calibration uses the balancing idea of page "Ling-3.0-flash-VL MoE sparse
routing" (lqnn.cn/news/282163), sec. 3 step 3: a per-expert additive bias on
the selection score steers load, raised for experts that are picked too
rarely and lowered for those picked too often. Here it is driven toward a
skewed target instead of toward balance:

  bias_e = beta[r_e]   (one value per rank, the same in every group)
  beta[r] += eta * clip(ln p*(r) - ln p_hat(r), -1, 1);  beta -= mean(beta)

p*(r) = r^-1.1 / sum_q q^-1.1; p_hat(r) = the share of slots routed to
rank-r experts (counts averaged over the groups, +0.5 smoothing), measured
by routing a separate calibration batch (8192 tokens of step 100, not the
workload's own tokens) with the oracle. 200 steps of eta = 0.01.
Only the oracle and the seeded input generators are used.

  python tests/golden/make_zipf_bias.py      (about a minute on the CPU)
"""
import os
import sys

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
import workloads  # noqa: E402

OUT = os.path.join(HERE, "zipf_bias_g64.txt")
CAL_TOKENS, CAL_STEP, STEPS, ETA = 8192, 100, 200, 0.01


def main():
    cfg = workloads.CONFIGS["zipf"]
    per = cfg.experts_per_group
    d = workloads.router_inputs(cfg, "cpu")
    Wr = d["Wr"].numpy()
    xc = workloads.tokens(cfg, CAL_TOKENS, CAL_STEP, "cpu").view(torch.int16).numpy().view(np.uint16)
    ranks = workloads.zipf_ranks(cfg)
    r = np.arange(1, per + 1)
    pstar = r ** -cfg.zipf_s
    pstar /= pstar.sum()
    s = oracle.sigmoid_scores(oracle.router_logits(xc, Wr))
    beta = np.zeros(per)
    for _ in range(STEPS):
        bias = beta[ranks - 1].astype(np.float32)
        idx, _, _ = oracle.group_limited_topk(oracle.biased_scores(s, bias), cfg.n_group,
                                              cfg.topk_group, cfg.K)
        c = np.bincount(idx.reshape(-1), minlength=cfg.E).astype(np.float64)
        m = np.array([c[ranks == q].mean() for q in r])
        phat = (m + 0.5) / (m.sum() + 0.5 * per)
        beta += ETA * np.clip(np.log(pstar) - np.log(phat), -1.0, 1.0)
        beta -= beta.mean()
    beta32 = beta.astype(np.float32)
    with open(OUT, "w") as f:
        f.write("# Selection bias per within-group popularity rank (1..64) of the skewed-routing\n"
                "# workload, written by make_zipf_bias.py (see its docstring). One fp32 value per\n"
                "# line as a hex bit pattern, then its decimal value.\n")
        for q in range(per):
            bits = int(np.array(beta32[q]).view(np.uint32))
            f.write(f"{q + 1} 0x{bits:08x} {float(beta32[q]):.9g}\n")
    print(OUT)


if __name__ == "__main__":
    main()
