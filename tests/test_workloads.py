"""The seeded workloads are what their names claim: the skewed-routing
workload's expert popularity follows Zipf's law inside every group (page
"Ling-3.0-flash-VL MoE sparse routing", sec. 3 step 3: the per-expert bias
is the lever on expert load; here it is calibrated to a skewed target)."""
import numpy as np
import torch

import oracle
import workloads


def test_zipf_bias_is_the_calibrated_table_by_rank():
    cfg = workloads.CONFIGS["zipf"]
    table = workloads.zipf_table(cfg.experts_per_group)
    assert table is not None and table.dtype == np.float32 and table.size == 64
    assert np.all(np.diff(table[:8]) < 0) and table[0] - table[-1] > 0.2   # favoured ranks first
    ranks = workloads.zipf_ranks(cfg)
    for g in range(cfg.n_group):                       # every group holds each rank once
        assert sorted(ranks[g * 64:(g + 1) * 64]) == list(range(1, 65))
    bias = workloads.selection_bias(cfg).numpy()
    assert np.array_equal(bias, table[ranks - 1])
    # the small layers have no table for their group size: fixed skewed formula
    tiny = workloads.CONFIGS["tiny"].with_(bias_kind="zipf")
    assert workloads.zipf_table(tiny.experts_per_group) is None
    tb = workloads.selection_bias(tiny).numpy()
    tr = workloads.zipf_ranks(tiny)
    assert np.allclose(tb, -tiny.zipf_beta * tiny.zipf_s * np.log(tr), rtol=1e-6)


def test_zipf_workload_popularity_slope():
    """Routing the workload's first 4096 tokens with the oracle: the mean count
    per within-group rank falls as r^-1.1 (log-log fit), and every expert is used."""
    cfg = workloads.CONFIGS["zipf"]
    d = workloads.router_inputs(cfg, "cpu", T=4096)
    x = d["x"].view(torch.int16).numpy().view(np.uint16)
    r = oracle.route(x, d["Wr"].numpy(), d["bias"].numpy(), cfg.n_group, cfg.topk_group, cfg.K)
    c = np.bincount(r["idx"].reshape(-1), minlength=cfg.E)
    ranks = workloads.zipf_ranks(cfg)
    m = np.array([c[ranks == q].mean() for q in range(1, 65)])
    slope = np.polyfit(np.log(np.arange(1, 65)), np.log(m), 1)[0]
    assert -1.25 < slope < -0.95, slope
    assert (c > 0).all()
