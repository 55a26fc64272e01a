"""Pins for the oracle's routing stages (sigmoid router, bias, group-limited
top-k, combine weights) and permutation. None of these re-types the oracle's
formula: each checks it against brute force, exact sums, a hand-worked
fixture, a reduction to a simpler textbook selection, or an invariant."""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_fixture(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            k, v = line.split("=", 1)
            vals[k.strip()] = v.split("|", 1)[0].strip()
    return vals


def _tiny_inputs(seed=0, T=64):
    cfg = workloads.CONFIGS["tiny"]
    d = workloads.generate(cfg.with_(seed=seed), "cpu", T=T)
    x = d["x"].view(torch.int16).numpy().view(np.uint16)
    return cfg, x, d["Wr"].numpy(), d["bias"].numpy()


# ---------------------------------------------------------------- constants

def test_config_constants_match_pages():
    g = _read_fixture("ling3_moe_constants.txt")
    full = workloads.CONFIGS["prefill"]
    assert full.H == int(g["hidden_size"])
    assert full.I == int(g["moe_intermediate_size"]) == full.I_shared
    assert full.E == int(g["num_experts"])
    assert full.n_group == int(g["n_group"])
    assert full.experts_per_group == int(g["experts_per_group"])
    assert full.topk_group == int(g["topk_group"])
    assert full.K == int(g["num_experts_per_tok"])
    assert full.topk_group * full.experts_per_group == int(g["candidates_after_group_limit"])
    assert full.scale == float(g["routed_scaling_factor"])
    assert full.renorm is True and g["norm_topk_prob"] == "true"
    z = workloads.CONFIGS["zipf"]
    assert z.limit_routed == float(g["swiglu_limit_routed"])
    assert z.limit_shared == float(g["swiglu_limit_shared"])
    # 3 * 2560 * 768 = 5 898 240 ~ 5.90 M parameters per expert
    assert workloads.expert_params(full) == 5_898_240
    assert round(workloads.expert_params(full) / 1e6, 2) == float(g["params_per_expert_millions"])
    assert int(g["moe_layers"]) * full.E * 3 == int(g["expert_tensors"])
    assert full.K / full.E == 1 / 64


# ---------------------------------------------------------------- logits and sigmoid

def test_router_logits_equal_exact_sums():
    """z is the exactly rounded dot product: compare with math.fsum (exact)."""
    cfg, x, Wr, _ = _tiny_inputs(T=6)
    z = oracle.router_logits(x, Wr)
    xf = oracle.bf16_bits_to_f64(x)
    for t in range(6):
        for e in range(0, cfg.E, 3):
            exact = math.fsum(float(a) * float(b) for a, b in zip(xf[t], Wr[e].astype(np.float64)))
            assert z[t, e] == np.float32(exact)


def test_sigmoid_special_values_and_library():
    z = np.array([0.0, -0.0, 1.0, -1.0, 20.0, -20.0, 100.0, -100.0, 3.5], dtype=np.float32)
    s = oracle.sigmoid_scores(z)
    assert s[0] == np.float32(0.5) and s[1] == np.float32(0.5)
    assert s[6] == np.float32(1.0)
    # against scipy's logistic function (independent library routine)
    from scipy.special import expit
    ref = expit(z.astype(np.float64)).astype(np.float32)
    assert np.array_equal(s, ref)
    # symmetry s(z) + s(-z) = 1 to fp32 resolution
    assert abs(float(s[2]) + float(s[3]) - 1.0) < 1e-7


def test_bias_addition_is_fp32_addition():
    rng = np.random.default_rng(5)
    s = rng.random((4, 8)).astype(np.float32)
    bias = rng.normal(size=8).astype(np.float32)
    b = oracle.biased_scores(s, bias)
    assert np.array_equal(b, s + bias[None, :])     # numpy fp32 add is IEEE fp32


# ---------------------------------------------------------------- group-limited top-k

def _brute_force_groups(gscore_row, topk_group):
    """Enumerate all subsets; the kept set is the one whose members, listed
    best first by (score desc, index asc), is lexicographically best."""
    n = len(gscore_row)
    best, best_key = None, None
    for sub in itertools.combinations(range(n), topk_group):
        key = sorted((-float(gscore_row[g]), g) for g in sub)
        if best_key is None or key < best_key:
            best, best_key = set(sub), key
    return best


@pytest.mark.parametrize("n_group,topk_group,K,E", [(4, 2, 4, 32), (8, 4, 8, 64), (8, 4, 3, 32)])
def test_group_subset_brute_force(n_group, topk_group, K, E):
    rng = np.random.default_rng(n_group * 100 + K)
    T = 200
    b = rng.normal(size=(T, E)).astype(np.float32)
    # inject exact ties between groups on some rows
    b[::7, : E // n_group] = b[::7, E // n_group: 2 * E // n_group]
    idx, _, _ = oracle.group_limited_topk(b, n_group, topk_group, K)
    per = E // n_group
    gscore = b.reshape(T, n_group, per).max(axis=2)
    for t in range(T):
        kept = _brute_force_groups(gscore[t], topk_group)
        assert {int(e) // per for e in idx[t]} <= kept
        # the chosen experts are the K best of the kept groups' experts
        cands = [e for e in range(E) if e // per in kept]
        by_rank = sorted(cands, key=lambda e: (-float(b[t, e]), e))[:K]
        assert list(idx[t]) == by_rank


def test_rank_count_rederivation():
    """e is chosen iff its group is kept and fewer than K candidates beat it
    (higher b, or equal b and lower index); its slot is that count."""
    cfg, x, Wr, bias = _tiny_inputs(seed=3)
    r = oracle.route(x, Wr, bias, cfg.n_group, cfg.topk_group, cfg.K)
    b, idx = r["b"], r["idx"]
    per = cfg.experts_per_group
    T = b.shape[0]
    gscore = b.reshape(T, cfg.n_group, per).max(axis=2)
    for t in range(T):
        # kept groups by counting too: g kept iff fewer than KG groups beat it
        kept = [g for g in range(cfg.n_group)
                if sum(1 for h in range(cfg.n_group)
                       if gscore[t, h] > gscore[t, g] or (gscore[t, h] == gscore[t, g] and h < g))
                < cfg.topk_group]
        cands = [e for e in range(cfg.E) if e // per in kept]
        chosen = {}
        for e in cands:
            beat = sum(1 for c in cands if b[t, c] > b[t, e] or (b[t, c] == b[t, e] and c < e))
            if beat < cfg.K:
                chosen[beat] = e
        assert [chosen[k] for k in range(cfg.K)] == list(idx[t])


def _plain_topk(row, K):
    """Textbook selection: K rounds of argmax (first index wins ties)."""
    row = row.astype(np.float64).copy()
    out = []
    for _ in range(K):
        e = int(np.argmax(row))
        out.append(e)
        row[e] = -np.inf
    return out


@pytest.mark.parametrize("n_group,topk_group", [(4, 4), (1, 1), (8, 8)])
def test_all_groups_kept_reduces_to_plain_topk(n_group, topk_group):
    rng = np.random.default_rng(11)
    b = rng.normal(size=(50, 64)).astype(np.float32)
    b[3, 10] = b[3, 20] = b[3].max() + 1      # an exact tie at the top
    idx, gm, _ = oracle.group_limited_topk(b, n_group, topk_group, 8)
    for t in range(50):
        assert list(idx[t]) == _plain_topk(b[t], 8)
    assert np.all(np.isinf(gm))
    # partial_sort-style library check: the chosen set equals numpy's top-8 set
    part = np.argpartition(-b.astype(np.float64), 8, axis=1)[:, :8]
    for t in range(50):
        if t != 3:
            assert set(idx[t]) == set(part[t])


def test_k1_is_argmax_over_kept_groups():
    rng = np.random.default_rng(12)
    b = rng.normal(size=(100, 32)).astype(np.float32)
    idx, _, _ = oracle.group_limited_topk(b, 4, 4, 1)
    assert np.array_equal(idx[:, 0], np.argmax(b, axis=1))


def test_all_scores_equal_pins_tie_rules():
    """Wr = 0 and bias = 0: every score is 0.5, so groups 0..KG-1 are kept,
    the first K experts of group 0 are chosen and each weight is 2.5/K."""
    cfg = workloads.CONFIGS["prefill"]
    T = 3
    x = np.full((T, cfg.H), 0x3F80, dtype=np.uint16)     # x = 1.0
    Wr = np.zeros((cfg.E, cfg.H), np.float32)
    r = oracle.route(x, Wr, np.zeros(cfg.E, np.float32), cfg.n_group, cfg.topk_group, cfg.K)
    assert np.all(r["s"] == np.float32(0.5))
    assert np.array_equal(r["idx"], np.tile(np.arange(8, dtype=np.int32), (T, 1)))
    assert np.all(r["w"] == np.float32(0.3125))
    assert np.all(r["gmargin"] == 0.0) and np.all(r["emargin"] == 0.0)


def test_hand_worked_example():
    g = _read_fixture("routing_hand_example.txt")
    s = np.array([[float(v) for v in g["s"].split()]], np.float32)
    bias = np.array([float(v) for v in g["bias"].split()], np.float32)
    b = oracle.biased_scores(s, bias)
    idx, _, _ = oracle.group_limited_topk(b, int(g["n_group"]), int(g["topk_group"]), int(g["K"]))
    assert list(idx[0]) == [int(v) for v in g["idx"].split()]
    w = oracle.combine_weights(s, idx, 2.5, True)
    assert np.allclose(w[0], [float(v) for v in g["w"].split()], rtol=0, atol=1e-7)
    _, gm, em = oracle.group_limited_topk(b, int(g["n_group"]), int(g["topk_group"]), int(g["K"]))
    assert gm[0] == float(g["gmargin"]) and em[0] == float(g["emargin"])


def test_hand_worked_margins():
    """Both near-tie margins nonzero and distinct, worked out on paper; a margin
    taken one rank too early, or over all experts instead of the kept groups'
    candidates, gives another value (the fixture lists them)."""
    g = _read_fixture("routing_hand_margins.txt")
    s = np.array([[float(v) for v in g["s"].split()]], np.float32)
    bias = np.array([float(v) for v in g["bias"].split()], np.float32)
    b = oracle.biased_scores(s, bias)
    idx, gm, em = oracle.group_limited_topk(b, int(g["n_group"]), int(g["topk_group"]), int(g["K"]))
    assert list(idx[0]) == [int(v) for v in g["idx"].split()]
    assert gm[0] == float(g["gmargin"]) and em[0] == float(g["emargin"])
    w = oracle.combine_weights(s, idx, 2.5, True)
    assert np.allclose(w[0], [float(v) for v in g["w"].split()], rtol=0, atol=1e-7)


def _py_margins(row, n_group, topk_group, K):
    """The two margins from plain sorted Python lists: groups by (max desc,
    index asc), candidates = experts of the kept groups by (b desc, e asc)."""
    E = len(row)
    per = E // n_group
    gs = [max(float(row[e]) for e in range(g * per, (g + 1) * per)) for g in range(n_group)]
    order = sorted(range(n_group), key=lambda g: (-gs[g], g))
    kept = set(order[:topk_group])
    gm = gs[order[topk_group - 1]] - gs[order[topk_group]] if topk_group < n_group else math.inf
    cands = sorted((e for e in range(E) if e // per in kept), key=lambda e: (-float(row[e]), e))
    em = float(row[cands[K - 1]]) - float(row[cands[K]]) if K < len(cands) else math.inf
    return gm, em


@pytest.mark.parametrize("n_group,topk_group,K,E", [(4, 2, 4, 32), (8, 4, 8, 512), (8, 4, 3, 64),
                                                    (4, 4, 4, 32), (8, 1, 8, 64)])
def test_margins_brute_force(n_group, topk_group, K, E):
    rng = np.random.default_rng(E + 7 * K + topk_group)
    T = 120
    b = rng.normal(scale=0.3, size=(T, E)).astype(np.float32)
    per = E // n_group
    b[::5, :per] = b[::5, per:2 * per]                  # tied groups
    b[1::7, 3] = b[1::7, 5]                             # tied experts
    b[2::9] = np.round(b[2::9] * 8) / 8                 # many exact ties at once
    _, gm, em = oracle.group_limited_topk(b, n_group, topk_group, K)
    for t in range(T):
        g_ref, e_ref = _py_margins(b[t], n_group, topk_group, K)
        assert gm[t] == g_ref and em[t] == e_ref


# ---------------------------------------------------------------- weights and invariants

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_routing_invariants(seed):
    cfg, x, Wr, bias = _tiny_inputs(seed=seed)
    r = oracle.route(x, Wr, bias, cfg.n_group, cfg.topk_group, cfg.K, cfg.scale, cfg.renorm)
    idx, w = r["idx"], r["w"]
    per = cfg.experts_per_group
    for t in range(idx.shape[0]):
        assert len(set(idx[t])) == cfg.K
        assert len({int(e) // per for e in idx[t]}) <= cfg.topk_group
    assert np.all(np.abs(w.astype(np.float64).sum(1) - 2.5) <= 1e-6)
    assert np.all(w > 0)
    # weights use the unbiased scores: ratios equal score ratios
    sel = np.take_along_axis(r["s"], idx, 1).astype(np.float64)
    assert np.allclose(w / w[:, :1], sel / sel[:, :1], rtol=1e-6)


def test_renorm_off_keeps_raw_scores():
    s = np.array([[0.2, 0.9, 0.4, 0.6]], np.float32)
    w = oracle.combine_weights(s, np.array([[1, 3]]), 2.5, False)
    assert np.allclose(w, [[2.25, 1.5]], atol=1e-7)


def test_weight_sum_underflow_is_an_error():
    s = np.zeros((1, 4), np.float32)
    with pytest.raises(FloatingPointError):
        oracle.combine_weights(s, np.array([[0, 1]]), 2.5, True)


# ---------------------------------------------------------------- permutation

def _counting_sort(flat, E):
    buckets = [[] for _ in range(E)]
    for j, e in enumerate(flat):
        buckets[e].append(j)
    return [j for b in buckets for j in b]


@pytest.mark.parametrize("T,K,E", [(1, 1, 4), (13, 4, 32), (64, 8, 512), (5, 3, 7)])
def test_permutation_is_stable_counting_sort(T, K, E):
    rng = np.random.default_rng(T * 7 + E)
    idx = rng.integers(0, E, size=(T, K)).astype(np.int32)
    counts, offsets, perm, inv = oracle.permute(idx, E)
    flat = idx.reshape(-1)
    assert list(perm) == _counting_sort(list(flat), E)
    assert counts.sum() == T * K and offsets[0] == 0 and offsets[-1] == T * K
    assert np.all(np.diff(offsets) == counts)
    assert np.array_equal(np.sort(perm), np.arange(T * K))
    assert np.array_equal(inv[perm], np.arange(T * K))
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)


def test_permutation_one_expert_takes_all():
    idx = np.full((10, 1), 5, np.int32)
    counts, offsets, perm, _ = oracle.permute(idx, 8)
    assert counts[5] == 10 and offsets[5] == 0 and offsets[6] == 10
    assert np.array_equal(perm, np.arange(10))


# ---------------------------------------------------------------- load statistics

@pytest.mark.parametrize("E", [2, 8, 128, 512])
def test_route_stats_uniform_load_has_full_entropy(E):
    st = oracle.route_stats(np.full(E, 3, np.int32), E)
    assert st[0] == pytest.approx(math.log2(E), rel=1e-14)   # H of a uniform law
    assert st[1] == pytest.approx(1.0, rel=1e-14)
    assert st[2] == 3 and st[3] == 3 and st[4] == 1 and st[5] == 0 and st[6] == 3 * E


def test_route_stats_one_expert_takes_all():
    c = np.zeros(64, np.int32)
    c[17] = 40
    st = oracle.route_stats(c, 64)
    assert st[0] == 0 and st[1] == 0
    assert st[2] == 40 and st[3] == 40 / 64 and st[4] == 64      # max/mean = E
    assert st[5] == 63 and st[6] == 40


def test_route_stats_worked_dyadic_law():
    # p = (1/4, 1/4, 1/2, 0): H = 2*(1/4)*2 + (1/2)*1 = 1.5 bits exactly
    st = oracle.route_stats(np.array([1, 1, 2, 0], np.int32), 4)
    assert st[0] == 1.5 and st[1] == 0.75
    assert st[2] == 2 and st[3] == 1 and st[4] == 2 and st[5] == 1 and st[6] == 4


def test_route_stats_no_slots():
    st = oracle.route_stats(np.zeros(32, np.int32), 32)
    assert list(st) == [0, 0, 0, 0, 0, 32, 0]


@pytest.mark.parametrize("seed", range(4))
def test_route_stats_against_counting_loop(seed):
    rng = np.random.default_rng(seed)
    E = int(rng.integers(2, 300))
    counts = rng.zipf(1.5, size=E).clip(max=1000) * (rng.random(E) < 0.7)
    tot = int(counts.sum())
    H = sum(-(n / tot) * math.log(n / tot) / math.log(2) for n in counts if n > 0)
    st = oracle.route_stats(counts.astype(np.int32), E)
    assert st[0] == pytest.approx(H, rel=1e-12)
    assert 0 <= st[0] <= math.log2(E - st[5]) + 1e-12          # H <= log2(#experts used)
    assert st[5] == sum(1 for n in counts if n == 0)
    assert st[2] == max(counts) and st[6] == tot
    # relabelling the experts changes nothing
    assert np.allclose(oracle.route_stats(rng.permutation(counts).astype(np.int32), E), st,
                       rtol=1e-14, atol=0)
