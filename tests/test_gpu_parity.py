"""GPU parity: the CUDA path (through the C-ABI) against the CPU oracle on the
same seeded inputs.

Bars: routing indices bit-exact except listed near-tie tokens (oracle margin
< 1e-6 between the 4th/5th group or the Kth/(K+1)th candidate); combine
weights within 1e-6; permutation bit-exact; layer output max |err| <=
2e-2 * RMS(oracle output) (bf16 weights, 5e-2 for MXFP4 weights expanded to
bf16). Full-size configs compare the routing and the output of every token:
that covers every (expert, row tile) work item of the expert FFN, the heavy
experts' ragged last tiles included.
"""
import numpy as np
import pytest
import torch

import oracle
import sigmoid_group_limited_b200 as sgl
import workloads
from helpers import (DeviceExperts, bits, check_routing, check_y, experts_of, host_inputs,
                     near_tie_tokens, run_layer, run_staged)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _oracle_layer(cfg, d, tokens=None):
    h = host_inputs(d)
    return oracle.layer_forward(cfg, h["x"], h["Wr"], h["bias"], experts_of(d), h["Wg_s"],
                                h["Wu_s"], h["Wd_s"], tokens=tokens)


def _tol(cfg):
    # MXFP4 through bf16: the 5e-2 bar of the format. Block-scaled (MXFP8 x
    # MXFP4): both sides quantise x and h the same way, so what differs is
    # fp32 accumulation order and rare h codes whose fp32 inputs straddle a
    # rounding midpoint; the bf16 bar holds.
    return 5e-2 if cfg.wfmt == workloads.MOE_W_MXFP4 else 2e-2


def _full_check(cfg, d, tokens=None):
    """Whole layer on the GPU vs the oracle; returns the oracle result."""
    g = run_layer(cfg, d)
    ref = _oracle_layer(cfg, d, tokens)
    near = check_routing(ref, g["idx"].cpu().numpy(), g["w"].cpu().numpy())
    counts = np.bincount(g["idx"].cpu().numpy().reshape(-1), minlength=cfg.E)
    assert np.array_equal(g["counts"].cpu().numpy(), counts)
    tok = ref["tokens"]
    keep = ~np.isin(tok, near)
    check_y(bits(g["y"])[tok[keep]], ref["y_f32"][keep], ref["y"][keep], tol=_tol(cfg))
    return g, ref, near


# ------------------------------------------------------------------ small configs

TINY = workloads.CONFIGS["tiny"]


@pytest.mark.parametrize("T", [64, 1, 7, 33, 300, 600])
def test_tiny_layer(T):
    cfg = TINY
    d = workloads.generate(cfg, DEV, T=T)
    _full_check(cfg, d)


@pytest.mark.parametrize("T,variant", [(300, {}), (600, {}), (600, dict(limit_routed=0.5, limit_shared=0.7)),
                                       (600, dict(I_shared=0)), (600, dict(I=192, I_shared=320))])
def test_tiny_layer_pair_ffn(T, variant, monkeypatch):
    """The CTA-pair expert FFN (tcgen05 cta_group::2), selected explicitly."""
    monkeypatch.setenv("SGL_MOE_FFN", "pair")
    cfg = TINY.with_(**variant)
    d = workloads.generate(cfg, DEV, T=T)
    _full_check(cfg, d)


@pytest.mark.parametrize("form", ["tokens_m", "narrow"])
@pytest.mark.parametrize("T,variant", [(600, {}), (600, dict(limit_routed=0.5, limit_shared=0.7)),
                                       (600, dict(I_shared=0)), (600, dict(I=192, I_shared=320)),
                                       (1500, dict(H=384))])
def test_tiny_layer_ffn_options(form, T, variant, monkeypatch):
    """The optional forms of the expert FFN for large batches, selected
    explicitly: token rows as the MMA's M with two partial accumulators
    (tokens_m), and 128-token tiles with double-buffered accumulators
    (narrow). The default, 256-token tiles, runs in every other test of a
    large batch."""
    monkeypatch.setenv("SGL_MOE_FFN", form)
    cfg = TINY.with_(**variant)
    d = workloads.generate(cfg, DEV, T=T)
    if cfg.I_shared == 0:
        d.update(Wg_s=None, Wu_s=None, Wd_s=None)
        g = run_layer(cfg, d)
        h = host_inputs({**d, "Wg_s": torch.zeros(1, dtype=torch.bfloat16),
                         "Wu_s": torch.zeros(1, dtype=torch.bfloat16),
                         "Wd_s": torch.zeros(1, dtype=torch.bfloat16)})
        z = np.zeros((64, cfg.H), np.uint16)
        ref = oracle.layer_forward(cfg.with_(I_shared=64), h["x"], h["Wr"], h["bias"],
                                   DeviceExperts(d), z, z, z.T.copy())
        check_routing(ref, g["idx"].cpu().numpy(), g["w"].cpu().numpy())
        keep = ~np.isin(np.arange(T), near_tie_tokens(ref))
        check_y(bits(g["y"])[keep], ref["y_f32"][keep], ref["y"][keep])
    else:
        _full_check(cfg, d)


@pytest.mark.slow
@pytest.mark.parametrize("form", ["pair", "narrow"])
def test_prefill_ffn_forms_all_tokens(form, monkeypatch):
    """The full prefill batch on the CTA-pair kernel and on 128-token tiles."""
    monkeypatch.setenv("SGL_MOE_FFN", form)
    cfg = workloads.CONFIGS["prefill"]
    d = workloads.generate(cfg, DEV)
    _full_check(cfg, d)
    del d
    torch.cuda.empty_cache()


@pytest.mark.parametrize("variant", [
    dict(limit_routed=0.5, limit_shared=0.7),           # clamps that bite
    dict(n_group=1, topk_group=1),                      # plain top-k
    dict(K=1),                                          # argmax routing
    dict(topk_group=4),                                 # all groups kept
    dict(I_shared=0),                                   # no shared expert
    dict(I=128, I_shared=192),                          # several output tiles, different sizes
    dict(renorm=False),
    dict(bias_kind="zero"),
    dict(bias_kind="zipf"),
])
def test_tiny_variants(variant):
    cfg = TINY.with_(**variant)
    d = workloads.generate(cfg, DEV, T=200)
    if cfg.I_shared == 0:
        d.update(Wg_s=None, Wu_s=None, Wd_s=None)
        g = run_layer(cfg, d)
        h = host_inputs({**d, "Wg_s": torch.zeros(1, dtype=torch.bfloat16),
                         "Wu_s": torch.zeros(1, dtype=torch.bfloat16),
                         "Wd_s": torch.zeros(1, dtype=torch.bfloat16)})
        # oracle with a zero shared expert (contributes exactly 0)
        z = np.zeros((64, cfg.H), np.uint16)
        ref = oracle.layer_forward(cfg.with_(I_shared=64), h["x"], h["Wr"], h["bias"],
                                   DeviceExperts(d), z, z, z.T.copy())
        check_routing(ref, g["idx"].cpu().numpy(), g["w"].cpu().numpy())
        keep = ~np.isin(np.arange(200), near_tie_tokens(ref))
        check_y(bits(g["y"])[keep], ref["y_f32"][keep], ref["y"][keep])
    else:
        _full_check(cfg, d)


def test_tiny_staged_with_oracle_routing_and_y_slot():
    cfg = TINY.with_(limit_routed=1.0, limit_shared=2.0)
    d = workloads.generate(cfg, DEV, T=64)
    ref = _oracle_layer(cfg, d)
    idx = torch.from_numpy(ref["idx"]).to(DEV)
    w = torch.from_numpy(ref["w"]).to(DEV)
    g = run_staged(cfg, d, idx, w)
    # permutation bit-exact against the oracle's stable counting sort
    assert np.array_equal(g["counts"].cpu().numpy(), ref["counts"])
    assert np.array_equal(g["offsets"].cpu().numpy(), ref["offsets"])
    assert np.array_equal(g["perm"].cpu().numpy(), ref["perm"])
    assert np.array_equal(g["inv"].cpu().numpy(), ref["inv_perm"])
    ys = g["y_slot"].double().cpu().numpy()
    T, K = 64, cfg.K
    routed = ys[:T * K].reshape(T, K, cfg.H)
    rs = ref["y_slot"].astype(np.float64)
    assert np.abs(routed - rs).max() <= 1e-2 * np.sqrt((rs ** 2).mean())
    sh = ys[T * K:]
    ro = ref["y_shared"].astype(np.float64)
    assert np.abs(sh - ro).max() <= 1e-2 * np.sqrt((ro ** 2).mean())
    check_y(bits(g["y"]), ref["y_f32"], ref["y"])


def test_tiny_identical_experts_closed_form():
    """All routed experts equal: y = bf16(2.5 FFN(x) + shared(x)) whatever the routing."""
    cfg = TINY
    d = workloads.generate(cfg, DEV, T=64)
    for k in ("Wg", "Wu", "Wd"):
        d[k] = d[k][:1].expand_as(d[k]).contiguous()
    g = run_layer(cfg, d)
    f = oracle.bf16_bits_to_f64
    x = f(bits(d["x"]))
    o, _ = oracle.swiglu_expert(x, f(bits(d["Wg"][0])), f(bits(d["Wu"][0])), f(bits(d["Wd"][0])))
    osh, _ = oracle.swiglu_expert(x, f(bits(d["Wg_s"])), f(bits(d["Wu_s"])), f(bits(d["Wd_s"])))
    expect = (2.5 * o.astype(np.float64) + osh).astype(np.float32)
    check_y(bits(g["y"]), expect, oracle.f32_to_bf16_bits(expect))


@pytest.mark.parametrize("T", [33, 600])
def test_scheduler_wait_runs_out_and_reports(T, monkeypatch):
    """The FFN's one cross-CTA wait (a down item waits for the gate/up tiles of
    its row tile) is bounded. With a test limit of about 1 ms and a target no
    tile count reaches, every CTA's wait runs out: the call returns, the error
    word reads MOE_DEVERR_TIMEOUT, and the next call on the same context is
    correct. No fault and no endless wait: the CTAs drain their queued items
    and leave."""
    import time
    cfg = TINY
    d = workloads.generate(cfg, DEV, T=T)
    monkeypatch.setenv("SGL_MOE_TEST_WAIT_CYCLES", "2000000")
    monkeypatch.setenv("SGL_MOE_TEST_READY_EXTRA", "1000000")
    from helpers import weights
    ws = sgl.alloc_workspace(cfg, T)
    y = torch.empty(T, cfg.H, dtype=torch.bfloat16, device=DEV)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    sgl.moe_layer_forward(cfg, d["x"], d["Wr"], d["bias"], weights(d), y, ws)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert sgl.moe_read_error(cfg, T, ws) == 2                 # MOE_DEVERR_TIMEOUT
    monkeypatch.delenv("SGL_MOE_TEST_WAIT_CYCLES")
    monkeypatch.delenv("SGL_MOE_TEST_READY_EXTRA")
    _full_check(cfg, d)                                        # the context is still usable


def test_deterministic_bits():
    cfg = TINY
    d = workloads.generate(cfg, DEV, T=300)
    a = run_layer(cfg, d)
    b = run_layer(cfg, d)
    assert torch.equal(a["y"].view(torch.int16), b["y"].view(torch.int16))
    assert torch.equal(a["idx"], b["idx"])


# ------------------------------------------------------------------ permutation alone

@pytest.mark.parametrize("T,skew", [(1, False), (32, False), (300, False), (4096, False),
                                    (16384, False), (4096, True), (2049, True)])
def test_permute_bit_exact(T, skew):
    cfg = workloads.CONFIGS["prefill"]
    g = torch.Generator().manual_seed(T)
    if skew:
        idx = torch.full((T, cfg.K), 7, dtype=torch.int32)
        idx[:, 1:] = torch.randint(0, 3, (T, cfg.K - 1), generator=g, dtype=torch.int32)
    else:
        idx = torch.randint(0, cfg.E, (T, cfg.K), generator=g, dtype=torch.int32)
    ws = sgl.alloc_workspace(cfg, T)
    out = [torch.empty(n, dtype=torch.int32, device=DEV)
           for n in (cfg.E, cfg.E + 1, T * cfg.K, T * cfg.K)]
    sgl.moe_permute(cfg, T, idx.to(DEV), *out, ws)
    torch.cuda.synchronize()
    ref = oracle.permute(idx.numpy(), cfg.E)
    for a, b in zip(out, ref):
        assert np.array_equal(a.cpu().numpy(), b)
    assert sgl.moe_read_error(cfg, T, ws) == 0


@pytest.mark.parametrize("T", [300, 16384])
def test_permute_forms_agree(T, monkeypatch):
    """Batches of several 2048-entry tiles take one cooperative launch; the
    three-kernel form (histograms, scan, scatter), kept for very large batches,
    gives the same bits."""
    cfg = workloads.CONFIGS["prefill"]
    g = torch.Generator().manual_seed(T + 1)
    idx = torch.randint(0, cfg.E, (T, cfg.K), generator=g, dtype=torch.int32).to(DEV)
    outs = []
    for form in ("fused", "split"):
        if form == "split":
            monkeypatch.setenv("SGL_MOE_PERM", "split")
        ws = sgl.alloc_workspace(cfg, T)
        out = [torch.full((n,), -3, dtype=torch.int32, device=DEV)
               for n in (cfg.E, cfg.E + 1, T * cfg.K, T * cfg.K)]
        sgl.moe_permute(cfg, T, idx, *out, ws)
        torch.cuda.synchronize()
        assert sgl.moe_read_error(cfg, T, ws) == 0
        outs.append(out)
    for a, b in zip(*outs):
        assert torch.equal(a, b)


@pytest.mark.parametrize("T", [40, 400])
def test_permute_bad_id_sets_error_word(T):
    cfg = workloads.CONFIGS["prefill"]
    idx = torch.randint(0, cfg.E, (T, cfg.K), dtype=torch.int32)
    idx[3, 2] = cfg.E + 5
    idx[9, 0] = -1
    ws = sgl.alloc_workspace(cfg, T)
    out = [torch.empty(n, dtype=torch.int32, device=DEV)
           for n in (cfg.E, cfg.E + 1, T * cfg.K, T * cfg.K)]
    sgl.moe_permute(cfg, T, idx.to(DEV), *out, ws)
    torch.cuda.synchronize()
    assert sgl.moe_read_error(cfg, T, ws) == 1
    assert out[0].sum().item() == T * cfg.K - 2       # bad slots are dropped
    assert sgl.moe_read_error(cfg, T, ws) == 0        # reading clears the word


# ------------------------------------------------------------------ full size

@pytest.mark.slow
def test_decode_full_size():
    cfg = workloads.CONFIGS["decode"]
    d = workloads.generate(cfg, DEV)
    _full_check(cfg, d)          # every one of the 32 tokens


@pytest.mark.slow
@pytest.mark.parametrize("E", [64, 128])
def test_decode_fewer_experts(E):
    # several row tiles per expert at decode size: down items that wait on the
    # gate/up tiles their own CTA is still finishing
    cfg = workloads.CONFIGS["decode"].with_(E=E)
    d = workloads.generate(cfg, DEV)
    _full_check(cfg, d)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["prefill", "prefill_bias0", "zipf", "mxfp4"])
def test_full_size_all_tokens(name):
    """Every token of the full-size workload against the oracle."""
    cfg = workloads.CONFIGS[name]
    d = workloads.generate(cfg, DEV)
    g, ref, near = _full_check(cfg, d)
    # permutation of the GPU's own routing, bit-exact, on every slot
    st = run_staged(cfg, d, g["idx"], g["w"])
    p_ref = oracle.permute(g["idx"].cpu().numpy(), cfg.E)
    assert np.array_equal(st["perm"].cpu().numpy(), p_ref[2])
    assert np.array_equal(st["offsets"].cpu().numpy(), p_ref[1])
    # staged path with the oracle's own routing covers the near-tie tokens too
    if near.size:
        st2 = run_staged(cfg, d, torch.from_numpy(ref["idx"]).to(DEV), torch.from_numpy(ref["w"]).to(DEV))
        check_y(bits(st2["y"])[near], ref["y_f32"][near], ref["y"][near], tol=_tol(cfg))
    del d, g, ref
    torch.cuda.empty_cache()


@pytest.mark.parametrize("T", [5, 200])
def test_all_scores_tied(T):
    """Wr = 0, bias = 0: every score is 0.5, every margin 0; groups 0..3 and
    experts 0..7 win by the lower-index rule and every weight is 2.5/8. At
    T > 32 every token goes through the exact-logit re-derivation."""
    cfg = workloads.CONFIGS["prefill"]
    x = torch.randn(T, cfg.H, device=DEV).to(torch.bfloat16)
    Wr = torch.zeros(cfg.E, cfg.H, device=DEV)
    ws = sgl.alloc_workspace(cfg, T)
    idx = torch.empty(T, cfg.K, dtype=torch.int32, device=DEV)
    w = torch.empty(T, cfg.K, dtype=torch.float32, device=DEV)
    sgl.moe_route(cfg, x, Wr, None, idx, w, ws)
    torch.cuda.synchronize()
    assert torch.equal(idx.cpu(), torch.arange(8, dtype=torch.int32).repeat(T, 1))
    assert torch.all(w == 0.3125)


@pytest.mark.parametrize("T,E", [(32, 512), (4096, 512), (32, 256), (700, 256), (32, 128)])
def test_route_full_size_every_token(T, E):
    """Routing of every token at full size, bit-exact outside listed near ties.
    Groups of 64 (E=512) and 32 (E=256) experts take the CTA-per-token
    selection at small T; groups of 16 (E=128) the warp-per-token one."""
    cfg = workloads.CONFIGS["prefill"].with_(E=E)
    g = torch.Generator(device=DEV).manual_seed(77 + T + E)
    x = torch.randn(T, cfg.H, device=DEV, generator=g).to(torch.bfloat16)
    Wr = torch.randn(cfg.E, cfg.H, device=DEV, generator=g) / cfg.H ** 0.5
    bias = torch.randn(cfg.E, device=DEV, generator=g) * 0.1 ** 0.5
    ws = sgl.alloc_workspace(cfg, T)
    idx = torch.empty(T, cfg.K, dtype=torch.int32, device=DEV)
    w = torch.empty(T, cfg.K, dtype=torch.float32, device=DEV)
    sgl.moe_route(cfg, x, Wr, bias, idx, w, ws)
    torch.cuda.synchronize()
    ref = oracle.route(bits(x), Wr.cpu().numpy(), bias.cpu().numpy(), cfg.n_group, cfg.topk_group, cfg.K)
    near = check_routing(ref, idx.cpu().numpy(), w.cpu().numpy())
    assert len(near) <= max(2, T // 500)


# ------------------------------------------------------------------ load statistics

def _stat_counts(kind, E, seed):
    rng = np.random.default_rng(seed)
    if kind == "uniform":
        return np.full(E, 64, np.int32)
    if kind == "zipf":
        c = rng.zipf(1.3, size=E).clip(max=1 << 20)
        return (c * (rng.random(E) < 0.6)).astype(np.int32)
    if kind == "one":
        c = np.zeros(E, np.int32)
        c[E // 3] = 4096 * 8
        return c
    return np.zeros(E, np.int32)


@pytest.mark.parametrize("E", [32, 128, 512, 1024])
@pytest.mark.parametrize("kind", ["uniform", "zipf", "one", "empty"])
def test_route_stats(E, kind):
    """Entropy, load and idle experts against the oracle on the same counts.
    Integer entries exact; entropy terms are summed in another order, so
    H and H / log2 E agree to 1e-12 relative."""
    cfg = workloads.CONFIGS["prefill"].with_(E=E, n_group=1, topk_group=1, K=1)
    counts = _stat_counts(kind, E, seed=E)
    st = torch.full((sgl.MOE_N_ROUTE_STATS,), float("nan"), dtype=torch.float64, device=DEV)
    sgl.moe_route_stats(cfg, torch.from_numpy(counts).to(DEV), st)
    torch.cuda.synchronize()
    got, ref = st.cpu().numpy(), oracle.route_stats(counts, E)
    assert np.array_equal(got[[2, 5, 6]], ref[[2, 5, 6]])
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_route_stats_after_routing():
    """The statistics read the counts that routing and the permutation left in
    device memory, on the same stream, with no copy in between."""
    cfg = workloads.CONFIGS["prefill"]
    T = 4096
    idx = torch.randint(0, cfg.E, (T, cfg.K), dtype=torch.int32,
                        generator=torch.Generator().manual_seed(5))
    ws = sgl.alloc_workspace(cfg, T)
    out = [torch.empty(n, dtype=torch.int32, device=DEV)
           for n in (cfg.E, cfg.E + 1, T * cfg.K, T * cfg.K)]
    st = torch.empty(sgl.MOE_N_ROUTE_STATS, dtype=torch.float64, device=DEV)
    sgl.moe_permute(cfg, T, idx.to(DEV), *out, ws)
    sgl.moe_route_stats(cfg, out[0], st)
    torch.cuda.synchronize()
    ref = oracle.route_stats(oracle.permute(idx.numpy(), cfg.E)[0], cfg.E)
    assert np.allclose(st.cpu().numpy(), ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("T,variant", [(64, {}), (300, dict(limit_routed=0.5, limit_shared=0.7)),
                                       (7, dict(I=128, I_shared=192))])
def test_tiny_mxfp4(T, variant):
    """Routed weights as MXFP4 codes + e8m0 scales; the oracle dequantises the
    same bytes (the bar for this format is 5e-2 x RMS)."""
    cfg = TINY.with_(wfmt=workloads.MOE_W_MXFP4, **variant)
    d = workloads.generate(cfg, DEV, T=T)
    assert "Wg" not in d and d["Wg_q"].dtype == torch.uint8
    _full_check(cfg, d)


def _tile_rule(counts, T):
    """The token tile the large-batch FFN picks from the expert loads: 256
    when 256-row tiles number at most 4/5 of the 128-row ones (the shared
    expert's T rows included), else 128."""
    rows = np.append(counts, T)
    t128 = int(np.sum((rows + 127) // 128))
    t256 = int(np.sum((rows + 255) // 256))
    return 256 if 5 * t256 <= 4 * t128 else 128


@pytest.mark.parametrize("wfmt", [workloads.MOE_W_BF16, workloads.MOE_W_MXFP4])
@pytest.mark.parametrize("T,bias_kind,tile", [(600, "zero", 128), (2000, "normal", 256)])
def test_tiny_adaptive_tile(wfmt, T, bias_kind, tile):
    """Batches above 48 rows per expert, with near-uniform loads and with one
    expert taking most rows: the bf16 FFN picks its token tile from the loads
    on the device (one case per tile); the MXFP4 one runs 256-row tiles on
    both. Each is checked against the oracle."""
    cfg = TINY.with_(wfmt=wfmt, bias_kind=bias_kind)
    d = workloads.generate(cfg, DEV, T=T)
    g, ref, near = _full_check(cfg, d)
    assert _tile_rule(g["counts"].cpu().numpy(), T) == tile


# ------------------------------------------------------------------ block-scaled MXFP8 x MXFP4

TINY_A8 = workloads.CONFIGS["tiny_a8"]


@pytest.mark.parametrize("T", [64, 1, 7, 33, 300])
def test_tiny_block_scaled(T):
    """Routed experts on tcgen05 kind::mxf8f6f4 (e2m1 weights x e4m3
    activations, e8m0 scales), shared expert on kind::f16, against the oracle
    with the same MXFP8 quantisation of x and h."""
    d = workloads.generate(TINY_A8, DEV, T=T)
    _full_check(TINY_A8, d)


@pytest.mark.parametrize("variant", [dict(limit_routed=0.5, limit_shared=0.7), dict(I=256, I_shared=192),
                                     dict(I_shared=0), dict(K=1, topk_group=1),
                                     dict(bias_kind="zipf")])
def test_tiny_block_scaled_variants(variant):
    cfg = TINY_A8.with_(**variant)
    d = workloads.generate(cfg, DEV, T=200)
    _full_check(cfg, d)


def test_block_scaled_one_expert_many_rows():
    """One expert takes every token: row tiles of 128 with a ragged tail, and
    the h scale atoms of several row tiles."""
    cfg = TINY_A8.with_(bias_kind="zero")
    d = workloads.generate(cfg, DEV, T=333)
    d["bias"] = torch.full_like(d["bias"], -1.0)
    d["bias"][5] = 1.0               # expert 5 always selected, in its group
    _full_check(cfg, d)


@pytest.mark.slow
def test_block_scaled_full_size_all_tokens():
    """The full T=8192 block-scaled layer, every token against the oracle (which
    quantises x and h the same way); the same layer with prepared scale atoms
    (MOE_W_MXFP4_A8P, which only moves scale bytes) is bit-identical to it."""
    cfg = workloads.CONFIGS["mxfp4_a8"]
    d = workloads.generate(cfg, DEV)
    g, _, _ = _full_check(cfg, d)
    pcfg = cfg.with_(wfmt=workloads.MOE_W_MXFP4_A8P)
    sg, su, sd = _prepared(pcfg, d)
    prep = run_layer(pcfg, {**d, "Wg_sc": sg, "Wu_sc": su, "Wd_sc": sd})
    assert torch.equal(g["idx"], prep["idx"]) and torch.equal(g["w"], prep["w"])
    assert np.array_equal(bits(g["y"]), bits(prep["y"]))
    del d, g, prep
    torch.cuda.empty_cache()


# ------------------------------------------------------------------ fused decode front

@pytest.mark.parametrize("T,E", [(1, 512), (7, 512), (32, 512), (32, 256), (16, 128), (32, 128),
                                 (33, 512), (48, 256), (64, 512), (64, 256)])
def test_fused_decode_front_matches_separate_kernels(T, E, monkeypatch):
    """Decode batches (up to 64 tokens) route and permute in one cooperative
    launch. Its fp32 logits add the hidden dimension in another order than the
    separate kernels, so scores may differ in the last bit; the certified
    decisions (experts, counts, permutation) are identical, the weights agree
    to 1e-6, and both outputs meet the bar against the oracle (every token
    above 32, where the separate path is the tensor-core router)."""
    cfg = workloads.CONFIGS["decode"].with_(E=E)
    d = workloads.generate(cfg, DEV, T=T)
    fused = run_layer(cfg, d)
    monkeypatch.setenv("SGL_MOE_FRONT", "separate")
    sep = run_layer(cfg, d)
    for k in ("idx", "counts"):
        assert torch.equal(fused[k], sep[k]), k
    assert torch.allclose(fused["w"], sep["w"], rtol=1e-6, atol=0)
    tok = list(range(min(T, 6))) if T <= 32 else None
    ref = _oracle_layer(cfg, d, tokens=tok)
    near = check_routing(ref, fused["idx"].cpu().numpy(), fused["w"].cpu().numpy())
    keep = ~np.isin(ref["tokens"], near)
    for g in (fused, sep):
        check_y(bits(g["y"])[ref["tokens"][keep]], ref["y_f32"][keep], ref["y"][keep], tol=_tol(cfg))



@pytest.mark.parametrize("T,E", [(32, 512), (8, 128), (64, 512)])
def test_front_l2_prefetch_changes_nothing(T, E, monkeypatch):
    """The decode front's L2 prefetch of the shared and first routed experts'
    weights only warms the cache: outputs are bit-identical with it off."""
    cfg = workloads.CONFIGS["decode"].with_(E=E)
    d = workloads.generate(cfg, DEV, T=T)
    on = run_layer(cfg, d)
    monkeypatch.setenv("SGL_MOE_PREFETCH", "0")
    off = run_layer(cfg, d)
    assert torch.equal(on["idx"], off["idx"])
    assert np.array_equal(bits(on["y"]), bits(off["y"]))


# ------------------------------------------------------------------ prepared block-scaled weights

def _prepared(cfg, d):
    """moe_prepare_weights on the generated scales; returns the atom arrays."""
    out = [torch.empty_like(d[k]) for k in ("Wg_sc", "Wu_sc", "Wd_sc")]
    sgl.moe_prepare_weights(cfg, sgl.make_weights(d["Wg_q"], d["Wu_q"], d["Wd_q"], d.get("Wg_s"),
                                                  d.get("Wu_s"), d.get("Wd_s"), d["Wg_sc"], d["Wu_sc"],
                                                  d["Wd_sc"]), *out)
    torch.cuda.synchronize()
    return out


def _atoms_host(sc: np.ndarray) -> np.ndarray:
    """The atom layout written out from its definition: [E, rows, kc] scale
    bytes -> [E, rows/128, kc/4, 512] with row r, chunk k of an atom at byte
    (r % 32) * 16 + (r / 32) * 4 + k."""
    E, rows, kc = sc.shape
    out = np.zeros((E, rows // 128, kc // 4, 512), np.uint8)
    for r in range(128):
        for k in range(4):
            out[:, :, :, (r % 32) * 16 + (r // 32) * 4 + k] = sc[:, r::128, :][:, :rows // 128, k::4]
    return out


@pytest.mark.parametrize("variant", [{}, dict(I=256, H=384)])
def test_prepare_weights_atom_layout(variant):
    cfg = TINY_A8.with_(wfmt=workloads.MOE_W_MXFP4_A8, **variant)
    d = workloads.generate(cfg, DEV, T=8)
    got = _prepared(cfg, d)
    for name, g in zip(("Wg_sc", "Wu_sc", "Wd_sc"), got):
        want = _atoms_host(d[name].cpu().numpy())
        assert np.array_equal(g.cpu().numpy().reshape(want.shape), want), name


@pytest.mark.parametrize("T,variant", [(1, {}), (64, {}), (300, {}), (64, dict(I_shared=0)),
                                       (200, dict(limit_routed=0.5, limit_shared=0.7))])
def test_prepared_block_scaled_is_bit_identical(T, variant):
    """MOE_W_MXFP4_A8P reads the prepared atoms by expert id instead of
    repacking the touched experts' scales per call; the arithmetic is the
    same, so y, idx and w are bit-identical to MOE_W_MXFP4_A8 (which is itself
    checked against the oracle above)."""
    cfg = TINY_A8.with_(**variant)
    d = workloads.generate(cfg, DEV, T=T)
    if cfg.I_shared == 0:
        d.update(Wg_s=None, Wu_s=None, Wd_s=None)
    base = run_layer(cfg, d)
    pcfg = cfg.with_(wfmt=workloads.MOE_W_MXFP4_A8P)
    g, u, dn = _prepared(pcfg, d)
    prep = run_layer(pcfg, {**d, "Wg_sc": g, "Wu_sc": u, "Wd_sc": dn})
    assert torch.equal(base["idx"], prep["idx"]) and torch.equal(base["w"], prep["w"])
    assert np.array_equal(bits(base["y"]), bits(prep["y"]))


@pytest.mark.parametrize("T,E", [(16, 128), (32, 256)])
def test_fused_front_without_shared_expert(T, E):
    """Decode batch with no shared expert: the fused front routes and
    permutes, and the FFN derives its work lists from the counts with no
    shared slot; checked against the oracle with a zero shared expert."""
    cfg = workloads.CONFIGS["decode"].with_(E=E, I_shared=0)
    d = workloads.generate(cfg, DEV, T=T)
    d.update(Wg_s=None, Wu_s=None, Wd_s=None)
    g = run_layer(cfg, d)
    h = host_inputs({**d, "Wg_s": torch.zeros(1, dtype=torch.bfloat16),
                     "Wu_s": torch.zeros(1, dtype=torch.bfloat16),
                     "Wd_s": torch.zeros(1, dtype=torch.bfloat16)})
    z = np.zeros((64, cfg.H), np.uint16)
    tok = list(range(min(T, 6)))
    ref = oracle.layer_forward(cfg.with_(I_shared=64), h["x"], h["Wr"], h["bias"], DeviceExperts(d), z, z,
                               z.T.copy(), tokens=tok)
    near = check_routing(ref, g["idx"].cpu().numpy(), g["w"].cpu().numpy())
    keep = ~np.isin(ref["tokens"], near)
    check_y(bits(g["y"])[ref["tokens"][keep]], ref["y_f32"][keep], ref["y"][keep])
