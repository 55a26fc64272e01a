"""bench.py host logic without a GPU: max-over-ranks timing on 2 gloo ranks,
replica sharding, and the roofline arithmetic."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench
import workloads


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, _ = bench.dist_env()
    bench.dist_init(w, "gloo")
    bench.barrier()
    m = bench.reduce_max(10.0 * (r + 1))
    q.put((r, m, bench.replica_tokens_seed(workloads.CONFIGS["decode"], r)))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    out = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [20.0, 20.0]          # every rank sees the max
    assert out[0][2] != out[1][2]                        # every rank draws its own batch


def test_reduce_max_single_process_identity():
    assert bench.reduce_max(3.5) == 3.5


def test_roofline_arithmetic():
    cfg = workloads.CONFIGS["decode"]
    w = bench.algorithmic_work(cfg, 32, touched=100)
    gu_b, gu_f = w["gateup"]
    assert gu_b == 100 * 2 * 768 * 2560 * 2 + 2 * 768 * 2560 * 2 + 32 * 2560 * 2
    assert gu_f == 2.0 * (32 * 8 * 2 * 768 * 2560 + 32 * 2 * 768 * 2560)
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1300.0}
    e = bench.roofline_entry(gu_b, gu_f, gu_b / 3000e9, peaks)       # half the HBM peak
    assert e["bound"] == "hbm" and abs(e["frac"] - 0.5) < 1e-6
    big = bench.algorithmic_work(workloads.CONFIGS["zipf"], 16384, touched=200)
    b, f = big["gateup"]
    e = bench.roofline_entry(b, f, f / 750e12, peaks)
    assert e["bound"] == "tensor" and abs(e["frac"] - 0.5) < 1e-6
    # the whole layer: 106.2 MFLOP per token in the experts (K routed + 1 shared)
    lb, lf = bench.algorithmic_work(cfg, 1, touched=8)["layer"]
    assert abs(lf - 106.17e6) / 106.17e6 < 1e-3


def test_block_scaled_formats_in_bench_accounting():
    """The prepared block-scaled format counts the same work as the per-call
    one (only where the scale atoms come from differs), two fewer launches,
    and every weight format has a dtype label."""
    import bench
    a8 = workloads.CONFIGS["mxfp4_a8"]
    a8p = workloads.CONFIGS["mxfp4_a8p"]
    assert a8p.wfmt == workloads.MOE_W_MXFP4_A8P and a8p.with_(wfmt=a8.wfmt, name=a8.name) == a8
    assert bench.algorithmic_work(a8, a8.T, 131) == bench.algorithmic_work(a8p, a8p.T, 131)
    assert bench.kernels_per_step(a8) - bench.kernels_per_step(a8p) == 2
    for fmt in (workloads.MOE_W_BF16, workloads.MOE_W_MXFP4, workloads.MOE_W_MXFP4_A8,
                workloads.MOE_W_MXFP4_A8P):
        assert fmt in bench.DTYPES
    # decode batches take the fused front: front, FFN, combine
    assert bench.kernels_per_step(workloads.CONFIGS["decode"]) == 3


def test_bench_helpers_used_by_the_gpu_arm():
    """Host helpers the GPU arm calls: the Zipf popularity slope of a count
    vector, the fused front's L2-prefetched bytes, the traffic lookup and the
    tensor-peak ratios (exercised here so that a missing name fails on CPU)."""
    import numpy as np
    cfg = workloads.CONFIGS["zipf"]
    ranks = workloads.zipf_ranks(cfg)
    counts = np.round(4000.0 * ranks.astype(np.float64) ** -1.1).astype(np.int64)
    assert abs(bench.popularity_slope(cfg, counts) + 1.1) < 0.01
    dec = workloads.CONFIGS["decode"]
    shared = 3 * 768 * 2560 * 2
    assert bench.front_prefetch_bytes(dec, 58) == shared + 4 * (2 * 768 * 2560 * 2)
    assert bench.front_prefetch_bytes(dec, 2) == shared + 2 * (2 * 768 * 2560 * 2)
    assert bench.front_prefetch_bytes(workloads.CONFIGS["prefill"], 122) == 0     # no fused front
    assert bench.ffn_traffic(dec) is None or len(bench.ffn_traffic(dec)) == 2
    # counters are tied to the full-size workload: a shrunk one reports none
    assert bench.ffn_traffic(dec.with_(E=128)) is None
    assert bench.ffn_traffic(workloads.CONFIGS["prefill"].with_(T=1024)) is None
    r = bench.tensor_ratios(None)
    assert r["source"] == "nominal" and r["fp8"] == 2.0 and r["fp4"] == 4.0
    probe = {"bf16": {"tflops": 1000.0}, "e2m1xe4m3": {"tflops": 2000.0}, "e2m1xe2m1": {"tflops": 4100.0}}
    r = bench.tensor_ratios(probe)
    assert r["fp8"] == 2.0 and abs(r["fp4"] - 4.1) < 1e-12
    assert set(bench.WORKLOAD_NOTES) >= {"decode", "prefill", "prefill_bias0", "zipf", "mxfp4", "mxfp4_a8"}
