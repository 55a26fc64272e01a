#!/usr/bin/env python
"""Benchmark of one sparse-MoE FFN layer forward on B200 (sm_100a).

A step is one whole-layer forward (router, top-k, permutation, grouped
SwiGLU experts + shared expert, combine) through the C-ABI on one synthetic
token batch whose inputs and weights are already resident in HBM. The L2 is
flushed (256 MB write) before every step, outside the step's CUDA events.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode|prefill|...]
                  [--impl reference]

With N > 1 (launched by torch.distributed.run) every rank runs an independent
replica of the layer on its own batch (tokens are independent: no data-path
collective); timing is the max over ranks and `value` counts all ranks'
tokens (weak scaling). `--impl reference` times the CPU oracle instead
(rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "MoE-layer tokens/s (T=4096 prefill, T=32 decode) and % of roofline"
L2_FLUSH_BYTES = 256 << 20
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ distributed plumbing

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def dist_init(world: int, backend: str):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def reduce_max(value: float, device=None) -> float:
    """Max of a scalar over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and str(device).startswith("cuda"):
            dist.barrier(device_ids=[int(str(device).split(":")[1])])
        else:
            dist.barrier()


def replica_config(cfg: workloads.MoEConfig, rank: int) -> workloads.MoEConfig:
    """Rank r's replica: same layer weights, its own token batch."""
    return cfg


def replica_tokens_seed(cfg: workloads.MoEConfig, rank: int) -> int:
    return rank  # step index offset for workloads.tokens(): every rank draws its own batch


# ------------------------------------------------------------------ peaks, clocks

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                    source="measured")
    return dict(PEAKS_FALLBACK, source="fallback")


class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU, polled through NVML
    every 2 ms while a timed loop runs (timed() windows), so that even a few
    milliseconds of timed steps get samples."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device: str):
        self.device = device
        self.samples = []
        self.active = False
        self.stop = False
        self.thread = None
        self.nvml = None

    def _handle(self):
        import torch
        nv = self.nvml
        idx = torch.device(self.device).index or 0
        try:
            uuid = str(torch.cuda.get_device_properties(idx).uuid)
            return nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(idx)

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = self._handle()
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.reason_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.masks = [(n, getattr(pynvml, a)) for n, a in self.REASONS]
        except Exception:
            self.nvml = None
            return self
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()
        return self

    def _run(self):
        nv = self.nvml
        while not self.stop:
            if self.active:
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                    bits = self.reason_fn(self.h)
                    self.samples.append((mhz, [n for n, m in self.masks if bits & m]))
                except Exception:
                    pass
            time.sleep(0.002)

    class _Window:
        def __init__(self, owner):
            self.owner = owner

        def __enter__(self):
            self.owner.active = True

        def __exit__(self, *a):
            self.owner.active = False

    def timed(self):
        return ClockSampler._Window(self)

    def __exit__(self, *a):
        self.stop = True
        if self.thread is not None:
            self.thread.join(timeout=5)
        if self.nvml is not None:
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass

    def summary(self):
        if self.nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"],
                    "samples": 0}
        reasons = sorted({r for _, rs in self.samples for r in rs})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples),
                "source": "NVML, every 2 ms during the timed loops"}


# ------------------------------------------------------------------ roofline arithmetic

def algorithmic_work(cfg, T: int, touched: int):
    """Bytes and FLOPs the layer must move / compute (intermediates not credited)."""
    H, I, Is, K, E = cfg.H, cfg.I, cfg.I_shared, cfg.K, cfg.E
    # bytes per routed weight: bf16, or MXFP4 (half a byte + one scale byte per 32)
    wb = 2 if cfg.wfmt == workloads.MOE_W_BF16 else 0.5 + 1.0 / 32
    gu_bytes = touched * 2 * I * H * wb + 2 * Is * H * 2 + T * H * 2
    dn_bytes = touched * H * I * wb + H * Is * 2
    gu_flops = 2.0 * (T * K * 2 * I * H + T * 2 * Is * H)
    dn_flops = 2.0 * (T * K * H * I + T * H * Is)
    router_bytes = E * H * 4 + E * 4 + T * H * 2 + T * K * 8
    layer_bytes = gu_bytes + dn_bytes + router_bytes - T * H * 2 + T * H * 2  # x counted once, y out
    layer_flops = gu_flops + dn_flops
    return dict(gateup=(gu_bytes, gu_flops), down=(dn_bytes, dn_flops),
                layer=(layer_bytes, layer_flops), router_flops=2.0 * T * H * E)


# the nominal dense fp8 / bf16 and fp4 / bf16 tensor ratios (4.5 and 9 against
# 2.25 PFLOP/s): used only when the tensor-core probe cannot run
FP8_OVER_BF16_NOMINAL = 2.0
FP4_OVER_BF16_NOMINAL = 4.0


def tensor_ratios(probe) -> dict:
    """Block-scaled / bf16 instruction-throughput ratios from the probe
    (sigmoid_group_limited_b200.peak), else the nominal ones."""
    if probe:
        b = probe["bf16"]["tflops"]
        return {"fp8": probe["e2m1xe4m3"]["tflops"] / b, "fp4": probe["e2m1xe2m1"]["tflops"] / b,
                "source": "measured (tcgen05 probe on this GPU)"}
    return {"fp8": FP8_OVER_BF16_NOMINAL, "fp4": FP4_OVER_BF16_NOMINAL, "source": "nominal"}


def roofline_entry(bytes_, flops, seconds, peaks, sustained=False, fp8_flops=0.0, fp8_ratio=None):
    """fp8_flops: the part of `flops` that runs block-scaled 8-bit, whose peak
    is fp8_ratio x the bf16 one; the entry's peak is then the effective rate of
    the mix, flops / (bf16 time + fp8 time)."""
    ratio = FP8_OVER_BF16_NOMINAL if fp8_ratio is None else fp8_ratio
    tp = (peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]) * 1e12
    bw = peaks["hbm_gbs"] * 1e9
    t_mem = bytes_ / bw
    t_tc = (flops - fp8_flops) / tp + fp8_flops / (ratio * tp)
    tp = flops / t_tc if t_tc > 0 else tp
    if t_mem >= t_tc:
        ach = bytes_ / seconds / 1e9
        return {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / peaks["hbm_gbs"], 4)}
    ach = flops / seconds / 1e12
    pk = tp / 1e12
    return {"bound": "tensor", "achieved": round(ach, 1), "peak": pk, "unit": "TFLOP/s",
            "frac": round(ach / pk, 4)}


# DRAM bytes (dram__bytes_read.sum, dram__bytes_write.sum) of one expert-FFN
# launch of each full-size workload, from one-pass ncu captures of the bench's
# own command at the same token count (profiles/ffn_traffic_full_size.md).
# Valid only for the FFN sources they were taken on (ffn.cu, ffn_mx.cu and
# ffn_common.cuh): another source reports traffic null.
FFN_TRAFFIC_SOURCES_SHA256 = "7cbaa6b3231673557d8c4dca5e4c259cc2ebed313273c28f71f0f90f755d8304"
FFN_TRAFFIC = {                      # workload name -> (read bytes, write bytes)
    "decode": (696.27e6, 5.08e6),
    "prefill": (1.72e9, 377.69e6),
    "prefill_bias0": (6.19e9, 376.59e6),
    "zipf": (7.97e9, 1.68e9),
    "mxfp4": (919.87e6, 809.59e6),
    "mxfp4_a8": (669.30e6, 761.82e6),
}


def ffn_sources_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    for name in ("ffn.cu", "ffn_mx.cu", "ffn_common.cuh"):
        with open(os.path.join(ROOT, "sigmoid_group_limited_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def ffn_traffic(cfg):
    """(read, write) DRAM bytes of one FFN launch of `cfg`'s workload, or None
    (other FFN sources, or a workload shrunk by --tokens / --experts)."""
    try:
        if FFN_TRAFFIC_SOURCES_SHA256 is None or ffn_sources_sha256() != FFN_TRAFFIC_SOURCES_SHA256:
            return None
    except OSError:
        return None
    full = workloads.CONFIGS.get(cfg.name)
    if full is None or (cfg.T, cfg.E) != (full.T, full.E):
        return None
    return FFN_TRAFFIC.get(cfg.name)


def popularity_slope(cfg, counts) -> float:
    """Slope of ln(mean expert count per within-group popularity rank) against
    ln(rank) (a Zipf law p(r) ~ r^-s has slope -s); ranks with no slot are
    left out of the fit."""
    ranks = workloads.zipf_ranks(cfg)
    per = cfg.experts_per_group
    m = np.array([counts[ranks == r].mean() for r in range(1, per + 1)], dtype=np.float64)
    ok = m > 0
    return float(np.polyfit(np.log(np.arange(1, per + 1)[ok]), np.log(m[ok]), 1)[0])


def front_prefetch_bytes(cfg, touched: int) -> int:
    """Bytes of FFN weights the fused decode front asks L2 for before the FFN
    starts (its rule: the shared expert's three matrices, then the gate and up
    matrices of the first touched experts, as many whole experts as fit the
    budget SGL_MOE_PREFETCH MiB, 32 when unset); 0 when the front is not used."""
    if not fused_front(cfg):
        return 0
    v = os.environ.get("SGL_MOE_PREFETCH")
    budget = (32 << 20) if not v else max(0, int(v)) << 20
    if budget == 0:
        return 0
    shared = 3 * cfg.I_shared * cfg.H * 2
    if cfg.wfmt != workloads.MOE_W_BF16:
        return shared
    gu = 2 * cfg.I * cfg.H * 2
    return shared + min(touched, budget // gu, 33) * gu


# ------------------------------------------------------------------ GPU arm

STAGES = ("route", "permute", "gateup", "down", "combine")


DTYPES = {workloads.MOE_W_BF16: "bf16",
          workloads.MOE_W_MXFP4: "mxfp4 weights expanded to bf16",
          workloads.MOE_W_MXFP4_A8: "mxfp8 x mxfp4 (routed, block-scaled), bf16 (shared)",
          workloads.MOE_W_MXFP4_A8P: "mxfp8 x mxfp4 (routed, block-scaled, prepared scales), bf16 (shared)"}


def kernels_per_step(cfg) -> int:
    """Library kernels launched by one moe_layer_forward: for decode batches
    the fused front (routing and permutation) 1; otherwise router 3 (logits,
    certified top-k, exact re-derivation; the logits take 2 kernels, split and
    tensor-core GEMM, above 32 tokens) and permutation 1 when all T*K slots
    fit one 2048-entry tile else 3; then the expert FFN 1 and combine 1; MXFP4 adds
    2 (touched-expert list, dequantisation); the block-scaled MXFP4_A8 adds 3
    (touched-expert list, weight-scale atoms, MXFP8 x), and with prepared scale
    atoms (MXFP4_A8P) 1 (MXFP8 x)."""
    if fused_front(cfg):
        n = 1 + 1 + 1  # fused decode front (routing + permutation), FFN, combine
    else:
        n = (3 if cfg.T <= 32 else 4) + (1 if cfg.T * cfg.K <= 2048 else 3) + 1 + 1
    return n + {workloads.MOE_W_MXFP4: 2, workloads.MOE_W_MXFP4_A8: 3, workloads.MOE_W_MXFP4_A8P: 1}.get(cfg.wfmt, 0)


def fused_front(cfg) -> bool:
    """Whether the library routes and permutes a batch in one launch (its
    decode_front_ok rule; SGL_MOE_FRONT=separate turns it off)."""
    per = cfg.E // cfg.n_group
    return (os.environ.get("SGL_MOE_FRONT") != "separate" and cfg.T <= 32 and cfg.E in (128, 256, 512)
            and per in (32, 64) and cfg.n_group <= 16 and cfg.K + 1 <= 33
            and cfg.topk_group * (cfg.K + 1) <= 64 and cfg.H <= 3072 and cfg.T * cfg.K <= 2048)


def measure_gpu(cfg, steps, warmup, device, rank, clk, with_e2e=True):
    import torch

    import sigmoid_group_limited_b200 as sgl

    T = cfg.T
    d = workloads.generate(replica_config(cfg, rank), device)
    if rank:
        d["x"] = workloads.tokens(cfg, T, replica_tokens_seed(cfg, rank), device)
    if "Wg_q" in d:
        W = sgl.make_weights(d["Wg_q"], d["Wu_q"], d["Wd_q"], d["Wg_s"], d["Wu_s"], d["Wd_s"],
                             d["Wg_sc"], d["Wu_sc"], d["Wd_sc"])
        if cfg.wfmt == workloads.MOE_W_MXFP4_A8P:
            # one-time weight preparation (load time), outside every timed region
            atoms = [torch.empty_like(d[k]) for k in ("Wg_sc", "Wu_sc", "Wd_sc")]
            sgl.moe_prepare_weights(cfg, W, *atoms)
            torch.cuda.synchronize()
            d["Wg_sc"], d["Wu_sc"], d["Wd_sc"] = atoms
            W = sgl.make_weights(d["Wg_q"], d["Wu_q"], d["Wd_q"], d["Wg_s"], d["Wu_s"], d["Wd_s"],
                                 d["Wg_sc"], d["Wu_sc"], d["Wd_sc"])
    else:
        W = sgl.make_weights(d["Wg"], d["Wu"], d["Wd"], d["Wg_s"], d["Wu_s"], d["Wd_s"])
    ws = sgl.alloc_workspace(cfg, T, device)
    y = torch.empty(T, cfg.H, dtype=torch.bfloat16, device=device)
    idx = torch.empty(T, cfg.K, dtype=torch.int32, device=device)
    w = torch.empty(T, cfg.K, dtype=torch.float32, device=device)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def fwd(ev=None):
        sgl.moe_layer_forward(cfg, d["x"], d["Wr"], d["bias"], W, y, ws, idx, w, counts,
                              stream=stream, stage_events=ev)

    for _ in range(warmup):
        flush.zero_()
        fwd()
    torch.cuda.synchronize(device)
    assert sgl.moe_read_error(cfg, T, ws) == 0
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    barrier(device)
    torch.cuda.synchronize(device)
    t0 = time.perf_counter()
    with clk.timed():
        for i in range(steps):
            flush.zero_()
            fwd(evs[i])
        torch.cuda.synchronize(device)
    barrier(device)
    wall = time.perf_counter() - t0
    per_step_plain = [evs[i][0].elapsed_time(evs[i][5]) for i in range(steps)]
    stage_ms = {s: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(steps))
                for j, s in enumerate(STAGES)}
    stage_ms["ffn"] = stage_ms.pop("gateup") + stage_ms.pop("down")
    assert sgl.moe_read_error(cfg, T, ws) == 0

    # the same forward captured once into a CUDA graph and replayed per step
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(device)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side, capture_error_mode="thread_local"):
            sgl.moe_layer_forward(cfg, d["x"], d["Wr"], d["bias"], W, y, ws, idx, w, counts,
                                  stream=side)
    stream.wait_stream(side)
    for _ in range(warmup):
        flush.zero_()
        graph.replay()
    g0 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    g1 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(device)
    torch.cuda.synchronize(device)
    with clk.timed():
        for i in range(steps):
            flush.zero_()
            g0[i].record(stream)
            graph.replay()
            g1[i].record(stream)
        torch.cuda.synchronize(device)
    barrier(device)
    per_step = [g0[i].elapsed_time(g1[i]) for i in range(steps)]
    dev_ms = sum(per_step)
    assert sgl.moe_read_error(cfg, T, ws) == 0
    del graph
    # load statistics of the last step's routing, from the library (outside the timed region)
    rstats = torch.empty(sgl.MOE_N_ROUTE_STATS, dtype=torch.float64, device=device)
    sgl.moe_route_stats(cfg, counts, rstats, stream=stream)
    st = dict(zip(sgl.ROUTE_STATS_NAMES, rstats.cpu().tolist()))
    slope = popularity_slope(cfg, counts.cpu().numpy()) if cfg.bias_kind == "zipf" else None
    out = dict(device_ms_total=dev_ms, plain_ms_total=sum(per_step_plain), wall_s=wall,
               per_step_ms=per_step, stage_ms=stage_ms,
               routing={"experts_touched": cfg.E - int(st["idle_experts"]),
                        "idle_experts": int(st["idle_experts"]), "load_max": int(st["load_max"]),
                        "load_mean": round(st["load_mean"], 2),
                        "max_over_mean": round(st["max_over_mean"], 3),
                        "entropy_bits": round(st["entropy_bits"], 4),
                        "entropy_normalized": round(st["entropy_normalized"], 4),
                        **({"popularity_slope": round(slope, 3),
                            "popularity_slope_fit": "least squares of ln(mean count per "
                                                    "within-group rank) on ln(rank), ranks 1..E/G, "
                                                    "from the library's expert counts; target -zipf_s"}
                           if slope is not None else {})},
               d=d, launches=kernels_per_step(cfg) * 2 * steps)

    if with_e2e:
        # end to end through the public API: pinned host x -> device, forward, y -> pinned host
        xh = d["x"].cpu().pin_memory()
        yh = torch.empty(T, cfg.H, dtype=torch.bfloat16).pin_memory()
        xd = torch.empty_like(d["x"])
        e0 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        e1 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        for i in range(warmup):
            xd.copy_(xh, non_blocking=True)
            sgl.moe_layer_forward(cfg, xd, d["Wr"], d["bias"], W, y, ws, stream=stream)
            yh.copy_(y, non_blocking=True)
        torch.cuda.synchronize(device)
        with clk.timed():
            for i in range(steps):
                flush.zero_()
                e0[i].record(stream)
                xd.copy_(xh, non_blocking=True)
                sgl.moe_layer_forward(cfg, xd, d["Wr"], d["bias"], W, y, ws, stream=stream)
                yh.copy_(y, non_blocking=True)
                e1[i].record(stream)
            torch.cuda.synchronize(device)
        out["e2e_ms_total"] = sum(e0[i].elapsed_time(e1[i]) for i in range(steps))
        out["launches"] += kernels_per_step(cfg) * steps
        out["e2e_h2d"] = T * cfg.H * 2
        out["e2e_d2h"] = T * cfg.H * 2
        assert torch.equal(yh.view(torch.int16), y.cpu().view(torch.int16))
    del flush
    return out


# ------------------------------------------------------------------ oracle (CPU) arm

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_inputs(d):
    """Host copies of the inputs (bytes as the GPU sees them)."""
    import torch

    def b16(t):
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    if "Wg_q" in d:
        import oracle

        def experts(e):
            q = lambda k: d[k][e].cpu().numpy()  # noqa: E731
            return (oracle.mxfp4_dequantize(q("Wg_q"), q("Wg_sc")),
                    oracle.mxfp4_dequantize(q("Wu_q"), q("Wu_sc")),
                    oracle.mxfp4_dequantize(q("Wd_q"), q("Wd_sc")))
        fmt = "mxfp4"
    else:
        def experts(e):
            return b16(d["Wg"][e]), b16(d["Wu"][e]), b16(d["Wd"][e])
        fmt = "bf16"
    return dict(x=b16(d["x"]), Wr=d["Wr"].cpu().numpy(), bias=d["bias"].cpu().numpy(),
                Wg_s=b16(d["Wg_s"]), Wu_s=b16(d["Wu_s"]), Wd_s=b16(d["Wd_s"]),
                experts=experts, fmt=fmt)


def time_oracle(cfg, h, tokens):
    """Oracle layer forward for `tokens` of the batch (routing covers the batch);
    the touched experts' weights are fetched to host before the clock starts."""
    import oracle
    r = oracle.route(h["x"], h["Wr"], h["bias"], cfg.n_group, cfg.topk_group, cfg.K)
    need = sorted(set(int(e) for e in r["idx"][tokens].reshape(-1)))
    host = {e: h["experts"](e) for e in need}

    def ew(e):
        g, u, dd = host[e]
        if h["fmt"] == "mxfp4":
            return g, u, dd
        f = oracle.bf16_bits_to_f64
        return f(g), f(u), f(dd)
    # prepared scale atoms only re-lay the scale bytes: the oracle's arithmetic
    # is that of the block-scaled format on the raw scales
    ocfg = cfg.with_(wfmt=workloads.MOE_W_MXFP4_A8) if cfg.wfmt == workloads.MOE_W_MXFP4_A8P else cfg
    t0 = time.perf_counter()
    oracle.layer_forward(ocfg, h["x"], h["Wr"], h["bias"], ew, h["Wg_s"], h["Wu_s"], h["Wd_s"],
                         tokens=tokens)
    return time.perf_counter() - t0


def oracle_sample_tokens(cfg, step: int, n: int):
    return np.array([(step * n + i) % cfg.T for i in range(n)])


# ------------------------------------------------------------------ main

def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode", choices=sorted(workloads.CONFIGS))
    ap.add_argument("--also", default="prefill,prefill_bias0,zipf,mxfp4,mxfp4_a8",
                    help="further workloads for the line, comma-separated ('' = none)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--oracle-tokens", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the workload's T (small profiling cases)")
    ap.add_argument("--experts", type=int, default=0,
                    help="override the workload's E (small profiling cases; E %% n_group == 0)")
    return ap.parse_args()


def workload_cfg(args):
    cfg = workloads.CONFIGS[args.workload]
    if args.tokens > 0:
        cfg = cfg.with_(T=args.tokens)
    if args.experts > 0:
        cfg = cfg.with_(E=args.experts)
    return cfg


WORKLOAD_NOTES = {
    "decode": "decode batch, bias N(0, 0.1) (memory-bound)",
    "prefill": "prefill batch, bias N(0, 0.1): skewed loads, about 122 experts touched",
    "prefill_bias0": "prefill batch with zero bias: near-uniform loads over all 512 experts "
                     "(memory-bound: 6 GB of weights)",
    "zipf": "skewed routing: bias calibrated so that expert popularity inside each group "
            "follows p(r) ~ r^-1.1; SwiGLU limits 4 (routed) / 7 (shared)",
    "mxfp4": "routed weights MXFP4 (e2m1 codes + e8m0 scale per 32); activations, router and "
             "shared expert bf16/fp32",
    "mxfp4_a8": "block-scaled variant: MXFP4 routed weights x MXFP8 routed activations "
                "(narrower activation arithmetic than the bf16-activation mxfp4 workload)",
    "mxfp4_a8p": "block-scaled variant with weight scales prepared once (load time)",
}


def config_block(cfg, world):
    return {"workload": f"{cfg.name} ({WORKLOAD_NOTES.get(cfg.name, 'custom')}): "
                        f"T={cfg.T} tokens per GPU, H={cfg.H}, E={cfg.E} experts "
                        f"({cfg.n_group} groups keep {cfg.topk_group}, top-{cfg.K}), I={cfg.I}, "
                        f"shared I={cfg.I_shared}",
            "T": cfg.T, "H": cfg.H, "E": cfg.E, "n_group": cfg.n_group,
            "topk_group": cfg.topk_group, "K": cfg.K, "I": cfg.I, "I_shared": cfg.I_shared,
            "bias": cfg.bias_kind, "limits": [cfg.limit_routed, cfg.limit_shared],
            "global_batch": cfg.T * world, "parallelism": f"replicas x{world} (tokens sharded, no collective)",
            "l2": "flushed before every step (256 MB write, outside the step events)"}


def run_reference(args, rank, world):
    cfg = workload_cfg(args)
    if rank != 0:
        return
    import torch
    dev = "cuda:0" if torch.cuda.is_available() else "cpu"
    d = workloads.generate(cfg, dev)
    h = oracle_inputs(d)
    n = min(args.oracle_tokens, cfg.T)
    for i in range(args.warmup):
        time_oracle(cfg, h, oracle_sample_tokens(cfg, i, n))
    ts = [time_oracle(cfg, h, oracle_sample_tokens(cfg, args.warmup + i, n)) for i in range(args.steps)]
    tot = sum(ts)
    value = n * args.steps / tot
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * tot / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(cfg, 1),
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": blas_threads(),
                             "kind": "oracle",
                             "sample": f"{n} tokens of the {cfg.T}-token batch per step (routing "
                                       f"of the whole batch + their {cfg.K} experts and the shared "
                                       f"expert, numpy float64)"},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_native(args, rank, world, local):
    import torch
    device = f"cuda:{local}"
    torch.cuda.set_device(device)
    peaks = load_peaks()
    cfg = workload_cfg(args)
    # tensor-core instruction throughput per kind on this GPU (about a second)
    try:
        from sigmoid_group_limited_b200 import peak as tcprobe
        probe = tcprobe.peaks(device)
    except Exception as exc:  # the line then says the ratios are nominal
        print(f"tensor-core probe unavailable: {exc}", file=sys.stderr)
        probe = None
    ratios = tensor_ratios(probe)
    with ClockSampler(device) as clk:
        m = measure_gpu(cfg, args.steps, args.warmup, device, rank, clk)
        also = []
        for name in [a for a in args.also.split(",") if a and a != args.workload]:
            acfg = workloads.CONFIGS[name]
            am = measure_gpu(acfg, args.steps, args.warmup, device, rank, clk, with_e2e=False)
            am.pop("d")                          # free this workload's weights before the next
            torch.cuda.empty_cache()
            also.append((acfg, am))
    clocks = clk.summary()
    dev_s = reduce_max(m["device_ms_total"], device) / 1e3
    plain_s = reduce_max(m["plain_ms_total"], device) / 1e3
    e2e_s = reduce_max(m["e2e_ms_total"], device) / 1e3
    tokens = cfg.T * args.steps * world

    def roof(cfg_, mm):
        work = algorithmic_work(cfg_, cfg_.T, mm["routing"]["experts_touched"])
        # the dominant kernel is the fused expert FFN (gate/up and down in one launch)
        b = work["gateup"][0] + work["down"][0]
        f = work["gateup"][1] + work["down"][1]
        t_ffn = (mm["stage_ms"]["ffn"]) / 1e3
        mx = cfg_.wfmt in (workloads.MOE_W_MXFP4_A8, workloads.MOE_W_MXFP4_A8P)
        # block-scaled: the routed experts' flops run at the fp8 rate, the shared expert's at bf16
        f_routed = 2.0 * cfg_.T * cfg_.K * 3 * cfg_.H * cfg_.I
        f8 = f_routed if mx else 0.0
        ent = roofline_entry(b, f, t_ffn, peaks, fp8_flops=f8, fp8_ratio=ratios["fp8"])
        src = "HBM copy" if ent["bound"] == "hbm" else (
            f"cuBLAS bf16 burst; routed MXFP8 x MXFP4 flops at {ratios['fp8']:.3f} x that "
            f"({ratios['source']} kind::mxf8f6f4 / kind::f16 ratio)" if mx else "cuBLAS bf16 burst")
        tr = ffn_traffic(cfg_)
        ent.update(kernel="moe_ffn_mx (block-scaled gate/up + down)" if mx else "moe_ffn (gate/up + down)",
                   traffic=(tr[0] + tr[1]) if tr else None,
                   traffic_unit="bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum, "
                                "one-pass capture of this workload at full size)",
                   peak_source=f"{peaks['source']} ({src})",
                   units_per_launch=f"{cfg_.T} tokens, {mm['routing']['experts_touched']} routed experts + shared")
        if tr:
            ent["traffic_read"], ent["traffic_write"] = tr
            ent["traffic_over_algorithmic"] = round((tr[0] + tr[1]) / b, 3)
            # the fp32 slot rows every token writes once: (T*K + T) rows of H floats
            ent["y_slot_bytes"] = (cfg_.T * cfg_.K + cfg_.T) * cfg_.H * 4
        if mx:
            ent["time"] = "FFN stage events: scale atoms and MXFP8 x included"
        if cfg_.wfmt != workloads.MOE_W_BF16:
            # the routed flops against the dense FP4 peak (kind::mxf4, e2m1 x e2m1)
            fp4_peak = peaks["bf16_tflops"] * ratios["fp4"]
            ent["fp4_peak_tflops"] = round(fp4_peak, 1)
            ent["frac_of_fp4_peak"] = round(f_routed / t_ffn / 1e12 / fp4_peak, 4)
            ent["fp4_peak_source"] = f"cuBLAS bf16 burst x {ratios['fp4']:.3f} ({ratios['source']} " \
                                     f"kind::mxf4 / kind::f16 ratio)"
        pf = front_prefetch_bytes(cfg_, mm["routing"]["experts_touched"])
        if ent["bound"] == "hbm" and pf > 0:
            # the fused front asks L2 for these bytes while routing runs; net of
            # them, the FFN's own HBM rate is
            net = (b - pf) / t_ffn / 1e9
            ent["l2_prefetched_bytes"] = pf
            ent["frac_net_of_l2_prefetch"] = round(net / peaks["hbm_gbs"], 4)
        lb, lf = work["layer"]
        tp = peaks["bf16_tflops"] * 1e12
        t_roof = max(lb / (peaks["hbm_gbs"] * 1e9), (lf - f8) / tp + f8 / (ratios["fp8"] * tp))
        step_s = statistics.mean(mm["per_step_ms"]) / 1e3
        return ent, round(t_roof / step_s, 4)

    ent, layer_frac = roof(cfg, m)
    line = {"metric": METRIC, "value": round(tokens / dev_s, 1), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * dev_s / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": DTYPES.get(cfg.wfmt, "bf16"), "data": "synthetic",
            "timing": "CUDA-event time of K graph replays of moe_layer_forward (one capture of "
                      "the C-ABI call); value_no_graph: the same K steps as plain C-ABI calls",
            "value_no_graph": round(tokens / plain_s, 1),
            "config": config_block(cfg, world), "roofline": ent,
            "layer_roofline_frac": layer_frac,
            "stage_ms": {k: round(v, 4) for k, v in m["stage_ms"].items()},
            "routing": m["routing"],
            "e2e": {"value": round(tokens / e2e_s, 1), "unit": "tokens/s",
                    "h2d_bytes_per_step": m["e2e_h2d"], "d2h_bytes_per_step": m["e2e_d2h"]},
            "gpu_launches": m["launches"], "clocks": clocks,
            "tensor_probe": ({k: {"tflops": round(v["tflops"], 1), "ns_per_mma": round(v["ns_per_mma"], 2),
                                  "shape": f"M=128 N={v['N']} K={v['K']}, {v['chains']} accumulator(s)"}
                              for k, v in probe.items()} if probe else None),
            "tensor_ratios": {"fp8_over_bf16": round(ratios["fp8"], 4),
                              "fp4_over_bf16": round(ratios["fp4"], 4), "source": ratios["source"]}}
    for acfg, am in also:
        a_s = reduce_max(am["device_ms_total"], device) / 1e3
        aent, afrac = roof(acfg, am)
        ap_s = reduce_max(am["plain_ms_total"], device) / 1e3
        line[acfg.name] = {"value": round(acfg.T * args.steps * world / a_s, 1), "unit": "tokens/s",
                           "value_no_graph": round(acfg.T * args.steps * world / ap_s, 1),
                           "ms_per_step": round(1e3 * a_s / args.steps, 4), "roofline": aent,
                           "layer_roofline_frac": afrac,
                           "stage_ms": {k: round(v, 4) for k, v in am["stage_ms"].items()},
                           "routing": am["routing"],
                           "dtype": DTYPES.get(acfg.wfmt, "bf16"),
                           "config": config_block(acfg, world)}
        line["gpu_launches"] += am["launches"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        h = oracle_inputs(m["d"])
        n = min(args.oracle_tokens, cfg.T)
        t = time_oracle(cfg, h, oracle_sample_tokens(cfg, 0, n))
        line["cpu_baseline"] = {"value": round(n / t, 3), "unit": "tokens/s", "cores": blas_threads(),
                                "kind": "oracle",
                                "sample": f"{n} of the {cfg.T} tokens (routing of the whole batch, "
                                          f"their experts and the shared expert; numpy float64)"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.gpus != world and world > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    dist_init(world, "nccl")
    try:
        run_native(args, rank, world, local)
    finally:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
