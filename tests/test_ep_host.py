"""Expert parallelism (sigmoid_group_limited_b200.ep) on CPU ranks: two and
four gloo processes, each routing its own token batch, exchange (token,
slot) rows with all-to-all-v, run their own expert block, and combine. The
local compute is the oracle's, so the exchange is what is tested: every
rank's output must equal the single-process oracle layer on its batch, bit
for bit (rows return to their slots and are summed in slot order). The
per-layer SwiGLU limit list is checked here too."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import workloads
from sigmoid_group_limited_b200 import ep


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


class OracleOps:
    """ep_forward's local compute with the oracle's arithmetic."""

    def __init__(self, cfg, d, rank, world):
        self.cfg = cfg
        self.d = d
        self.e0, _ = ep.expert_block(cfg.E, cfg.n_group, world, rank)
        f = oracle.bf16_bits_to_f64
        self.W = [(f(_bits(d["Wg"][e])), f(_bits(d["Wu"][e])), f(_bits(d["Wd"][e]))) for e in range(cfg.E)]

    def route(self, x):
        c = self.cfg
        r = oracle.route(_bits(x), self.d["Wr"].numpy(), self.d["bias"].numpy(), c.n_group, c.topk_group,
                         c.K, c.scale, c.renorm)
        return torch.from_numpy(r["idx"]), torch.from_numpy(r["w"])

    def experts(self, x_in, ids, w):
        c = self.cfg
        x64 = oracle.bf16_bits_to_f64(x_in.numpy().view(np.uint16))
        out = np.zeros((x_in.shape[0], c.H), np.float32)
        ids, w = ids.numpy(), w.numpy()
        for e in np.unique(ids):
            rows = np.nonzero(ids == e)[0]
            o, _ = oracle.swiglu_expert(x64[rows], *self.W[self.e0 + int(e)], c.limit_routed)
            out[rows] = (w[rows][:, None].astype(np.float32) * o).astype(np.float32)
        return torch.from_numpy(out)

    def combine(self, x, y_slot):
        c = self.cfg
        T = x.shape[0]
        f = oracle.bf16_bits_to_f64
        o_sh, _ = oracle.swiglu_expert(f(_bits(x)), f(_bits(self.d["Wg_s"])), f(_bits(self.d["Wu_s"])),
                                       f(_bits(self.d["Wd_s"])), c.limit_shared)
        ys = y_slot.numpy().reshape(T, c.K, c.H)
        acc = np.zeros((T, c.H), np.float32)
        for k in range(c.K):
            acc = (acc + ys[:, k]).astype(np.float32)
        acc = (acc + o_sh).astype(np.float32)
        return torch.from_numpy(oracle.f32_to_bf16_bits(acc).view(np.int16))


def _worker(rank, world, port, cfg, T, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        d = workloads.generate(cfg, "cpu", T=T)
        x = workloads.tokens(cfg, T, rank, "cpu")            # this rank's own batch
        y = ep.ep_forward(cfg, x, OracleOps(cfg, d, rank, world))
        ref = oracle.layer_forward(cfg, _bits(x), d["Wr"].numpy(), d["bias"].numpy(),
                                   oracle.dense_expert_weights(_bits(d["Wg"]), _bits(d["Wu"]), _bits(d["Wd"])),
                                   _bits(d["Wg_s"]), _bits(d["Wu_s"]), _bits(d["Wd_s"]))
        same = bool(np.array_equal(y.numpy().view(np.uint16), ref["y"]))
        counts = np.bincount(ref["idx"].reshape(-1) // (cfg.E // world), minlength=world).tolist()
        q.put((rank, same, counts))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,T,variant", [(2, 40, {}), (2, 7, dict(limit_routed=0.5, limit_shared=0.7)),
                                             (4, 33, {})])
def test_expert_parallel_equals_single_process(world, T, variant):
    cfg = workloads.CONFIGS["tiny"].with_(**variant)          # 4 groups of 8 experts
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, world, port, cfg, T, q)) for r in range(world)]
    for p in ps:
        p.start()
    out = sorted(q.get(timeout=300) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [True] * world
    # the batches reach more than one rank (the exchange is exercised)
    assert all(sum(1 for c in o[2] if c > 0) > 1 for o in out)


def test_expert_blocks_follow_the_groups():
    assert ep.expert_block(512, 8, 8, 3) == (192, 256)       # one group of 64 per rank
    assert ep.expert_block(512, 8, 2, 1) == (256, 512)
    with pytest.raises(ValueError):
        ep.expert_block(512, 8, 3, 0)


def test_layer_limits_list():
    """Page 3 sec. 4: +-4 on the routed experts of the last 6 of the 40 MoE
    layers, +-5 / +-7 on the shared expert there; no limit elsewhere."""
    lim = [ep.layer_limits(l) for l in range(40)]
    assert all(l == (0.0, 0.0) for l in lim[:34])
    assert [l[0] for l in lim[34:]] == [4.0] * 6
    assert [l[1] for l in lim[34:]] == [5.0, 5.0, 5.0, 7.0, 7.0, 7.0]
    seen = []
    ep.stack_forward(lambda l, x, lr, ls: seen.append((l, lr, ls)) or x + 1, 0, n_layers=4, first_layer=33)
    assert seen == [(33, 0.0, 0.0), (34, 4.0, 5.0), (35, 4.0, 5.0), (36, 4.0, 5.0)]
    with pytest.raises(ValueError):
        ep.layer_limits(40)
