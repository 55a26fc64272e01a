"""The expert-parallel layer's library-backed local compute (ep.LibraryOps)
on one GPU: a process group of one rank (NCCL), so the exchange is a copy to
itself and every pair runs through moe_permute + moe_grouped_swiglu with one
slot per token, the shared expert and moe_combine. Each pair's row depends
only on its token, expert and weight, so the result equals the whole-layer
call bit for bit. Runs on one GPU; more ranks are covered on CPU ranks in
test_ep_host.py."""
import os
import socket

import numpy as np
import pytest
import torch

import workloads
from helpers import bits, run_layer
from sigmoid_group_limited_b200 import ep

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.mark.parametrize("T,variant", [(200, {}), (600, dict(limit_routed=0.5, limit_shared=0.7))])
def test_library_ops_single_rank_equals_layer(T, variant):
    import torch.distributed as dist
    cfg = workloads.CONFIGS["tiny"].with_(**variant)
    d = workloads.generate(cfg, "cuda", T=T)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        ops = ep.LibraryOps(cfg, 0, 1, d["Wr"], d["bias"], d["Wg"], d["Wu"], d["Wd"], d["Wg_s"],
                            d["Wu_s"], d["Wd_s"])
        y = ep.ep_forward(cfg, d["x"], ops)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref = run_layer(cfg, d)
    assert np.array_equal(bits(y), bits(ref["y"]))
