"""moe_permute_static: the permutation for callers that cannot allocate device
memory (for example a plugin whose host framework owns all device memory and
offers no workspace, or a real-time loop that must not allocate). Its scratch
lives in a fixed array inside the library instead of a caller-provided
workspace. It must give exactly what moe_permute gives, and what the oracle's
stable counting sort gives.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import sigmoid_group_limited_b200 as sgl
import workloads

CFG = workloads.CONFIGS["prefill"]   # 512 experts, 8 groups, K = 8


def _outputs(T, fill, cfg=CFG):
    n = T * cfg.K
    return [torch.full((m,), fill, dtype=torch.int32, device="cuda")
            for m in (cfg.E, cfg.E + 1, n, n)]


@pytest.mark.gpu
def test_static_permutation_equals_workspace_permutation_twice():
    # two calls in a row on the shared static scratch, with different sizes and loads
    for T, skew, seed in ((4096, False, 1), (300, True, 2)):
        g = torch.Generator().manual_seed(seed)
        if skew:
            idx = torch.randint(0, 4, (T, CFG.K), generator=g, dtype=torch.int32)
        else:
            idx = torch.randint(0, CFG.E, (T, CFG.K), generator=g, dtype=torch.int32)
        idx = idx.cuda()
        ws = sgl.alloc_workspace(CFG, T)
        ref = _outputs(T, -1)
        sgl.moe_permute(CFG, T, idx, *ref, ws)
        got = _outputs(T, -7)
        sgl.moe_permute_static(CFG, T, idx, *got)
        torch.cuda.synchronize()
        for r, o in zip(ref, got):       # integer work: bit-exact
            assert torch.equal(r, o)
        counts = np.bincount(idx.cpu().numpy().reshape(-1), minlength=CFG.E)
        assert np.array_equal(got[0].cpu().numpy(), counts)
        for o, r in zip(got, oracle.permute(idx.cpu().numpy(), CFG.E)):
            assert np.array_equal(o.cpu().numpy(), r)


@pytest.mark.gpu
@pytest.mark.parametrize("E", [512, 1024])
def test_static_permutation_at_its_size_limit(E):
    """T*K = 65536 slots (the largest the scratch takes) with 512 and 1024
    experts: every per-(expert, tile) count and base of the scratch is used."""
    cfg = CFG.with_(E=E)
    T = 65536 // cfg.K
    g = torch.Generator().manual_seed(E)
    idx = torch.randint(0, E, (T, cfg.K), generator=g, dtype=torch.int32)
    idx[: T // 2, 0] = E - 1                          # one heavy expert at the top of the range
    idx = idx.cuda()
    ws = sgl.alloc_workspace(cfg, T)
    ref = _outputs(T, -1, cfg)
    sgl.moe_permute(cfg, T, idx, *ref, ws)
    got = _outputs(T, -7, cfg)
    sgl.moe_permute_static(cfg, T, idx, *got)
    torch.cuda.synchronize()
    for r, o, p in zip(ref, got, oracle.permute(idx.cpu().numpy(), E)):
        assert torch.equal(r, o)
        assert np.array_equal(o.cpu().numpy(), p)


def test_static_permutation_rejects_sizes_beyond_its_scratch():
    L = sgl.lib()
    c = sgl.make_cfg(CFG)
    A = 1 << 20  # aligned fake addresses: the call must refuse before touching them
    T = 65536 // CFG.K + 1
    st = L.moe_permute_static(ctypes.byref(c), T, A, A, A, A, A, None)
    assert st == -4                                   # MOE_ERR_WORKSPACE
    with pytest.raises(sgl.MoEError):
        sgl._check(st, "moe_permute_static")
