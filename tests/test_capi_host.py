"""The C-ABI library without a GPU: it loads, exports every function that
include/moe.h declares, sizes workspaces, and rejects bad arguments on the
host (before any launch)."""
import ctypes
import os
import re

import pytest

import sigmoid_group_limited_b200 as sgl
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return set(re.findall(r"MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(", src))


def test_library_exports_every_declared_function():
    L = sgl.lib()
    decl = _declared()
    assert decl == set(sgl.C_FUNCTIONS)
    for name in decl:
        assert hasattr(L, name), name
    assert "sm_100a" in sgl.version()


def test_status_strings():
    L = sgl.lib()
    for code, name in sgl.STATUS.items():
        assert L.moe_status_string(code).decode().startswith(name)


def test_workspace_size_full_configs():
    for name in ("decode", "prefill", "zipf"):
        cfg = workloads.CONFIGS[name]
        n = sgl.workspace_size(cfg, cfg.T)
        # dominated by y_slot: (T*K + T) rows of H fp32, plus h (T*K rows of I bf16)
        lower = (cfg.T * cfg.K + cfg.T) * cfg.H * 4 + cfg.T * cfg.K * cfg.I * 2
        assert lower <= n <= lower * 1.5 + (64 << 20)


@pytest.mark.parametrize("field,value", [("H", 100), ("E", 48), ("n_group", 3), ("topk_group", 9),
                                         ("K", 0), ("K", 33), ("I", 96), ("I_shared", -64),
                                         ("wfmt", 7), ("scale", float("nan"))])
def test_bad_config_rejected(field, value):
    cfg = workloads.CONFIGS["decode"].with_(**{field: value})
    c = sgl.make_cfg(cfg)
    assert sgl.lib().moe_workspace_size(ctypes.byref(c), 32) == 0
    st = sgl.lib().moe_route(ctypes.byref(c), 32, 16, 16, None, 16, 16, 16, 1 << 30, None)
    assert st == -1


def test_bad_token_count_rejected():
    c = sgl.make_cfg(workloads.CONFIGS["decode"])
    for T in (0, -1, (1 << 20) + 1):
        assert sgl.lib().moe_workspace_size(ctypes.byref(c), T) == 0
        assert sgl.lib().moe_permute(ctypes.byref(c), T, 16, 16, 16, 16, 16, 16, 1 << 30, None) == -1


def test_null_misaligned_and_small_workspace_rejected_before_launch():
    L = sgl.lib()
    cfg = workloads.CONFIGS["decode"]
    c = sgl.make_cfg(cfg)
    need = sgl.workspace_size(cfg, 32)
    A = 1 << 20  # fake, aligned "device" addresses: never dereferenced on these paths
    assert L.moe_route(ctypes.byref(c), 32, None, A, None, A, A, A, need, None) == -2
    assert L.moe_route(ctypes.byref(c), 32, A + 2, A, None, A, A, A, need, None) == -3
    assert L.moe_route(ctypes.byref(c), 32, A, A, None, A, A, A, need - 1, None) == -4
    assert L.moe_route(ctypes.byref(c), 32, A, A, None, A, None, A, need, None) == -2
    assert L.moe_route(ctypes.byref(c), 32, A, A, None, A, A, None, need, None) == -4
    w = sgl.moe_weights(A, A, A, None, None, None, A, A, None)   # shared Wd missing
    assert L.moe_layer_forward(ctypes.byref(c), 32, A, A, None, ctypes.byref(w), A, None, None,
                               None, A, need, None, None) == -2
    w = sgl.moe_weights(A, A + 8, A, None, None, None, A, A, A)
    assert L.moe_layer_forward(ctypes.byref(c), 32, A, A, None, ctypes.byref(w), A, None, None,
                               None, A, need, None, None) == -3
    assert L.moe_combine(ctypes.byref(c), 32, None, 1, A, None) == -2
    assert L.moe_grouped_swiglu(ctypes.byref(c), 32, A, A, A, A, None, A, A, need, None) == -2


def test_block_scaled_format_validation():
    """MOE_W_MXFP4_A8 needs H and I multiples of 128 and 32-byte aligned codes."""
    L = sgl.lib()
    full = workloads.CONFIGS["mxfp4_a8"]
    assert sgl.workspace_size(full, 32) > 0
    assert sgl.workspace_size(workloads.CONFIGS["tiny_a8"], 64) > 0
    assert L.moe_workspace_size(ctypes.byref(sgl.make_cfg(full.with_(I=704))), 32) == 0
    assert L.moe_workspace_size(ctypes.byref(sgl.make_cfg(full.with_(H=2496))), 32) == 0
    assert L.moe_workspace_size(ctypes.byref(sgl.make_cfg(full.with_(wfmt=4))), 32) == 0
    # the prepared variant takes the same shapes and needs no per-call scale atoms
    prep = full.with_(wfmt=workloads.MOE_W_MXFP4_A8P)
    assert 0 < sgl.workspace_size(prep, 32) < sgl.workspace_size(full, 32)
    assert L.moe_workspace_size(ctypes.byref(sgl.make_cfg(prep.with_(I=704))), 32) == 0
    c = sgl.make_cfg(full)
    need = sgl.workspace_size(full, 32)
    A = 1 << 20
    w = sgl.moe_weights(A, A + 16, A, A, A, A, A, A, A)         # 16- but not 32-byte aligned codes
    assert L.moe_layer_forward(ctypes.byref(c), 32, A, A, None, ctypes.byref(w), A, None, None,
                               None, A, need, None, None) == -3
    w = sgl.moe_weights(A, A, A, None, A, A, A, A, A)           # a scale array missing
    assert L.moe_layer_forward(ctypes.byref(c), 32, A, A, None, ctypes.byref(w), A, None, None,
                               None, A, need, None, None) == -2


def test_prepare_weights_validation():
    """moe_prepare_weights: block-scaled formats only, every pointer present
    and 16-byte aligned; all checked on the host before any device work."""
    L = sgl.lib()
    A = 1 << 20
    full = workloads.CONFIGS["mxfp4_a8"]
    w = sgl.moe_weights(A, A, A, A, A, A, A, A, A)
    for bad in (workloads.CONFIGS["prefill"], workloads.CONFIGS["mxfp4"], full.with_(I=704)):
        assert L.moe_prepare_weights(ctypes.byref(sgl.make_cfg(bad)), ctypes.byref(w), A, A, A, None) == -1
    c = sgl.make_cfg(full)
    assert L.moe_prepare_weights(ctypes.byref(c), None, A, A, A, None) == -2
    assert L.moe_prepare_weights(ctypes.byref(c), ctypes.byref(w), A, None, A, None) == -2
    no_scale = sgl.moe_weights(A, A, A, A, None, A, A, A, A)
    assert L.moe_prepare_weights(ctypes.byref(c), ctypes.byref(no_scale), A, A, A, None) == -2
    assert L.moe_prepare_weights(ctypes.byref(c), ctypes.byref(w), A, A, A + 8, None) == -3
    odd = sgl.moe_weights(A, A, A, A, A + 4, A, A, A, A)
    assert L.moe_prepare_weights(ctypes.byref(c), ctypes.byref(odd), A, A, A, None) == -3


def test_peak_probe_library_loads_and_checks_arguments():
    """The tensor-core throughput probe (a separate library) exports its entry
    point and refuses bad shapes on the host, before any CUDA call."""
    from sigmoid_group_limited_b200 import peak
    L = peak.lib()
    status = ctypes.c_void_p(1 << 20)  # never dereferenced: every call below is refused first
    for args in ((3, 256, 1, 10, 148, 0), (0, 8, 1, 10, 148, 0), (1, 264, 1, 10, 148, 0),
                 (2, 136, 3, 10, 148, 0), (0, 128, 1, 0, 148, 0), (0, 128, 1, 10, 0, 0),
                 (0, 256, 3, 10, 148, 0), (0, 256, 2, 10, 148, 1), (0, 128, 2, 10, 148, 3),
                 (0, 128, 2, 10, 148, 32)):
        assert L.sgl_mma_peak(*args, status, None) == 1          # cudaErrorInvalidValue
    assert L.sgl_mma_peak(0, 128, 1, 10, 148, 0, None, None) == 1   # no status word
    assert set(peak.KINDS) == {"bf16", "e2m1xe4m3", "e2m1xe2m1"}
