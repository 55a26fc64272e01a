"""Expert parallelism for the MoE layer, and the per-layer SwiGLU limit list.

Expert parallelism (one process per GPU, torch.distributed for the exchange).
Page "Ling-3.0-flash-VL MoE sparse routing" (lqnn.cn/news/282163), sec. 3
step 2: a token's experts come from at most topk_group of the n_group
groups. Rank r of W holds the routed experts of groups
[r*G/W, (r+1)*G/W), a contiguous block of E/W experts, plus the router and
the shared expert (both small, replicated); every rank routes its own token
batch. A forward is

  1. route the rank's tokens (idx, w);
  2. dispatch: every (token, slot) pair goes to the rank that owns its
     expert - one all-to-all-v of the pairs' token rows (bf16 bits, sent as
     32-bit words), local expert ids and routing weights, pairs ordered by
     (destination rank, flat slot j = t*K + k);
  3. every rank runs its experts on the pairs it received, producing
     w * Expert(x) per pair (fp32);
  4. combine: one all-to-all-v sends each pair's row back to the rank of its
     token, where it lands at row j of the slot buffer; the shared expert's
     rows and the fp32 sum over k in slot order follow, as on one GPU.

Because a pair's row depends only on its own token, expert and weight, and
the final sum runs in the same order as on one GPU, the result equals the
single-GPU layer's bit for bit when the local compute is the same. The
exchange carries one row per pair each way (eight rows per token), not the
per-rank partial sums: that keeps the sum order of the single-GPU combine.

The arithmetic runs in an `ops` object: `LibraryOps` calls the library's
C-ABI on the GPU (routing, permutation + grouped SwiGLU of the received
pairs, shared expert and combine); the CPU tests pass the oracle's
functions. This module only moves rows between ranks.

Not measured on hardware: every run here has one GPU.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist


# ------------------------------------------------------------------ per-layer limits

def layer_limits(layer: int, n_moe_layers: int = 40) -> Tuple[float, float]:
    """SwiGLU limits (routed, shared) of MoE layer `layer` (0-based) of
    `n_moe_layers`. Page "Ling-3.0-flash-VL MoE sparse routing", sec. 4: the
    config's expert_swiglu_limit_list clamps the routed experts to +-4 in the
    last 6 layers, and the shared expert to +-5/+-7 there. Reading: the first
    three of those six layers clamp the shared expert to 5, the last three to
    7; every other layer has no limit (0.0)."""
    if not 0 <= layer < n_moe_layers:
        raise ValueError(f"layer {layer} outside 0..{n_moe_layers - 1}")
    first = n_moe_layers - 6
    if layer < first:
        return 0.0, 0.0
    return 4.0, (5.0 if layer < first + 3 else 7.0)


def stack_forward(layer_fn, x, n_layers: int, n_moe_layers: int = 40, first_layer: int = 0):
    """Runs `n_layers` consecutive MoE layers starting at `first_layer`, each
    with its limits from layer_limits: x <- layer_fn(l, x, limit_routed,
    limit_shared). layer_fn holds the layer's weights and calls the library
    (or, in tests, the oracle)."""
    for l in range(first_layer, first_layer + n_layers):
        lr, ls = layer_limits(l, n_moe_layers)
        x = layer_fn(l, x, lr, ls)
    return x


# ------------------------------------------------------------------ expert parallelism

def expert_block(E: int, n_group: int, world: int, rank: int) -> Tuple[int, int]:
    """Experts [e0, e1) held by `rank`: the groups [rank*G/W, (rank+1)*G/W)."""
    if n_group % world != 0:
        raise ValueError(f"{n_group} groups do not split over {world} ranks")
    per = E // world
    return rank * per, (rank + 1) * per


def _exchange(send: torch.Tensor, send_counts, recv_counts, group) -> torch.Tensor:
    """all-to-all-v of the rows of `send` (split by send_counts) -> the rows
    every rank sent here (split by recv_counts)."""
    out = torch.empty((sum(recv_counts),) + tuple(send.shape[1:]), dtype=send.dtype,
                      device=send.device)
    dist.all_to_all_single(out, send.contiguous(), list(recv_counts), list(send_counts), group=group)
    return out


def ep_forward(cfg, x: torch.Tensor, ops, group: Optional[dist.ProcessGroup] = None) -> torch.Tensor:
    """One expert-parallel layer forward of this rank's tokens x [T, H]
    (bf16, or its 16-bit words). Returns y [T, H] as produced by
    ops.combine (bf16 on the GPU, 16-bit words in the CPU tests)."""
    world = dist.get_world_size(group)
    T, K, E = x.shape[0], cfg.K, cfg.E
    per = E // world
    expert_block(E, cfg.n_group, world, 0)  # checks that the groups split
    idx, w = ops.route(x)                                    # [T, K] int32, fp32
    flat = idx.reshape(-1).to(torch.int64)
    dest = torch.div(flat, per, rounding_mode="floor")
    order = torch.sort(dest, stable=True).indices            # pairs by (rank, flat slot)
    send_counts = torch.bincount(dest, minlength=world).tolist()
    cnt = torch.tensor(send_counts, dtype=torch.int64, device=x.device)
    recv = torch.empty_like(cnt)
    dist.all_to_all_single(recv, cnt, group=group)
    recv_counts = recv.tolist()
    # bf16 rows travel as 32-bit words (H is even): every backend moves those unchanged
    rows = x.view(torch.int16)[torch.div(order, K, rounding_mode="floor")].view(torch.int32)
    x_in = _exchange(rows, send_counts, recv_counts, group).view(torch.int16)
    id_in = _exchange((flat[order] - dest[order] * per).to(torch.int32), send_counts, recv_counts, group)
    w_in = _exchange(w.reshape(-1)[order], send_counts, recv_counts, group)
    y_in = ops.experts(x_in, id_in, w_in)                   # [pairs received, H] fp32
    y_back = _exchange(y_in, recv_counts, send_counts, group)
    y_slot = torch.empty((T * K, cfg.H), dtype=torch.float32, device=x.device)
    y_slot[order] = y_back
    return ops.combine(x, y_slot)


class LibraryOps:
    """The local compute of ep_forward through the library's C-ABI on this
    rank's GPU. W_local: the moe_weights of this rank's expert block (routed
    pointers at its first expert) with the shared expert's weights; Wr, bias:
    the router (replicated)."""

    def __init__(self, cfg, rank: int, world: int, Wr, bias, Wg, Wu, Wd, Wg_s, Wu_s, Wd_s):
        import sigmoid_group_limited_b200 as sgl
        self.sgl = sgl
        self.cfg = cfg
        self.Wr, self.bias = Wr, bias
        e0, e1 = expert_block(cfg.E, cfg.n_group, world, rank)
        self.local = cfg.with_(E=e1 - e0, n_group=1, topk_group=1, K=1, I_shared=0)
        self.W_local = sgl.make_weights(Wg, Wu, Wd)            # this rank's experts only
        self.W_full = sgl.make_weights(Wg, Wu, Wd, Wg_s, Wu_s, Wd_s)

    def route(self, x):
        sgl, c = self.sgl, self.cfg
        T = x.shape[0]
        idx = torch.empty(T, c.K, dtype=torch.int32, device=x.device)
        w = torch.empty(T, c.K, dtype=torch.float32, device=x.device)
        sgl.moe_route(c, x, self.Wr, self.bias, idx, w, sgl.alloc_workspace(c, T, x.device))
        return idx, w

    def experts(self, x_in, ids, w):
        """w * Expert(x) for every received pair: one token per pair (K = 1)."""
        sgl, c = self.sgl, self.local
        P = x_in.shape[0]
        if P == 0:
            return torch.empty(0, c.H, dtype=torch.float32, device=x_in.device)
        dev = x_in.device
        ws = sgl.alloc_workspace(c, P, dev)
        counts = torch.empty(c.E, dtype=torch.int32, device=dev)
        offsets = torch.empty(c.E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(P, dtype=torch.int32, device=dev)
        y_slot = torch.empty(2 * P, c.H, dtype=torch.float32, device=dev)
        sgl.moe_permute(c, P, ids.view(P, 1), counts, offsets, perm, None, ws)
        sgl.moe_grouped_swiglu(c, P, x_in, perm, offsets, w.view(P, 1), self.W_local, y_slot, ws)
        return y_slot[:P]

    def combine(self, x, y_slot_routed):
        """The shared expert's rows, then y = bf16(sum_k y_slot + shared)."""
        sgl, c = self.sgl, self.cfg
        T = x.shape[0]
        dev = x.device
        ws = sgl.alloc_workspace(c, T, dev)
        y_slot = torch.empty(T * c.K + T, c.H, dtype=torch.float32, device=dev)
        y_slot[:T * c.K] = y_slot_routed
        # no routed rows (all expert counts 0): only the shared expert's items run
        offsets = torch.zeros(c.E + 1, dtype=torch.int32, device=dev)
        dummy_perm = torch.zeros(max(1, T * c.K), dtype=torch.int32, device=dev)
        dummy_w = torch.zeros(max(1, T * c.K), dtype=torch.float32, device=dev)
        sgl.moe_grouped_swiglu(c, T, x, dummy_perm, offsets, dummy_w, self.W_full, y_slot, ws)
        y = torch.empty(T, c.H, dtype=torch.bfloat16, device=dev)
        sgl.moe_combine(c, T, y_slot, c.I_shared > 0, y)
        return y
