"""One GQE layer split over its KV groups across ranks (tensor parallelism).

Each rank owns a contiguous block of G / P groups: the query-head experts of
those groups (their W_q columns), the groups' K/V heads (W_k, W_v columns) and
the W_O rows of their routed slots. The router is replicated -- x . W_r is
small, and its weights (omega) are normalised over every group of the token,
so each rank runs it for the whole layer. Every rank adds its groups' part of
the weighted slot, sum over local g of omega[g, s] o[g, s]; the slot enters
W_O linearly, so each rank multiplies its partial slot by the weighted slot's
W_O rows. The rank holding group 0 also runs the shared head (which attends to
KV group 0). The partial outputs of the ranks sum to the layer's y: one
all-reduce.

("Within each GQA group, a router selects k query-head experts per token
while all key-value heads remain dense and unchanged": chatpaper / hotpaper
abstract; the groups never exchange data before W_O, which is what makes the
split possible.)

This module holds the partition (which columns and rows a rank owns) and the
driver that issues a rank's calls through the C ABI. The shard's routing is
copied out of the layer's routing with torch (a layout copy: the groups of a
row are contiguous in idx / omega), and the partial outputs are summed with
torch.distributed.all_reduce.
"""
from __future__ import annotations

import dataclasses

import numpy as np


@dataclasses.dataclass(frozen=True)
class GroupShard:
    """Rank `rank` of `world` in a split of G groups (M experts each, k
    selected, head dim d_head)."""
    world: int
    rank: int
    G: int
    M: int
    k: int
    d_head: int

    def __post_init__(self):
        if self.world < 1 or not 0 <= self.rank < self.world or self.G % self.world != 0:
            raise ValueError("the groups must split evenly over the ranks")

    @property
    def G_local(self) -> int:
        return self.G // self.world

    @property
    def g0(self) -> int:
        return self.rank * self.G_local

    @property
    def g1(self) -> int:
        return self.g0 + self.G_local

    @property
    def shared(self) -> bool:
        """This rank holds group 0, so it runs the shared head."""
        return self.g0 == 0

    def wq_cols(self) -> slice:
        """W_q columns of the local experts (expert e = g*M + j)."""
        dh = self.d_head
        return slice(self.g0 * self.M * dh, self.g1 * self.M * dh)

    def kv_cols(self) -> slice:
        """W_k / W_v columns of the local KV heads."""
        return slice(self.g0 * self.d_head, self.g1 * self.d_head)

    def wo_rows(self) -> np.ndarray:
        """W_O rows of this rank's slots, in the rank's slot order: its routed
        slots (g, s), then the shared head's (rank of group 0 only), then the
        weighted slot's."""
        dh, k, G = self.d_head, self.k, self.G
        rows = [np.arange(self.g0 * k * dh, self.g1 * k * dh)]
        if self.shared:
            rows.append(np.arange(k * G * dh, (k * G + 1) * dh))
        rows.append(np.arange((k * G + 1) * dh, (k * G + 2) * dh))
        return np.concatenate(rows)

    def local_slots(self) -> int:
        return self.k * self.G_local + (2 if self.shared else 1)


def shard_weights(shard: GroupShard, W_q, W_k, W_v, W_o):
    """The rank's slices of the layer's weights (numpy arrays or torch
    tensors, rows = input features): W_q, W_k, W_v columns and W_O rows, each
    contiguous."""
    def cont(a):
        return a.contiguous() if hasattr(a, "contiguous") else np.ascontiguousarray(a)

    rows = shard.wo_rows()
    if hasattr(W_o, "index_select"):
        import torch
        Wo = W_o.index_select(0, torch.as_tensor(rows, device=W_o.device))
    else:
        Wo = W_o[rows]
    return (cont(W_q[:, shard.wq_cols()]), cont(W_k[:, shard.kv_cols()]), cont(W_v[:, shard.kv_cols()]),
            cont(Wo))


def shard_flags(shard: GroupShard, base: int = 0) -> int:
    """gqe_config flags of the rank's calls: the shared head only on the rank
    of group 0."""
    import routed_sparse_query_b200 as rsq
    return base | (0 if shard.shared else rsq.GQE_FLAG_NO_SHARED_HEAD)


def local_shape(shard: GroupShard, shape):
    """The rank's layer shape: its groups only."""
    return dataclasses.replace(shape, G=shard.G_local)


class ShardLayer:
    """Device buffers of one rank's part of the layer and its calls."""

    def __init__(self, rsq, shard: GroupShard, shape, base_flags: int = 0):
        import torch
        self.rsq, self.shard, self.shape = rsq, shard, shape
        s, ls = shape, local_shape(shard, shape)
        dev = torch.device("cuda")
        R, k, dh = s.R, s.k, s.d_head
        self.cfg = rsq.GQEConfig.of(s, base_flags)  # the whole layer (router)
        self.cfg_l = rsq.GQEConfig.of(ls, shard_flags(shard, base_flags))
        e = torch.empty
        self.idx = e(R, s.G, k, dtype=torch.int32, device=dev)
        self.r = e(R, s.G, k, dtype=torch.float32, device=dev)
        self.omega = e(R, s.G, k, dtype=torch.float32, device=dev)
        Gl, Nl = ls.G, ls.G * ls.M
        self.counts = e(Nl * s.B, dtype=torch.int32, device=dev)
        self.offsets = e(Nl * s.B + 1, dtype=torch.int32, device=dev)
        self.tok = e(k * Gl * R, dtype=torch.int32, device=dev)
        self.slot_pos = e(R, Gl, k, dtype=torch.int32, device=dev)
        self.Qv = e(s.B, Gl, k, s.T, dh, dtype=torch.bfloat16, device=dev)
        self.Qs = e(s.B, s.T, dh, dtype=torch.bfloat16, device=dev) if shard.shared else None
        self.K = e(s.B, Gl, s.T, dh, dtype=torch.bfloat16, device=dev)
        self.V = e(s.B, Gl, s.T, dh, dtype=torch.bfloat16, device=dev)
        self.slots = e(R, shard.local_slots() * dh, dtype=torch.bfloat16, device=dev)
        self.wsd = e(max(16, rsq.gqe_workspace_bytes(self.cfg_l, rsq.GQE_WS_DISPATCH)), dtype=torch.uint8,
                     device=dev)
        self.wsa = e(rsq.gqe_workspace_bytes(self.cfg_l, rsq.GQE_WS_ATTENTION), dtype=torch.uint8, device=dev)

    def forward(self, x, W_r, b_r, W_q_l, W_qs, W_k_l, W_v_l, W_o_l, y, group=None, stream=None):
        """The rank's partial y (all-reduced over `group` when given).
        W_*_l are the rank's slices (shard_weights); W_qs is used on the rank
        of group 0 only."""
        rsq, sh = self.rsq, self.shard
        rsq.gqe_router_topk(self.cfg, x, W_r, b_r, self.idx, self.r, self.omega, stream)
        idx_l = self.idx[:, sh.g0:sh.g1].contiguous()
        om_l = self.omega[:, sh.g0:sh.g1].contiguous()
        rsq.gqe_dispatch(self.cfg_l, idx_l, x, W_q_l, W_qs if sh.shared else None, self.counts,
                         self.offsets, self.tok, self.slot_pos, self.Qv, self.Qs, self.wsd, stream)
        rsq.gqe_kv_proj(self.cfg_l, x, W_k_l, W_v_l, self.K, self.V, stream)
        rsq.gqe_attention_fwd(self.cfg_l, self.Qv, self.Qs, self.K, self.V, self.slots, self.wsa, stream)
        rsq.gqe_output_proj(self.cfg_l, self.slots, om_l, W_o_l, y, stream)
        if group is not None:
            import torch.distributed as dist
            dist.all_reduce(y, op=dist.ReduceOp.SUM, group=group)
        return y
