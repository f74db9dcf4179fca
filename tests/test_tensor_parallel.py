"""The layer split over KV groups (routed_sparse_query_b200.tp) on CPU.

Each rank computes its shard's partial output with the oracle's arithmetic on
the rank's slices of the weights (its groups' W_q, W_k, W_v columns and W_O
rows, the routing of the whole layer); the partial outputs, summed by a gloo
all-reduce over 2 and 4 ranks, must equal the oracle's whole layer. The
partition itself (which columns and rows a rank owns) is the product's.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth
from synth import LayerShape
from routed_sparse_query_b200.tp import GroupShard, shard_weights


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def shard_partial_y(inp: synth.LayerInputs, shard: GroupShard) -> np.ndarray:
    """One rank's partial y from the oracle's steps on the rank's slices."""
    s = inp.shape
    B, T, M, k, dh = s.B, s.T, s.M, s.k, s.d_head
    Gl = shard.G_local
    f = oracle._f64_inputs(inp)
    rt = oracle.router(f["x"], f["W_r"], f["b_r"], s.G, M, k)  # replicated router
    idx = rt["idx"][:, shard.g0:shard.g1]
    omega = rt["omega"][:, shard.g0:shard.g1]
    Wq, Wk, Wv, Wo = shard_weights(shard, f["W_q"], f["W_k"], f["W_v"], f["W_o"])
    K = oracle.kv_proj(f["x"], Wk, B, T, Gl, dh)
    V = oracle.kv_proj(f["x"], Wv, B, T, Gl, dh)
    q = oracle.q_routed_rows(f["x"], Wq, idx, Gl, M, dh)
    R = B * T
    o = np.zeros((R, Gl, k, dh))
    o_s = np.zeros((R, dh))
    for b in range(B):
        rows = slice(b * T, (b + 1) * T)
        for g in range(Gl):
            for si in range(k):
                o[rows, g, si] = oracle.causal_attention(q[rows, g, si], K[b, g], V[b, g])
        if shard.shared:  # local group 0 is the layer's group 0
            qs = f["x"][rows] @ f["W_qs"]
            o_s[rows] = oracle.causal_attention(qs, K[b, 0], V[b, 0])
    parts = [o.reshape(R, Gl * k * dh)]
    if shard.shared:
        parts.append(o_s)
    parts.append(np.einsum("rgs,rgsd->rd", omega, o))  # this rank's part of the weighted slot
    slots = np.concatenate(parts, axis=1)
    assert slots.shape[1] == shard.local_slots() * dh
    return slots @ Wo


SHAPE = LayerShape(B=2, T=24, d_model=64, G=4, M=3, k=2, d_head=8)


def _worker(rank, world, port, out):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        inp = synth.make_layer_inputs(SHAPE, seed=88, skew=False)
        shard = GroupShard(world, rank, SHAPE.G, SHAPE.M, SHAPE.k, SHAPE.d_head)
        y = torch.from_numpy(shard_partial_y(inp, shard))
        dist.all_reduce(y, op=dist.ReduceOp.SUM)
        if rank == 0:
            out["err"] = float(np.abs(y.numpy() - oracle.gqe_layer(inp)["y"]).max())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_split_over_groups_sums_to_the_layer(repo_root, world):
    os.environ.setdefault("PYTHONPATH", repo_root)
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out["err"] < 1e-12


def test_shard_partition_covers_every_column_and_row_once():
    G, M, k, dh = 8, 2, 1, 4
    for world in (1, 2, 4, 8):
        shards = [GroupShard(world, r, G, M, k, dh) for r in range(world)]
        q = np.concatenate([np.arange(G * M * dh)[s.wq_cols()] for s in shards])
        kv = np.concatenate([np.arange(G * dh)[s.kv_cols()] for s in shards])
        assert np.array_equal(q, np.arange(G * M * dh)) and np.array_equal(kv, np.arange(G * dh))
        rows = np.concatenate([s.wo_rows() for s in shards])
        # routed and shared rows once each; the weighted slot's rows on every rank
        wrows = np.arange((k * G + 1) * dh, (k * G + 2) * dh)
        assert np.array_equal(np.sort(rows[~np.isin(rows, wrows)]), np.arange((k * G + 1) * dh))
        assert sum(np.isin(s.wo_rows(), wrows).sum() for s in shards) == world * dh
        assert [s.shared for s in shards] == [True] + [False] * (world - 1)
    with pytest.raises(ValueError):
        GroupShard(3, 0, G, M, k, dh)
