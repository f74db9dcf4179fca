"""The layer split over KV groups through the C ABI on one B200: each rank's
part (routing of the whole layer, its groups' dispatch, K/V, attention and
W_O rows, the shared head on the rank of group 0) runs one after another on
the same GPU, with no collective; the partial outputs summed on the device
must match the oracle's layer (within the layer tolerance plus the bf16
rounding of each shard's partial output), and each shard's token lists must be
the oracle's lists of its groups."""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import LayerShape
from gpu_common import assert_close, device_inputs
from routed_sparse_query_b200.tp import GroupShard, ShardLayer, shard_weights

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rsq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import routed_sparse_query_b200 as m
    return m


@pytest.mark.parametrize("world,shape", [
    (2, LayerShape(B=1, T=640, d_model=256, G=8, M=2, k=1, d_head=64)),
    (4, LayerShape(B=2, T=300, d_model=256, G=8, M=4, k=2, d_head=64)),
    (2, LayerShape(B=1, T=200, d_model=128, G=4, M=2, k=1, d_head=32)),
])
def test_group_shards_sum_to_the_layer(rsq, world, shape):
    inp = synth.make_layer_inputs(shape, seed=89, skew=shape.M == 4)
    ref = oracle.gqe_layer(inp)
    d = device_inputs(inp)
    y_sum = torch.zeros(shape.R, shape.d_model, dtype=torch.float32, device="cuda")
    rounding = 0.0  # each shard's y is rounded to bf16 (unit roundoff 2^-9) before the sum
    for rank in range(world):
        shard = GroupShard(world, rank, shape.G, shape.M, shape.k, shape.d_head)
        Wq, Wk, Wv, Wo = shard_weights(shard, d["W_q"], d["W_k"], d["W_v"], d["W_o"])
        layer = ShardLayer(rsq, shard, shape)
        y = torch.empty(shape.R, shape.d_model, dtype=torch.bfloat16, device="cuda")
        layer.forward(d["x"], d["W_r"], d["b_r"], Wq, d["W_qs"], Wk, Wv, Wo, y)
        torch.cuda.synchronize()
        assert rsq.gqe_read_status() == 0
        y_sum += y.float()
        rounding += float(y.float().abs().max()) * 2.0 ** -9
        lists = oracle.dispatch(ref["idx"][:, shard.g0:shard.g1], shape.B, shape.T, shard.G_local, shape.M)
        assert np.array_equal(layer.tok.cpu().numpy(), lists["tok"])
        assert np.array_equal(layer.offsets.cpu().numpy(), lists["offsets"])
    # The layer's bounds, plus the bf16 rounding of each shard's partial output.
    assert_close(y_sum, ref["y"], f"sum of {world} shards", max_abs=2e-2 + rounding)
