"""gqe_dispatch_noalloc: the dispatch entry point for callers that cannot give
the library a workspace (their device memory is owned by another allocator,
so they cannot allocate per call). Its scratch is a fixed device array of the
library. Checked through the C ABI against gqe_dispatch (which takes a
workspace) on two calls in a row, so that contents left by the first call
cannot leak into the second.

Collected last on purpose (file name), so a run that stops at the first
failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import synth
from synth import LayerShape
from gpu_common import device_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rsq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import routed_sparse_query_b200 as m
    return m


def _outputs(shape):
    B, T, G, M, k, dh = shape.B, shape.T, shape.G, shape.M, shape.k, shape.d_head
    R, N = B * T, G * M
    e = lambda *s, dt: torch.full(s, -7, dtype=dt, device="cuda")  # noqa: E731
    return {"counts": e(N * B, dt=torch.int32), "offsets": e(N * B + 1, dt=torch.int32),
            "tok": e(k * G * R, dt=torch.int32), "slot_pos": e(R, G, k, dt=torch.int32),
            "Qv": e(B, G, k, T, dh, dt=torch.bfloat16), "Qs": e(B, T, dh, dt=torch.bfloat16)}


@pytest.mark.parametrize("shape", [
    LayerShape(B=2, T=777, d_model=256, G=4, M=2, k=1, d_head=64),
    LayerShape(B=1, T=2048, d_model=512, G=8, M=4, k=2, d_head=64),
])
def test_noalloc_dispatch_matches_workspace_dispatch(rsq, shape):
    cfg = rsq.GQEConfig.of(shape)
    results = []
    for seed in (31, 32):  # two calls in a row, different routing
        inp = synth.make_layer_inputs(shape, seed=seed, skew=shape.M == 4)
        d = device_inputs(inp)
        idx = torch.empty(shape.R, shape.G, shape.k, dtype=torch.int32, device="cuda")
        r = torch.empty_like(idx, dtype=torch.float32)
        om = torch.empty_like(idx, dtype=torch.float32)
        rsq.gqe_router_topk(cfg, d["x"], d["W_r"], d["b_r"], idx, r, om)

        ref = _outputs(shape)
        ws = torch.empty(rsq.gqe_workspace_bytes(cfg, rsq.GQE_WS_DISPATCH), dtype=torch.uint8,
                         device="cuda")
        rsq.gqe_dispatch(cfg, idx, d["x"], d["W_q"], d["W_qs"], ref["counts"], ref["offsets"],
                         ref["tok"], ref["slot_pos"], ref["Qv"], ref["Qs"], ws)

        got = _outputs(shape)
        rsq.gqe_dispatch_noalloc(cfg, idx, d["x"], d["W_q"], d["W_qs"], got["counts"],
                                 got["offsets"], got["tok"], got["slot_pos"], got["Qv"], got["Qs"])
        torch.cuda.synchronize()
        assert rsq.gqe_read_status() == 0
        # Same kernels, tiles and inputs; only the scratch's place differs, so
        # every output is bitwise equal (a stale tile-table entry would change
        # which rows a tile covers).
        for name in ("counts", "offsets", "tok", "slot_pos", "Qv", "Qs"):
            assert torch.equal(got[name], ref[name]), name
        results.append(got["tok"].cpu().numpy())
    assert not np.array_equal(results[0], results[1])  # the second call really re-dispatched


def test_noalloc_rejects_configs_beyond_its_scratch(rsq):
    # 1e6 tokens, 32 groups, k = 2: the tile table alone needs ~8 MB > 4 MiB.
    shape = LayerShape(B=1, T=1_000_000, d_model=64, G=32, M=2, k=2, d_head=32)
    cfg = rsq.GQEConfig.of(shape)
    assert rsq.gqe_workspace_bytes(cfg, rsq.GQE_WS_DISPATCH) > 4 << 20
    p = torch.empty(16, dtype=torch.uint8, device="cuda")  # never touched: rejected on the host
    st = rsq.lib().gqe_dispatch_noalloc(rsq._cfg(cfg), *([p.data_ptr()] * 10), None)
    assert st == rsq.GQE_ERR_WORKSPACE
