"""Decode step on a B200 through the C ABI, against the fp64 oracle.

The cache holds the K/V of the first T-1 tokens of each sequence (computed on
the GPU by gqe_kv_proj, so both sides read the same bf16 bits); the step adds
token T-1. y must be within the layer tolerance of the oracle's decode step,
the new K/V written into the cache within the K/V tolerance, and nothing else
of the cache may change.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import LayerShape
from gpu_common import assert_close, bf16_dev, device_inputs, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rsq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import routed_sparse_query_b200 as m
    return m


CASES = {
    "empty_cache": LayerShape(B=2, T=1, d_model=128, G=2, M=2, k=1, d_head=64),
    "t5_k2": LayerShape(B=3, T=5, d_model=128, G=2, M=3, k=2, d_head=32),
    "chunk_edge_256": LayerShape(B=2, T=256, d_model=256, G=4, M=2, k=1, d_head=64),
    "chunk_edge_257": LayerShape(B=2, T=257, d_model=256, G=4, M=2, k=1, d_head=64),
    "pool4_k2": LayerShape(B=2, T=700, d_model=256, G=8, M=4, k=2, d_head=64),
    "long_2k": LayerShape(B=2, T=2048, d_model=1024, G=8, M=2, k=1, d_head=64),
    # 128 (sequence, group) pairs: spans of 2 chunks of 256 keys (the streaming
    # form's online softmax across chunks), the last span one partial chunk.
    "spans_4097": LayerShape(B=16, T=4097, d_model=256, G=8, M=2, k=1, d_head=64),
}


def _setup(rsq, shape, seed=77):
    inp = synth.make_layer_inputs(shape, seed=seed)
    d = device_inputs(inp)
    B, T, G, dh = shape.B, shape.T, shape.G, shape.d_head
    cap = T + 3
    Kc = torch.zeros(B, G, cap, dh, dtype=torch.bfloat16, device="cuda")
    Vc = torch.zeros_like(Kc)
    if T > 1:
        pre = LayerShape(B, T - 1, shape.d_model, G, shape.M, shape.k, dh)
        xp = d["x"].view(B, T, -1)[:, :T - 1].contiguous().view(B * (T - 1), -1)
        Kp = torch.empty(B, G, T - 1, dh, dtype=torch.bfloat16, device="cuda")
        Vp = torch.empty_like(Kp)
        rsq.gqe_kv_proj(rsq.GQEConfig.of(pre), xp, d["W_k"], d["W_v"], Kp, Vp)
        Kc[:, :, :T - 1] = Kp
        Vc[:, :, :T - 1] = Vp
    x_new = d["x"].view(B, T, -1)[:, T - 1].contiguous()
    torch.cuda.synchronize()
    return inp, d, Kc, Vc, x_new


def _oracle_inputs(inp, Kc, Vc, T):
    f = oracle._f64_inputs(inp)
    B = inp.shape.B
    rows = [b * T + T - 1 for b in range(B)]
    Kf = to_f64(Kc[:, :, :T - 1])
    Vf = to_f64(Vc[:, :, :T - 1])
    return f, f["x"][rows], Kf, Vf


@pytest.mark.parametrize("name", list(CASES))
def test_decode_step_matches_oracle(rsq, name):
    shape = CASES[name]
    inp, d, Kc, Vc, x_new = _setup(rsq, shape)
    B, T, G, dh = shape.B, shape.T, shape.G, shape.d_head
    f, xn, Kf, Vf = _oracle_inputs(inp, Kc, Vc, T)
    K_before, V_before = Kc.clone(), Vc.clone()
    cfg = rsq.GQEConfig.of(shape)
    ws = torch.empty(rsq.gqe_workspace_bytes(cfg, rsq.GQE_WS_DECODE), dtype=torch.uint8, device="cuda")
    y = torch.empty(B, shape.d_model, dtype=torch.bfloat16, device="cuda")
    rsq.gqe_decode_step(cfg, x_new, d["W_r"], d["b_r"], d["W_q"], d["W_qs"], d["W_k"], d["W_v"],
                        d["W_o"], Kc, Vc, y, ws)
    torch.cuda.synchronize()
    assert rsq.gqe_read_status() == 0
    ref = oracle.gqe_decode_step(xn, Kf, Vf, f["W_r"], f["b_r"], f["W_q"], f["W_qs"], f["W_k"],
                                 f["W_v"], f["W_o"], G, shape.M, shape.k, dh)
    # The step's routing: bit-exact indices, weights within 2e-6.
    sel = (B, G, shape.k)
    idx = rsq.workspace_view(ws, cfg, rsq.GQE_WS_DECODE, "idx", torch.int32, sel)
    assert np.array_equal(idx.cpu().numpy(), ref["idx"]), "decode router indices differ"
    for item in ("r", "omega"):
        got = rsq.workspace_view(ws, cfg, rsq.GQE_WS_DECODE, item, torch.float32, sel)
        np.testing.assert_allclose(got.cpu().numpy(), ref[item], rtol=0, atol=2e-6)
    short = T < 128  # a few cached keys: o is close to single V rows
    assert_close(y, ref["y"], "y", allow_scale=short)
    assert_close(Kc[:, :, T - 1], ref["k_new"], "new K", allow_scale=short)
    assert_close(Vc[:, :, T - 1], ref["v_new"], "new V", allow_scale=short)
    # Only position T-1 of the cache changed.
    keep = torch.ones(Kc.shape[2], dtype=torch.bool, device="cuda")
    keep[T - 1] = False
    assert torch.equal(Kc[:, :, keep], K_before[:, :, keep])
    assert torch.equal(Vc[:, :, keep], V_before[:, :, keep])


@pytest.mark.parametrize("name", ["t5_k2", "chunk_edge_257", "pool4_k2", "spans_4097"])
def test_dense_decode_step_matches_oracle(rsq, name):
    shape = CASES[name]
    inp, d, Kc, Vc, x_new = _setup(rsq, shape, seed=78)
    B, T, G, dh = shape.B, shape.T, shape.G, shape.d_head
    f, xn, Kf, Vf = _oracle_inputs(inp, Kc, Vc, T)
    cfg = rsq.GQEConfig.of(shape)
    ws = torch.empty(rsq.gqe_workspace_bytes(cfg, rsq.GQE_WS_DENSE_DECODE), dtype=torch.uint8,
                     device="cuda")
    y = torch.empty(B, shape.d_model, dtype=torch.bfloat16, device="cuda")
    rsq.gqa_dense_decode_step(cfg, x_new, d["W_q"], d["W_k"], d["W_v"], d["W_o_dense"], Kc, Vc, y, ws)
    torch.cuda.synchronize()
    assert rsq.gqe_read_status() == 0
    ref = oracle.gqa_dense_decode_step(xn, Kf, Vf, f["W_q"], f["W_k"], f["W_v"], f["W_o_dense"], G,
                                       shape.M, dh)
    assert_close(y, ref["y"], "y (dense decode)", allow_scale=T < 128)


def test_decode_step_agrees_with_prefill_layer(rsq):
    # The GPU decode of token T-1 and the GPU prefill layer's row T-1 are two
    # computations of the same definition: within the layer tolerance of each
    # other.
    shape = CASES["long_2k"]
    inp, d, Kc, Vc, x_new = _setup(rsq, shape, seed=79)
    B, T = shape.B, shape.T
    cfg = rsq.GQEConfig.of(shape)
    ws = torch.empty(rsq.gqe_workspace_bytes(cfg, rsq.GQE_WS_DECODE), dtype=torch.uint8, device="cuda")
    y = torch.empty(B, shape.d_model, dtype=torch.bfloat16, device="cuda")
    rsq.gqe_decode_step(cfg, x_new, d["W_r"], d["b_r"], d["W_q"], d["W_qs"], d["W_k"], d["W_v"],
                        d["W_o"], Kc, Vc, y, ws)
    wsl = torch.empty(rsq.gqe_workspace_bytes(cfg, rsq.GQE_WS_LAYER), dtype=torch.uint8, device="cuda")
    yl = torch.empty(B * T, shape.d_model, dtype=torch.bfloat16, device="cuda")
    rsq.gqe_layer_fwd(cfg, d["x"], d["W_r"], d["b_r"], d["W_q"], d["W_qs"], d["W_k"], d["W_v"],
                      d["W_o"], yl, wsl)
    torch.cuda.synchronize()
    assert rsq.gqe_read_status() == 0
    assert_close(y, to_f64(yl.view(B, T, -1)[:, T - 1]), "decode vs prefill row")
