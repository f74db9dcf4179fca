"""The layer's backward (gqe_layer_bwd) through the C ABI against the fp64
backward oracle (oracle.backward) on the same seeded inputs, with the
router's selection of both (bit-exact, checked first) held fixed.

Tolerance: the GPU path takes the forward's bf16 intermediates (Q, K, V and
the slots, each rounded once: relative 2^-9) and accumulates in fp32, so each
gradient is compared normwise: max |g - ref| <= 3e-2 * max |ref| and
mean |g - ref| <= 1e-2 * mean |ref|."""
import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import backward as bw
from synth import LayerShape
from gpu_common import device_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rsq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import routed_sparse_query_b200 as m
    return m


CASES = {
    "b1_t130_dh32": LayerShape(B=1, T=130, d_model=128, G=2, M=3, k=2, d_head=32),
    "b2_t70_dh64": LayerShape(B=2, T=70, d_model=64, G=2, M=2, k=1, d_head=64),
    "b1_t300_g4": LayerShape(B=1, T=300, d_model=256, G=4, M=2, k=1, d_head=64),
}


def _close(got, want, what):
    g = got.double().cpu().numpy().reshape(want.shape)
    err = np.abs(g - want)
    scale_max, scale_mean = float(np.abs(want).max()), float(np.abs(want).mean())
    assert np.isfinite(g).all(), f"{what}: non-finite"
    assert err.max() <= 3e-2 * scale_max, f"{what}: max err {err.max():.3e} vs max |ref| {scale_max:.3e}"
    assert err.mean() <= 1e-2 * scale_mean, f"{what}: mean err {err.mean():.3e} vs mean |ref| {scale_mean:.3e}"


@pytest.mark.parametrize("name", list(CASES))
def test_layer_backward_matches_oracle(rsq, name):
    _check(rsq, CASES[name], 0)


def test_layer_backward_at_the_bench_workload(rsq):
    # seq2k (B=1, T=2048, d_model=1024, G=8, M=2, k=1, d_head=64), the call
    # `bench.py --backward` times, with its flags (a zeroed workspace declared
    # clean): the full attention-backward grid (two CTAs per 128-row tile,
    # 16 x 16 tiles per stream), every gradient against the fp64 oracle.
    _check(rsq, synth.SEQ2K, rsq.GQE_FLAG_WS_CLEAN)


def _check(rsq, s, flags):
    inp = synth.make_layer_inputs(s, seed=31)
    f = oracle._f64_inputs(inp)
    rt = oracle.router(f["x"], f["W_r"], f["b_r"], s.G, s.M, s.k)
    rng = np.random.default_rng(7)
    dy = rng.standard_normal((s.R, s.d_model)).astype(np.float32)
    ref = bw.backward(f["x"], f["W_r"], f["b_r"], f["W_q"], f["W_qs"], f["W_k"], f["W_v"], f["W_o"],
                      B=s.B, T=s.T, G=s.G, M=s.M, dh=s.d_head, idx=rt["idx"], dy=dy.astype(np.float64))
    d = device_inputs(inp)
    cfg = rsq.GQEConfig.of(s, flags)
    ws = torch.zeros(rsq.gqe_workspace_bytes(cfg, rsq.GQE_WS_BACKWARD), dtype=torch.uint8, device="cuda")
    dev = lambda *shape: torch.empty(*shape, dtype=torch.float32, device="cuda")  # noqa: E731
    N, dh, R, dm = s.N, s.d_head, s.R, s.d_model
    out = {"dx": dev(R, dm), "dW_r": dev(dm, N), "db_r": dev(N), "dW_q": dev(dm, N * dh), "dW_qs": dev(dm, dh),
           "dW_k": dev(dm, s.G * dh), "dW_v": dev(dm, s.G * dh), "dW_o": dev((s.k * s.G + 2) * dh, dm)}
    rsq.gqe_layer_bwd(cfg, d["x"], d["W_r"], d["b_r"], d["W_q"], d["W_qs"], d["W_k"], d["W_v"], d["W_o"],
                      torch.from_numpy(dy).cuda(), out["dx"], out["dW_r"], out["db_r"], out["dW_q"],
                      out["dW_qs"], out["dW_k"], out["dW_v"], out["dW_o"], ws)
    torch.cuda.synchronize()
    assert rsq.gqe_read_status() == 0
    idx = rsq.workspace_view(ws, cfg, rsq.GQE_WS_LAYER, "idx", torch.int32, (R, s.G, s.k))
    assert np.array_equal(idx.cpu().numpy(), rt["idx"]), "the recomputed routing differs"
    for key in ("dx", "dW_r", "db_r", "dW_q", "dW_qs", "dW_k", "dW_v", "dW_o"):
        _close(out[key], ref[key], key)


def test_backward_rejects_other_output_constructions(rsq):
    s = CASES["b2_t70_dh64"]
    cfg = rsq.GQEConfig.of(s, rsq.GQE_FLAG_OUT_HARD)
    assert rsq.gqe_workspace_bytes(cfg, rsq.GQE_WS_BACKWARD) == 0
