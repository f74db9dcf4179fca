"""Parity at the measured workloads' full sizes, in the launch configuration the
benchmark times (the five step entry points on one stream), on a B200.

The oracle evaluates the router, the token lists and K/V in full and the
attention, slots and y at sampled rows: the first and last rows of each
sequence, rows on both sides of 128-row tile boundaries (the first tile, the
middle, the last full and the ragged last tile) and a few seeded random rows.
Integer outputs must be bit-exact; floating-point outputs within the layer
tolerance (max-abs 2e-2, mean-abs 2e-3). The two long-context workloads
(262144 and 1048576 tokens) are checked the same way, with the oracle's K/V
built only up to each sequence's last sampled row and K/V compared at the
sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_common import assert_close, device_inputs, run_layer, run_steps

pytestmark = pytest.mark.gpu

WORKLOADS = {
    "b4x8k": (synth.BATCH4_8K, {}),
    "seq32k": (synth.SEQ32K, {}),
    "pool4_k1_skew": (synth.POOL4_K1, {"skew": True}),
    "pool4_k2_skew": (synth.POOL4_K2, {"skew": True}),
    "pool4_k2_balanced": (synth.POOL4_K2, {}),
}


@pytest.fixture(scope="module")
def rsq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import routed_sparse_query_b200 as m
    return m


def sample_rows(shape: synth.LayerShape, seed: int = 7) -> np.ndarray:
    T = shape.T
    pos = {0, 1, 127, 128, 129, T // 2 - 1, T // 2, T - 129, T - 128, T - 2, T - 1}
    rng = np.random.default_rng(seed)
    pos |= set(int(v) for v in rng.integers(0, T, 5))
    pos = sorted(p for p in pos if 0 <= p < T)
    return np.array([b * T + p for b in range(shape.B) for p in pos], dtype=np.int64)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_full_size_sampled_rows(rsq, name):
    shape, kw = WORKLOADS[name]
    inp = synth.make_layer_inputs(shape, seed=2024, with_dense=False, **kw)
    rows = sample_rows(shape)
    ref = oracle.gqe_layer(inp, rows=rows)
    o = run_steps(rsq, shape, device_inputs(inp))
    # Router and lists: bit-exact in full.
    assert np.array_equal(o["idx"].cpu().numpy(), ref["idx"]), "router indices differ"
    assert np.array_equal(o["counts"].cpu().numpy().reshape(shape.N, shape.B), ref["counts"])
    assert np.array_equal(o["offsets"].cpu().numpy(), ref["offsets"])
    assert np.array_equal(o["tok"].cpu().numpy(), ref["tok"]), "token lists differ"
    assert np.array_equal(o["slot_pos"].cpu().numpy(), ref["slot_pos"])
    np.testing.assert_allclose(o["r"].cpu().numpy(), ref["r"], rtol=0, atol=2e-6)
    np.testing.assert_allclose(o["omega"].cpu().numpy(), ref["omega"], rtol=0, atol=2e-6)
    assert_close(o["K"], ref["K"], "K")
    assert_close(o["V"], ref["V"], "V")
    # Attention, slots and y at the sampled rows.
    sel = torch.from_numpy(rows).cuda()
    assert_close(o["slots"].index_select(0, sel), ref["slots"], "slots")
    assert_close(o["y"].index_select(0, sel), ref["y"], "y")
    # The fused entry point gives the same y.
    y, _ = run_layer(rsq, shape, device_inputs(inp))
    assert torch.equal(y, o["y"]), "gqe_layer_fwd differs from the step calls"


LONG = {"seq256k": synth.SEQ256K, "seq1m": synth.SEQ1M}


def sample_rows_long(shape: synth.LayerShape, strata: int = 24, seed: int = 11) -> np.ndarray:
    """Tile edges at the start, middle and end of the sequence, plus one
    seeded row in each of `strata` equal stretches of positions."""
    T = shape.T
    pos = {0, 1, 127, 128, 129, T // 2 - 1, T // 2, T - 129, T - 128, T - 2, T - 1}
    rng = np.random.default_rng(seed)
    edges = np.linspace(0, T, strata + 1).astype(np.int64)
    pos |= {int(rng.integers(lo, hi)) for lo, hi in zip(edges[:-1], edges[1:])}
    pos = sorted(p for p in pos if 0 <= p < T)
    return np.array([b * T + p for b in range(shape.B) for p in pos], dtype=np.int64)


@pytest.mark.parametrize("name", list(LONG))
def test_long_context_sampled_rows(rsq, name):
    # The long-context workloads (262144 and 1048576 tokens) against the
    # oracle: router output and token lists bit-exact in full; K, V, slots
    # and y at stratified sampled rows, each evaluated from the definition
    # against the full causal prefix of its sequence.
    shape = LONG[name]
    inp = synth.make_layer_inputs(shape, seed=2026, with_dense=False)
    rows = sample_rows_long(shape)
    ref = oracle.gqe_layer(inp, rows=rows, full_kv=False)
    o = run_steps(rsq, shape, device_inputs(inp))
    assert np.array_equal(o["idx"].cpu().numpy(), ref["idx"]), "router indices differ"
    assert np.array_equal(o["counts"].cpu().numpy().reshape(shape.N, shape.B), ref["counts"])
    assert np.array_equal(o["offsets"].cpu().numpy(), ref["offsets"])
    assert np.array_equal(o["tok"].cpu().numpy(), ref["tok"]), "token lists differ"
    assert np.array_equal(o["slot_pos"].cpu().numpy(), ref["slot_pos"])
    np.testing.assert_allclose(o["r"].cpu().numpy(), ref["r"], rtol=0, atol=2e-6)
    np.testing.assert_allclose(o["omega"].cpu().numpy(), ref["omega"], rtol=0, atol=2e-6)
    b = torch.from_numpy(rows // shape.T).cuda()
    t = torch.from_numpy(rows % shape.T).cuda()
    assert_close(o["K"][b, :, t], ref["K_rows"], "K")
    assert_close(o["V"][b, :, t], ref["V_rows"], "V")
    sel = torch.from_numpy(rows).cuda()
    assert_close(o["slots"].index_select(0, sel), ref["slots"], "slots")
    assert_close(o["y"].index_select(0, sel), ref["y"], "y")
    y_steps = o["y"]
    del o
    torch.cuda.empty_cache()
    y, _ = run_layer(rsq, shape, device_inputs(inp))
    assert torch.equal(y, y_steps), "gqe_layer_fwd differs from the step calls"


def test_long_sequence_layouts_agree_bitwise(rsq):
    # 256k tokens: the slot-major attention runs its stream-major CTA order
    # (1024 tile pairs per stream) and no split-KV; the expert-major layout
    # computes every row with the same online softmax over the same K/V
    # tiles, so the slots must agree bitwise (and the lists stay valid).
    from gpu_common import run_expert_major, run_steps
    shape = synth.LayerShape(B=1, T=262144, d_model=1024, G=8, M=2, k=1, d_head=64)
    g = torch.Generator(device="cuda").manual_seed(262144)
    sd = shape.d_model ** -0.5
    d = {"x": torch.randn(shape.R, shape.d_model, device="cuda", generator=g).to(torch.bfloat16),
         "W_r": torch.randn(shape.d_model, shape.N, device="cuda", generator=g) * sd, "b_r": None}
    for nm, shp in (("W_q", (shape.d_model, shape.N * shape.d_head)), ("W_qs", (shape.d_model, shape.d_head)),
                    ("W_k", (shape.d_model, shape.G * shape.d_head)),
                    ("W_v", (shape.d_model, shape.G * shape.d_head)),
                    ("W_o", (shape.n_slots * shape.d_head, shape.d_model))):
        d[nm] = (torch.randn(*shp, device="cuda", generator=g) * sd).to(torch.bfloat16)
    o = run_steps(rsq, shape, d)
    counts = o["counts"].view(shape.N, shape.B)
    assert int(counts.sum()) == shape.k * shape.G * shape.R
    e = run_expert_major(rsq, shape, d, o)
    n = (shape.k * shape.G + 1) * shape.d_head
    assert torch.equal(e["slots"][:, :n], o["slots"][:, :n]), "layouts differ at 256k"
    assert torch.isfinite(o["y"].float()).all()
