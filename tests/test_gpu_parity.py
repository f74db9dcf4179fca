"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on a B200.

Integer outputs (router indices, token lists, counts, offsets, slot positions)
must be bit-exact; floating-point outputs must be within max-abs 2e-2 and
mean-abs 2e-3 of the oracle (bf16 inputs, fp32 accumulation).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import LayerShape
from gpu_common import (assert_close, device_inputs, qv_in_list_order, run_dense, run_expert_major,
                        run_layer, run_steps, to_f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rsq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import routed_sparse_query_b200 as m
    return m


def _check_integer_parts(o, ref, shape):
    assert np.array_equal(o["idx"].cpu().numpy(), ref["idx"]), "router indices differ"
    assert np.array_equal(o["counts"].cpu().numpy().reshape(shape.N, shape.B), ref["counts"])
    assert np.array_equal(o["offsets"].cpu().numpy(), ref["offsets"])
    assert np.array_equal(o["tok"].cpu().numpy(), ref["tok"]), "token lists differ"
    assert np.array_equal(o["slot_pos"].cpu().numpy(), ref["slot_pos"])


def _check_float_parts(o, ref, shape):
    np.testing.assert_allclose(o["r"].cpu().numpy(), ref["r"], rtol=0, atol=2e-6)
    np.testing.assert_allclose(o["omega"].cpu().numpy(), ref["omega"], rtol=0, atol=2e-6)
    short = shape.T < 128  # only sequences shorter than one tile may scale the bounds
    for key in ("K", "V", "Qv", "Qs", "slots", "y"):
        assert_close(o[key], ref[key], key, allow_scale=short)


CASES = {
    "tiny": (synth.TINY, {}),
    "ragged_b2": (LayerShape(B=2, T=333, d_model=256, G=4, M=2, k=1, d_head=64), {}),
    "pool4_k2_skew": (LayerShape(B=1, T=700, d_model=512, G=8, M=4, k=2, d_head=64), {"skew": True}),
    "pool4_k1_skew": (LayerShape(B=2, T=300, d_model=512, G=8, M=4, k=1, d_head=64), {"skew": True}),
    "k_equals_m": (LayerShape(B=1, T=260, d_model=256, G=4, M=2, k=2, d_head=32), {}),
    "t1": (LayerShape(B=3, T=1, d_model=128, G=2, M=2, k=1, d_head=64), {}),
    "t5_dh32": (LayerShape(B=2, T=5, d_model=64, G=2, M=3, k=2, d_head=32), {}),
    # Query-projection weights of one expert larger than the resident limit
    # (d_model x d_head bf16 > 128 KB): the per-tile routed Q GEMM.
    "wide_d1536": (LayerShape(B=1, T=300, d_model=1536, G=4, M=2, k=1, d_head=64), {}),
    # The same width with d_head = 32: 24 K blocks resident.
    "d1536_dh32": (LayerShape(B=2, T=200, d_model=1536, G=2, M=3, k=2, d_head=32), {}),
    # At least two query tiles per SM: the routed Q GEMM with the expert's
    # weights resident in shared memory (routed tiles, then shared-head tiles).
    "resident_w": (LayerShape(B=2, T=2400, d_model=256, G=8, M=2, k=1, d_head=64), {}),
}


@pytest.mark.parametrize("name", list(CASES))
def test_layer_steps_match_oracle(rsq, name):
    shape, kw = CASES[name]
    inp = synth.make_layer_inputs(shape, seed=101, **kw)
    ref = oracle.gqe_layer(inp)
    o = run_steps(rsq, shape, device_inputs(inp))
    _check_integer_parts(o, ref, shape)
    _check_float_parts(o, ref, shape)


def test_large_batch_dispatch_is_bit_exact(rsq):
    # 21000 rows in three sequences with a ragged last dispatch tile, 12
    # experts, k = 2; the last query tile of each stream is alone in its CTA
    # with 55 KV tiles (a long single-tile loop of the attention kernel).
    shape = LayerShape(B=3, T=7000, d_model=128, G=4, M=3, k=2, d_head=32)
    inp = synth.make_layer_inputs(shape, seed=23)
    import oracle as orc
    f = orc._f64_inputs(inp)
    rt = orc.router(f["x"], f["W_r"], f["b_r"], shape.G, shape.M, shape.k)
    ref = dict(rt)
    ref.update(orc.dispatch(rt["idx"], shape.B, shape.T, shape.G, shape.M))
    o = run_steps(rsq, shape, device_inputs(inp))
    _check_integer_parts(o, ref, shape)


def test_seq2k_layer_matches_oracle(rsq):
    shape = synth.SEQ2K
    inp = synth.make_layer_inputs(shape)
    ref = oracle.gqe_layer(inp)
    d = device_inputs(inp)
    o = run_steps(rsq, shape, d)
    _check_integer_parts(o, ref, shape)
    _check_float_parts(o, ref, shape)
    y, ws = run_layer(rsq, shape, d)
    assert torch.equal(y, o["y"]), "gqe_layer_fwd differs from the step calls"


def test_split_kv_attention_repeated_calls(rsq):
    # T = 3072 (9 streams): the split-KV attention with pairs of unequal chunk
    # counts; the layer matches the oracle, and further calls on the same
    # scratch (merge counters reset by the previous call) give the same slots,
    # with and without GQE_FLAG_WS_CLEAN.
    shape = LayerShape(B=1, T=3072, d_model=1024, G=8, M=2, k=1, d_head=64)
    inp = synth.make_layer_inputs(shape, seed=12)
    ref = oracle.gqe_layer(inp)
    d = device_inputs(inp)
    o = run_steps(rsq, shape, d)
    _check_integer_parts(o, ref, shape)
    _check_float_parts(o, ref, shape)
    y, ws = run_layer(rsq, shape, d)
    assert torch.equal(y, o["y"]), "gqe_layer_fwd differs from the step calls"
    cfg = rsq.GQEConfig.of(shape)
    wsa = torch.empty(rsq.gqe_workspace_bytes(cfg, rsq.GQE_WS_ATTENTION), dtype=torch.uint8,
                      device="cuda")
    assert wsa.numel() > 256
    for _ in range(2):
        slots = torch.zeros_like(o["slots"])
        rsq.gqe_attention_fwd(cfg, o["Qv"], o["Qs"], o["K"], o["V"], slots, wsa)
        torch.cuda.synchronize()
        assert torch.equal(slots[:, :(shape.k * shape.G + 1) * shape.d_head],
                           o["slots"][:, :(shape.k * shape.G + 1) * shape.d_head])
    # GQE_FLAG_WS_CLEAN: a zero-filled scratch, not cleared by the calls, stays
    # valid from call to call (every call leaves the counters zero).
    cfg_c = rsq.GQEConfig.of(shape, rsq.GQE_FLAG_WS_CLEAN)
    wsz = torch.zeros_like(wsa)
    for _ in range(3):
        slots = torch.zeros_like(o["slots"])
        rsq.gqe_attention_fwd(cfg_c, o["Qv"], o["Qs"], o["K"], o["V"], slots, wsz)
        torch.cuda.synchronize()
        assert rsq.gqe_read_status() == 0
        assert torch.equal(slots[:, :(shape.k * shape.G + 1) * shape.d_head],
                           o["slots"][:, :(shape.k * shape.G + 1) * shape.d_head])
    wsl = torch.zeros(rsq.gqe_workspace_bytes(cfg_c, rsq.GQE_WS_LAYER), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        y2 = torch.empty_like(y)
        rsq.gqe_layer_fwd(cfg_c, d["x"], d["W_r"], d["b_r"], d["W_q"], d["W_qs"], d["W_k"], d["W_v"],
                          d["W_o"], y2, wsl)
        torch.cuda.synchronize()
        assert rsq.gqe_read_status() == 0
        assert torch.equal(y2, y)


def test_dense_gqa_matches_oracle(rsq):
    for shape in (synth.TINY, synth.SEQ2K, LayerShape(B=2, T=200, d_model=256, G=2, M=3, k=1, d_head=64)):
        inp = synth.make_layer_inputs(shape, seed=7)
        ref = oracle.gqa_dense_layer(inp)
        d = device_inputs(inp)
        y, ws = run_dense(rsq, shape, d)
        assert_close(y, ref["y"], f"dense y {shape}")
        O = rsq.workspace_view(ws, rsq.GQEConfig.of(shape), rsq.GQE_WS_DENSE, "dense_O",
                               torch.bfloat16, (shape.R, shape.N * shape.d_head))
        assert_close(O, ref["O"], f"dense O {shape}")


def test_kv_is_identical_in_both_layers(rsq):
    shape = synth.SEQ2K
    inp = synth.make_layer_inputs(shape, seed=3)
    d = device_inputs(inp)
    cfg = rsq.GQEConfig.of(shape)
    _, ws_g = run_layer(rsq, shape, d)
    _, ws_d = run_dense(rsq, shape, d)
    kv_shape = (shape.B, shape.G, shape.T, shape.d_head)
    for item in ("K", "V"):
        a = rsq.workspace_view(ws_g, cfg, rsq.GQE_WS_LAYER, item, torch.bfloat16, kv_shape)
        b = rsq.workspace_view(ws_d, cfg, rsq.GQE_WS_DENSE, item, torch.bfloat16, kv_shape)
        assert torch.equal(a, b)


def test_k_equals_m_routed_slots_are_dense_heads(rsq):
    # With k = M every expert of every group is selected in ascending order,
    # so routed slot (g, s) is dense head g*M + s, computed by the same kernels.
    shape = LayerShape(B=1, T=384, d_model=256, G=4, M=2, k=2, d_head=64)
    inp = synth.make_layer_inputs(shape, seed=9)
    d = device_inputs(inp)
    o = run_steps(rsq, shape, d)
    _, ws = run_dense(rsq, shape, d)
    O = rsq.workspace_view(ws, rsq.GQEConfig.of(shape), rsq.GQE_WS_DENSE, "dense_O", torch.bfloat16,
                           (shape.R, shape.N * shape.d_head))
    routed = o["slots"][:, :shape.N * shape.d_head]
    assert torch.equal(routed, O)


def test_empty_expert_lists(rsq):
    shape = LayerShape(B=2, T=150, d_model=128, G=2, M=3, k=1, d_head=64)
    inp = synth.make_layer_inputs(shape, seed=5)
    inp.b_r = np.array([40.0, 0, 0, 40.0, 0, 0], dtype=np.float32)  # every token picks j = 0
    ref = oracle.gqe_layer(inp)
    o = run_steps(rsq, shape, device_inputs(inp))
    _check_integer_parts(o, ref, shape)
    _check_float_parts(o, ref, shape)
    assert (o["counts"].cpu().numpy().reshape(shape.N, shape.B)[[1, 2, 4, 5]] == 0).all()


def test_router_zero_weights_ties_go_low(rsq):
    shape = LayerShape(B=1, T=128, d_model=256, G=4, M=4, k=2, d_head=64)
    inp = synth.make_layer_inputs(shape, seed=4)
    inp.W_r = np.zeros_like(inp.W_r)
    o = run_steps(rsq, shape, device_inputs(inp))
    assert (o["idx"].cpu().numpy() == np.array([0, 1])[None, None, :]).all()
    np.testing.assert_allclose(o["omega"].cpu().numpy(), 1.0 / 8, rtol=1e-6)


@pytest.mark.parametrize("B,T,M,k", [(2, 300, 2, 1), (1, 4500, 2, 1), (1, 700, 4, 2)])
def test_router_near_ties_decided_exactly(rsq, B, T, M, k):
    # Every group's columns of W_r differ by a perturbation of ~1e-7, far
    # below the certified fp32 bound, so nearly every group is decided by the
    # fp64 path. The selection must still be the exact one (the oracle's);
    # 4500 rows take the wide token blocks, 300 and 700 the narrow ones.
    shape = LayerShape(B=B, T=T, d_model=1024, G=8, M=M, k=k, d_head=64)
    inp = synth.make_layer_inputs(shape, seed=31)
    rng = np.random.default_rng(3)
    W = inp.W_r.copy()
    for g in range(shape.G):
        for j in range(1, M):
            W[:, g * M + j] = W[:, g * M] + (rng.standard_normal(W.shape[0]) * 1e-7).astype(np.float32)
    inp.W_r = W
    f = oracle._f64_inputs(inp)
    ref = oracle.router(f["x"], f["W_r"], f["b_r"], shape.G, M, k)
    d = device_inputs(inp)
    R = B * T
    idx = torch.empty(R, shape.G, k, dtype=torch.int32, device="cuda")
    r = torch.empty(R, shape.G, k, dtype=torch.float32, device="cuda")
    om = torch.empty_like(r)
    rsq.gqe_router_topk(rsq.GQEConfig.of(shape), d["x"], d["W_r"], d["b_r"], idx, r, om)
    torch.cuda.synchronize()
    assert rsq.gqe_read_status() == 0
    assert np.array_equal(idx.cpu().numpy(), ref["idx"]), "near-tie selection differs from the exact one"
    np.testing.assert_allclose(r.cpu().numpy(), ref["r"], rtol=0, atol=2e-6)
    np.testing.assert_allclose(om.cpu().numpy(), ref["omega"], rtol=0, atol=2e-6)


def _router_on_gpu(rsq, shape, inp):
    d = device_inputs(inp)
    R = shape.R
    idx = torch.empty(R, shape.G, shape.k, dtype=torch.int32, device="cuda")
    r = torch.empty(R, shape.G, shape.k, dtype=torch.float32, device="cuda")
    om = torch.empty_like(r)
    rsq.gqe_router_topk(rsq.GQEConfig.of(shape), d["x"], d["W_r"], d["b_r"], idx, r, om)
    torch.cuda.synchronize()
    assert rsq.gqe_read_status() == 0
    return idx.cpu().numpy(), r.cpu().numpy(), om.cpu().numpy()


def _check_router_exact(rsq, shape, inp):
    f = oracle._f64_inputs(inp)
    ref = oracle.router(f["x"], f["W_r"], f["b_r"], shape.G, shape.M, shape.k)
    idx, r, om = _router_on_gpu(rsq, shape, inp)
    assert np.array_equal(idx, ref["idx"]), "selection differs from the exact one"
    np.testing.assert_allclose(r, ref["r"], rtol=0, atol=2e-6)
    np.testing.assert_allclose(om, ref["omega"], rtol=0, atol=2e-6)
    return ref


@pytest.mark.parametrize("T,M,k", [(300, 2, 1), (4500, 2, 1), (700, 4, 2)])
def test_router_exact_ties_from_swapped_rows(rsq, T, M, k):
    # x has equal columns 2m and 2m+1, and in half of the groups expert 1 (and
    # for M = 4 expert 2) holds expert 0's column with rows 2m and 2m+1
    # swapped: their exact logits are equal for every token, while any fixed
    # summation order rounds the two sums differently. Ties go to the lower
    # index, which only the exact decision gives. d = 1024; 4500 tokens take
    # the wide token blocks.
    shape = LayerShape(B=1, T=T, d_model=1024, G=8, M=M, k=k, d_head=64)
    inp = synth.make_layer_inputs(shape, seed=61, with_dense=False)
    x = inp.x.copy()
    x[:, 1::2] = x[:, 0::2]
    inp.x = x
    W = inp.W_r.copy()
    swapped = np.arange(W.shape[0]).reshape(-1, 2)[:, ::-1].reshape(-1)
    for g in range(0, shape.G, 2):
        for j in range(1, min(M, 3)):
            W[:, g * M + j] = W[swapped, g * M]
    inp.W_r = W
    ref = _check_router_exact(rsq, shape, inp)
    tied = ref["idx"][:, 0::2]
    if k == 1:
        # expert 0 or 1 only loses to nothing in a two-expert group: always 0
        assert (tied[..., 0] == 0).all()


@pytest.mark.parametrize("T,k", [(256, 1), (4500, 1)])
def test_router_sub_ulp_and_1e15_differences(rsq, T, k):
    # In every group expert 1's column is expert 0's with one entry (row i_g)
    # one fp32 ulp larger, and x at row i_g is +-2^-e with e drawn in [20, 70]
    # per token: z_1 - z_0 = x[i_g] * ulp runs from ~1e-15 of the logits
    # (settled by the fp64 bound) down to ~1e-28 (only the exact sums order
    # them). The sign of x[i_g] decides which expert wins.
    shape = LayerShape(B=1, T=T, d_model=1024, G=8, M=2, k=k, d_head=64)
    inp = synth.make_layer_inputs(shape, seed=62, with_dense=False)
    rng = np.random.default_rng(62)
    W = inp.W_r.copy()
    x = inp.x.copy()
    rows = rng.choice(shape.d_model, size=shape.G, replace=False)
    for g in range(shape.G):
        W[:, 2 * g + 1] = W[:, 2 * g]
        W[rows[g], 2 * g + 1] = np.nextafter(W[rows[g], 2 * g], np.float32(np.inf))
        mag = 2.0 ** -rng.integers(20, 71, size=T).astype(np.float64)
        sgn = rng.choice([-1.0, 1.0], size=T)
        x[:, rows[g]] = synth.f32_to_bf16_bits((mag * sgn).astype(np.float32))
    inp.W_r, inp.x = W, x
    ref = _check_router_exact(rsq, shape, inp)
    # both outcomes occur, so the decision is not a fixed tie-break
    assert 0 < ref["idx"].mean() < 1


def test_dispatch_lists_with_separate_scan(rsq):
    # 16 experts x 1026 tiles of 256 tokens = 16416 tile counts: more than one
    # fused scan + scatter launch takes, so the lists come from the
    # stand-alone scan kernel and the scatter kernel (the path of the 1M
    # workload). Router output and lists must be bit-exact.
    shape = LayerShape(B=1, T=262401, d_model=256, G=8, M=2, k=1, d_head=64)
    assert shape.N * shape.B * -(-shape.T // 256) > 16384
    inp = synth.make_layer_inputs(shape, seed=47, with_dense=False)
    f = oracle._f64_inputs(inp)
    ref = oracle.router(f["x"], f["W_r"], f["b_r"], shape.G, shape.M, shape.k)
    lists = oracle.dispatch(ref["idx"], shape.B, shape.T, shape.G, shape.M)
    d = device_inputs(inp)
    cfg = rsq.GQEConfig.of(shape)
    B, T, G, k, dh, R, N = shape.B, shape.T, shape.G, shape.k, shape.d_head, shape.R, shape.N
    dev = torch.device("cuda")
    idx = torch.empty(R, G, k, dtype=torch.int32, device=dev)
    r = torch.empty(R, G, k, dtype=torch.float32, device=dev)
    om = torch.empty_like(r)
    rsq.gqe_router_topk(cfg, d["x"], d["W_r"], d["b_r"], idx, r, om)
    counts = torch.empty(N * B, dtype=torch.int32, device=dev)
    offsets = torch.empty(N * B + 1, dtype=torch.int32, device=dev)
    tok = torch.empty(k * G * R, dtype=torch.int32, device=dev)
    slot_pos = torch.empty(R, G, k, dtype=torch.int32, device=dev)
    Qv = torch.empty(B, G, k, T, dh, dtype=torch.bfloat16, device=dev)
    Qs = torch.empty(B, T, dh, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(rsq.gqe_workspace_bytes(cfg, rsq.GQE_WS_DISPATCH), dtype=torch.uint8, device=dev)
    rsq.gqe_dispatch(cfg, idx, d["x"], d["W_q"], d["W_qs"], counts, offsets, tok, slot_pos, Qv, Qs, ws)
    torch.cuda.synchronize()
    assert rsq.gqe_read_status() == 0
    assert np.array_equal(idx.cpu().numpy(), ref["idx"]), "router indices differ"
    assert np.array_equal(counts.cpu().numpy().reshape(N, B), lists["counts"])
    assert np.array_equal(offsets.cpu().numpy(), lists["offsets"])
    assert np.array_equal(tok.cpu().numpy(), lists["tok"]), "token lists differ"
    assert np.array_equal(slot_pos.cpu().numpy(), lists["slot_pos"])


def test_dispatch_reports_malformed_selections(rsq):
    # Selections the router never writes -- a repeated expert, j = M, a pair
    # not in ascending order -- are dropped by the dispatch kernels (every
    # write stays inside the lists) and reported as GQE_ERR_DEVICE_CHECK; the
    # next call with valid selections is exact again.
    shape = LayerShape(B=2, T=300, d_model=128, G=4, M=3, k=2, d_head=64)
    inp = synth.make_layer_inputs(shape, seed=71)
    f = oracle._f64_inputs(inp)
    good = oracle.router(f["x"], f["W_r"], f["b_r"], shape.G, shape.M, shape.k)["idx"]
    bad = good.copy()
    bad[5, 1] = [1, 1]      # repeated expert: the second entry is dropped
    bad[17, 2, 1] = 3       # j = M: dropped
    bad[400, 0] = [2, 0]    # descending: the second entry is dropped
    d = device_inputs(inp)
    cfg = rsq.GQEConfig.of(shape)
    B, T, G, k, dh, R, N = shape.B, shape.T, shape.G, shape.k, shape.d_head, shape.R, shape.N
    dev = torch.device("cuda")
    ws = torch.empty(rsq.gqe_workspace_bytes(cfg, rsq.GQE_WS_DISPATCH), dtype=torch.uint8, device=dev)

    def run(sel):
        out = {"counts": torch.empty(N * B, dtype=torch.int32, device=dev),
               "offsets": torch.empty(N * B + 1, dtype=torch.int32, device=dev),
               "tok": torch.full((k * G * R,), -1, dtype=torch.int32, device=dev),
               "slot_pos": torch.empty(R, G, k, dtype=torch.int32, device=dev),
               "Qv": torch.zeros(B, G, k, T, dh, dtype=torch.bfloat16, device=dev),
               "Qs": torch.empty(B, T, dh, dtype=torch.bfloat16, device=dev)}
        idx = torch.from_numpy(np.ascontiguousarray(sel)).to(dev)
        rsq.gqe_dispatch(cfg, idx, d["x"], d["W_q"], d["W_qs"], out["counts"], out["offsets"],
                         out["tok"], out["slot_pos"], out["Qv"], out["Qs"], ws)
        torch.cuda.synchronize()
        return out, rsq.gqe_read_status()

    out, st = run(bad)
    assert st == rsq.GQE_ERR_DEVICE_CHECK
    assert rsq.gqe_read_status() == 0  # reading clears it
    assert int(out["counts"].sum()) == k * G * R - 3
    assert int(out["offsets"][-1]) == k * G * R - 3
    tok = out["tok"].cpu().numpy()
    assert (tok[:k * G * R - 3] >= 0).all() and (tok[:k * G * R - 3] < T).all()
    out, st = run(good)
    assert st == 0
    ref = oracle.dispatch(good, B, T, G, shape.M)
    assert np.array_equal(out["tok"].cpu().numpy(), ref["tok"])
    assert np.array_equal(out["slot_pos"].cpu().numpy(), ref["slot_pos"])


def test_device_wait_timeout_is_reported_and_recoverable(rsq):
    rsq.gqe_selftest_wait_timeout(2_000_000)  # 2 ms bound on a barrier nothing completes
    assert rsq.gqe_read_status() == rsq.GQE_ERR_TIMEOUT
    assert rsq.gqe_read_status() == 0  # reading clears it
    shape = synth.TINY
    inp = synth.make_layer_inputs(shape, seed=1)
    ref = oracle.gqe_layer(inp)
    y, _ = run_layer(rsq, shape, device_inputs(inp))
    assert_close(y, ref["y"], "y after timeout self-test")


EM_CASES = ["tiny", "ragged_b2", "pool4_k2_skew", "k_equals_m", "t5_dh32"]


@pytest.mark.parametrize("name", EM_CASES)
def test_expert_major_layout_matches_oracle(rsq, name):
    # Compacted, expert-major query tiles (rows masked by their positions):
    # the same Q rows, and slots and y within the layer tolerance.
    shape, kw = CASES[name]
    inp = synth.make_layer_inputs(shape, seed=101, **kw)
    ref = oracle.gqe_layer(inp)
    d = device_inputs(inp)
    o = run_steps(rsq, shape, d)
    e = run_expert_major(rsq, shape, d, o)
    assert torch.equal(e["Qe"], qv_in_list_order(o, shape)), "Q rows differ between layouts"
    assert torch.equal(e["Qs"], o["Qs"])
    assert_close(e["slots"], ref["slots"], "slots (expert-major)", allow_scale=shape.T < 128)
    assert_close(e["y"], ref["y"], "y (expert-major)", allow_scale=shape.T < 128)


def test_expert_major_long_sequences_equal_slot_major(rsq):
    # No split-KV at this size (27 streams x 28 tile pairs): both layouts run
    # the same online softmax over the same K/V tiles for every row, so the
    # slots are bitwise equal; three sequences, 12 experts, k = 2, ragged tiles.
    shape = LayerShape(B=3, T=7000, d_model=128, G=4, M=3, k=2, d_head=32)
    inp = synth.make_layer_inputs(shape, seed=23)
    d = device_inputs(inp)
    o = run_steps(rsq, shape, d)
    e = run_expert_major(rsq, shape, d, o)
    assert torch.equal(e["slots"], o["slots"]), "expert-major slots differ from slot-major"
    assert torch.equal(e["y"], o["y"])
    # The whole layer with the flag gives the same y.
    cfg = rsq.GQEConfig.of(shape, rsq.GQE_FLAG_EXPERT_MAJOR)
    ws = torch.empty(rsq.gqe_workspace_bytes(cfg, rsq.GQE_WS_LAYER), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(o["y"])
    rsq.gqe_layer_fwd(cfg, d["x"], d["W_r"], d["b_r"], d["W_q"], d["W_qs"], d["W_k"], d["W_v"],
                      d["W_o"], y, ws)
    torch.cuda.synchronize()
    assert rsq.gqe_read_status() == 0
    assert torch.equal(y, o["y"])


MODES = ["group_mean", "hard", "weighted_concat"]


@pytest.mark.parametrize("name", ["ragged_b2", "pool4_k2_skew", "t5_dh32"])
@pytest.mark.parametrize("mode", MODES)
def test_output_constructions_match_oracle(rsq, name, mode):
    # The ablation constructions (hard concatenation; weighted concatenation by
    # the in-group probability; both without the weighted slot and the shared
    # head) and the group-mean weighted slot, through the step calls and the
    # whole-layer call, against the oracle's construction of the same name.
    import dataclasses
    shape, kw = CASES[name]
    inp = synth.make_layer_inputs(shape, seed=103, **kw)
    S = oracle.mode_slots(mode, shape.G, shape.k)
    inp = dataclasses.replace(inp, W_o=inp.W_o[:S * shape.d_head].copy())
    ref = oracle.gqe_layer(inp, mode=mode)
    flags = rsq.OUTPUT_MODE_FLAGS[mode]
    d = device_inputs(inp)
    o = run_steps(rsq, shape, d, flags)
    _check_integer_parts(o, ref, shape)
    want_w = {"group_mean": ref["r"] / shape.G, "hard": ref["omega"],
              "weighted_concat": np.take_along_axis(ref["p"], ref["idx"].astype(np.int64), axis=-1)}[mode]
    np.testing.assert_allclose(o["omega"].cpu().numpy(), want_w, rtol=0, atol=2e-6)
    short = shape.T < 128
    assert_close(o["slots"], ref["slots"], f"slots ({mode})", allow_scale=short)
    assert_close(o["y"], ref["y"], f"y ({mode})", allow_scale=short)
    y, _ = run_layer(rsq, shape, d, flags)
    assert torch.equal(y, o["y"]), "gqe_layer_fwd differs from the step calls"
