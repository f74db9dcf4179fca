"""Host-side logic of bench.py (CPU only): the FLOP model against the values
the active-FLOP formula gives for the measured workloads, the launch counts,
the per-call roofline fractions, the short summary table and the
configuration of the expert-pool sweep."""
import math

import bench
import synth


def test_attention_flops_match_the_active_pair_count():
    # 4 * d_head FLOPs per unmasked (query, key) pair, T(T+1)/2 pairs per
    # causal stream; 9 streams for GQE (8 routed + shared), 16 for dense.
    s = synth.SEQ2K
    gqe, dense = bench.flops(s)["attention"], bench.flops(s, dense=True)["attention"]
    assert math.isclose(gqe, 4 * 64 * 9 * 2048 * 2049 / 2)
    assert math.isclose(dense, 4 * 64 * 16 * 2048 * 2049 / 2)
    assert round(gqe / 1e9, 2) == 4.83 and round(dense / 1e9, 2) == 8.59
    # 1M tokens: 1267 / 2252 TFLOP.
    s = synth.SEQ1M
    assert round(bench.flops(s)["attention"] / 1e12) == 1267
    assert round(bench.flops(s, dense=True)["attention"] / 1e12) == 2252


def test_projection_flops():
    s = synth.SEQ2K
    f = bench.flops(s)
    R, d, dh = s.R, s.d_model, s.d_head
    assert f["q"] == 2 * R * d * dh * 9
    assert f["kv"] == 4 * R * d * dh * 8
    assert f["wo"] == 2 * R * 10 * dh * d
    assert f["router"] == 2 * R * d * 16


def test_backward_flops():
    # seq2k (B=1, T=2048, d=1024, G=8, M=2, k=1, dh=64): attention 5 products
    # x 2*64 FLOPs x 2048*2049/2 pairs x 9 streams; dS and dW_O 2*2048*1024*640
    # each; dx and the weight gradients 2*2048*1024*(1024 + 64 + 1024 + 16) each.
    s = synth.SEQ2K
    attn = 5 * 128 * (2048 * 2049 // 2) * 9
    proj = 2 * (2 * 2048 * 1024 * 640) + 2 * (2 * 2048 * 1024 * 2128)
    assert bench.backward_flops(s) == attn + proj
    assert round(bench.backward_flops(s) / 1e9, 1) == 35.3


def test_launch_counts():
    # seq2k and 4 x 8k: the tile counts (8 or 128 tiles x 16 experts) fit the
    # fused scan + scatter after the count kernel; 1M tokens: 4096 x 16 tile
    # counts take the separate scan.
    assert bench.launches(synth.SEQ2K) == {"router": 1, "dispatch": 3, "kv": 1, "attention": 1,
                                           "output": 1}
    # gqe_layer_fwd at seq2k takes the short-batch path: router, shared-head Q
    # GEMM, fused K/V/Q GEMM, attention, W_O.
    assert bench.layer_launches(synth.SEQ2K) == 5
    # 4 x 8k: the step kernels (router, 3 dispatch, K/V, attention, W_O) + shared Q.
    assert bench.layer_launches(synth.BATCH4_8K) == 8
    assert bench.launches(synth.BATCH4_8K)["dispatch"] == 3
    assert bench.launches(synth.SEQ1M)["dispatch"] == 4
    # d_head = 32: the weighted slot is its own kernel before W_O.
    assert bench.launches(synth.TINY)["output"] == 2


def test_pool_sweep_configuration():
    for name, skew in bench.POOL_SWEEP:
        s = bench.WORKLOADS[name]
        assert (s.G, s.M, s.T, s.d_model) == (8, 4, 32768, 1024)
        if skew:
            assert (s.M, s.k) in synth.SKEW_BETA


def test_call_fractions():
    # 1 ms per call over 2 steps: each fraction is work / 0.5 ms / peak.
    s = synth.SEQ2K
    pk = {"bf16": 1000.0, "hbm": 5000.0}
    per = {c: 1.0 for c in ("router", "dispatch", "kv", "attention", "output")}
    fr = bench.call_fractions(s, per, 2, pk)
    rb = 2048 * 1024 * 2 + 1024 * 16 * 4 + 2048 * 8 * 12
    assert math.isclose(fr["router_hbm_frac"], round(rb / 0.5e-3 / 1e9 / 5000.0, 4))
    f = bench.flops(s)
    assert math.isclose(fr["kv_tensor_frac"], round(f["kv"] / 0.5e-3 / 1e12 / 1000.0, 4))
    assert math.isclose(fr["dispatch_tensor_frac"], round(f["q"] / 0.5e-3 / 1e12 / 1000.0, 4))
    assert math.isclose(fr["attention_tensor_frac"], round(f["attention"] / 0.5e-3 / 1e12 / 1000.0, 4))


def test_summary_table():
    out = {"config": {"workload": "seq2k: x"}, "ms_per_step": 0.07, "roofline": {"frac": 0.1},
           "dense_gqa": {"ms_per_step": 0.06, "speedup_gqe_over_dense": 0.857},
           "fractions": {"router_hbm_frac": 0.05},
           "sweep": [{"workload": "seq32k: y", "gqe_ms": 2.0, "dense_ms": 3.0, "speedup": 1.5,
                      "attn_frac_of_bf16_peak": 0.5}],
           "pool_sweep": [{"workload": "pool4_k1 (skewed): z", "gqe_ms": 1.0, "dense_ms": 3.0,
                           "speedup": 3.0, "attn_frac_of_bf16_peak": 0.4, "hot_expert_share": 0.8}]}
    rows = bench.summary_of(out)["per_workload"]
    assert [r["workload"] for r in rows] == ["seq2k", "seq32k", "pool4_k1 (skewed)"]
    assert rows[0]["speedup"] == 0.857 and rows[0]["router_hbm_frac"] == 0.05
    assert rows[2]["hot_expert_share"] == 0.8
