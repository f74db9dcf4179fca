"""Host-side logic of bench.py (CPU only): the FLOP model against the values
the active-FLOP formula gives for the measured workloads, the launch counts,
and the configuration of the opt-in expert-pool sweep."""
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


def test_launch_counts():
    # seq2k: 8 dispatch tiles x 16 experts fit the fused scan + scatter.
    assert bench.launches(synth.SEQ2K) == {"router": 1, "dispatch": 3, "kv": 1, "attention": 1,
                                           "output": 1}
    assert bench.layer_launches(synth.SEQ2K) == 8
    # d_head = 32: the weighted slot is its own kernel before W_O.
    assert bench.launches(synth.TINY)["output"] == 2


def test_pool_sweep_configuration():
    for name, skew in bench.POOL_SWEEP:
        s = bench.WORKLOADS[name]
        assert (s.G, s.M, s.T, s.d_model) == (8, 4, 32768, 1024)
        if skew:
            assert (s.M, s.k) in synth.SKEW_BETA
