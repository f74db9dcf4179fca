"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test checks the oracle against something it does not compute the same
way: values worked by hand from the definitions (tests/golden), closed forms,
brute force on tiny inputs, a library attention routine on the dense special
case, and the invariants the pages state for the layer ("Grouped Query
Experts: Mixture-of-Experts on GQA Self-Attention").
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import LayerShape, bf16_to_f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _num(s):
    return math.log(float(s[2:])) if isinstance(s, str) and s.startswith("ln") else float(s)


# --------------------------------------------------------------------------
# input generator
# --------------------------------------------------------------------------

def test_synth_is_deterministic_and_normal():
    a = synth.normal_f64(7, 3, 200001)
    b = synth.normal_f64(7, 3, 200001)
    assert np.array_equal(a, b)
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1.0) < 0.01
    # chunked draw equals the one-shot draw
    c = np.concatenate([synth.normal_f64(7, 3, 100000, 0), synth.normal_f64(7, 3, 100001, 100000)])
    assert np.array_equal(a, c)
    assert not np.array_equal(a[:1000], synth.normal_f64(7, 4, 1000))


def test_bf16_rounding_nearest_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 3.0e38],
                    dtype=np.float32)
    got = synth.bf16_to_f64(synth.f32_to_bf16_bits(vals))
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> even (1.0); 1 + 3*2^-8 -> 1 + 2^-6
    assert list(got[:5]) == [1.0, 1.0, 1.0 + 2 ** -6, 1.0, -2.5]
    assert torch.equal(torch.tensor(got[:5], dtype=torch.float32),
                       torch.tensor(vals[:5]).to(torch.bfloat16).to(torch.float32))


# --------------------------------------------------------------------------
# router (a1-a4)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("case", _golden("router_hand_cases.json")["cases"],
                         ids=lambda c: c["name"])
def test_router_hand_cases(case):
    G, M, k = case["G"], case["M"], case["k"]
    b = np.array([_num(v) for v in case["b"]])
    x = np.ones((3, 8))
    rt = oracle.router(x, np.zeros((8, G * M)), b, G, M, k)
    for row in range(3):
        assert rt["idx"][row].tolist() == case["idx"]
        np.testing.assert_allclose(rt["p"][row], case["p"], rtol=0, atol=1e-15)
        np.testing.assert_allclose(rt["r"][row], case["r"], rtol=0, atol=1e-15)
        np.testing.assert_allclose(rt["omega"][row], case["omega"], rtol=0, atol=1e-15)


def test_router_logits_one_hot_rows():
    # x = e_i picks row i of W_r: pins the orientation of x . W_r (+ b).
    rng = np.random.default_rng(1)
    d, G, M = 12, 3, 2
    W = rng.standard_normal((d, G * M))
    b = rng.standard_normal(G * M)
    x = np.eye(d)
    rt = oracle.router(x, W, b, G, M, 1)
    np.testing.assert_allclose(rt["z"], W + b[None, :], rtol=0, atol=1e-15)


def test_router_softmax_two_expert_closed_form():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((50, 16))
    W = rng.standard_normal((16, 8))
    rt = oracle.router(x, W, None, 4, 2, 1)
    z = x @ W
    for g in range(4):
        p0 = 1.0 / (1.0 + np.exp(z[:, 2 * g + 1] - z[:, 2 * g]))
        np.testing.assert_allclose(rt["p"][:, g, 0], p0, rtol=1e-13)


@pytest.mark.parametrize("M,k", [(2, 1), (4, 1), (4, 2), (4, 3), (3, 3)])
def test_router_topk_brute_force(M, k):
    # Brute force over every k-subset: the selected set is the one whose
    # members all beat every non-member (higher logit, or equal and lower
    # index). Integer-valued logits make ties frequent.
    rng = np.random.default_rng(3 + M * 10 + k)
    G, R = 3, 40
    W = np.zeros((4, G * M))
    x = np.zeros((R, 4))
    rows = []
    for t in range(R):
        b = rng.integers(-2, 3, size=G * M).astype(np.float64)
        rt = oracle.router(x[t:t + 1], W, b, G, M, k)
        for g in range(G):
            zz = b[g * M:(g + 1) * M]
            best = [S for S in itertools.combinations(range(M), k)
                    if all((zz[j] > zz[i]) or (zz[j] == zz[i] and j < i)
                           for j in S for i in range(M) if i not in S)]
            assert len(best) == 1
            assert rt["idx"][0, g].tolist() == list(best[0])
        rows.append(rt)


def test_router_invariants_random():
    s = LayerShape(B=2, T=64, d_model=32, G=4, M=4, k=2, d_head=8)
    inp = synth.make_layer_inputs(s, seed=11)
    rt = oracle.router(bf16_to_f64(inp.x), inp.W_r, inp.b_r, s.G, s.M, s.k)
    idx = rt["idx"]
    assert idx.dtype == np.int32 and idx.shape == (s.R, s.G, s.k)
    assert (np.diff(idx, axis=-1) > 0).all() and idx.min() >= 0 and idx.max() < s.M
    np.testing.assert_allclose(rt["r"].sum(-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(rt["omega"].sum((1, 2)), 1.0, rtol=1e-14)
    np.testing.assert_allclose(rt["p"].sum(-1), 1.0, rtol=1e-14)


def test_router_zero_weights_selects_lowest_indices():
    G, M, k = 8, 4, 2
    rt = oracle.router(np.ones((5, 16)), np.zeros((16, G * M)), None, G, M, k)
    assert (rt["idx"] == np.arange(k)[None, None, :]).all()
    np.testing.assert_allclose(rt["r"], 1.0 / k)
    np.testing.assert_allclose(rt["omega"], 1.0 / (k * G))


def test_router_exact_tie_through_reordered_sum():
    # Column 1 holds the entries of column 0 in another row order and x is the
    # same on the permuted rows, so the exact logits are equal while a blocked
    # fp64 sum may round them apart; the exact fallback must see the tie and
    # pick the lower index.
    rng = np.random.default_rng(5)
    d = 1024
    w0 = rng.standard_normal(d).astype(np.float32).astype(np.float64)
    perm = rng.permutation(d)
    W = np.stack([w0, w0[perm]], axis=1)
    x = np.full((4, d), 0.37109375)  # a bf16 value
    rt = oracle.router(x, W, None, 1, 2, 1)
    assert (rt["idx"] == 0).all()
    # A perturbation of one x entry by 2^-20 decides the order; the oracle's
    # decision must agree with the correctly rounded exact logits.
    x2 = x.copy()
    x2[:, perm[0]] += 2.0 ** -20
    z0 = math.fsum(x2[0] * W[:, 0])
    z1 = math.fsum(x2[0] * W[:, 1])
    assert z0 != z1
    rt2 = oracle.router(x2, W, None, 1, 2, 1)
    assert (rt2["idx"][:, 0, 0] == (0 if z0 > z1 else 1)).all()


def _bf16_value(v: float) -> float:
    return float(bf16_to_f64(synth.f32_to_bf16_bits(np.array([v], dtype=np.float32)))[0])


def _sub_ulp_pair(seed: int, tiny: float):
    """Two router columns equal except one entry one fp32 ulp apart, and an x
    row whose entry on that row is `tiny`: the exact logits differ by
    tiny * ulp, far below one fp64 ulp of the logits themselves."""
    rng = np.random.default_rng(seed)
    d = 1024
    w0 = (rng.standard_normal(d) / 32).astype(np.float32)
    i0 = int(rng.integers(d))
    w1 = w0.copy()
    w1[i0] = np.nextafter(w0[i0], np.float32(np.inf))
    x = bf16_to_f64(synth.f32_to_bf16_bits(rng.standard_normal(d).astype(np.float32)))
    x[i0] = _bf16_value(tiny)
    return x, np.stack([w0, w1], axis=1).astype(np.float64), i0


@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_router_sub_ulp_difference_decided_exactly(sign):
    # z_1 - z_0 = x[i0] * ulp(w0[i0]): about 2^-88, so the correctly rounded
    # logits are equal and only the exact values order them. x[i0] > 0 makes
    # expert 1 the larger (selected although it has the higher index);
    # x[i0] < 0 makes expert 0 the larger.
    x, W, i0 = _sub_ulp_pair(17, sign * 2.0 ** -60)
    assert math.fsum(x * W[:, 0]) == math.fsum(x * W[:, 1])  # rounding alone cannot decide
    rt = oracle.router(x[None, :], W, None, 1, 2, 1)
    assert rt["idx"][0, 0, 0] == (1 if sign > 0 else 0)


def test_router_exact_selection_matches_rational_arithmetic():
    # Independent exact method: Fraction sums of the same terms. Near-tied
    # groups of 4 experts (columns one ulp apart at one row, the x entry there
    # between 2^-70 and 2^-10), k = 2; the oracle's selection must be the one
    # the rational logits give (largest first, ties to the lower index).
    from fractions import Fraction
    rng = np.random.default_rng(41)
    d, M, k = 256, 4, 2
    for case in range(24):
        w = (rng.standard_normal(d) / 16).astype(np.float32)
        cols = []
        rows_hit = rng.choice(d, size=M, replace=False)
        for j in range(M):
            c = w.copy()
            steps = int(rng.integers(-1, 2))  # -1, 0 or +1 ulp at this column's row
            for _ in range(abs(steps)):
                c[rows_hit[j]] = np.nextafter(c[rows_hit[j]], np.float32(np.inf * steps))
            cols.append(c)
        W = np.stack(cols, axis=1).astype(np.float64)
        x = bf16_to_f64(synth.f32_to_bf16_bits(rng.standard_normal(d).astype(np.float32)))
        for r in rows_hit:
            x[r] = _bf16_value(float(rng.choice([-1.0, 1.0])) * 2.0 ** -float(rng.integers(10, 71)))
        b = np.zeros(M)
        rt = oracle.router(x[None, :], W, b, 1, M, k)
        zq = [sum((Fraction(float(xi)) * Fraction(float(wi)) for xi, wi in zip(x, W[:, j])), Fraction(0))
              for j in range(M)]
        want = sorted(sorted(range(M), key=lambda j: (-zq[j], j))[:k])
        assert rt["idx"][0, 0].tolist() == want, (case, zq)


def test_router_skew_bias_gives_80_percent():
    # Bias beta on expert 0 of each group: P(hot expert in top-k) = 0.80 for
    # iid N(0,1) logits (the load-skew workload).
    for (M, k), beta in synth.SKEW_BETA.items():
        s = LayerShape(B=1, T=8192, d_model=64, G=8, M=M, k=k, d_head=8)
        inp = synth.make_layer_inputs(s, seed=21, skew=True, with_dense=False)
        rt = oracle.router(bf16_to_f64(inp.x), inp.W_r, inp.b_r, s.G, s.M, s.k)
        frac = (rt["idx"] == 0).any(axis=-1).mean()
        assert abs(frac - 0.80) < 0.015, (M, k, frac)


# --------------------------------------------------------------------------
# dispatch (a5)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("M,k", [(2, 1), (4, 2), (3, 3)])
def test_dispatch_matches_selection(M, k):
    rng = np.random.default_rng(30 + M + k)
    B, T, G = 3, 37, 2
    idx = np.stack([np.sort(rng.choice(M, size=k, replace=False)) for _ in range(B * T * G)])
    idx = idx.reshape(B * T, G, k).astype(np.int32)
    dp = oracle.dispatch(idx, B, T, G, M)
    N = G * M
    counts, offsets, tok, sp = dp["counts"], dp["offsets"], dp["tok"], dp["slot_pos"]
    assert offsets[0] == 0 and offsets[-1] == k * G * B * T
    assert (counts.reshape(G, M, B).sum(axis=1) == k * T).all()
    for e in range(N):
        g, j = divmod(e, M)
        for b in range(B):
            lo, hi = offsets[e * B + b], offsets[e * B + b + 1]
            want = [t for t in range(T) if j in idx[b * T + t, g]]
            assert hi - lo == counts[e, b] == len(want)
            assert tok[lo:hi].tolist() == want
    for row in range(B * T):
        b, t = divmod(row, T)
        for g in range(G):
            for s in range(k):
                e = g * M + idx[row, g, s]
                p = sp[row, g, s]
                assert offsets[e * B + b] <= p < offsets[e * B + b + 1] and tok[p] == t


def test_dispatch_empty_lists():
    B, T, G, M = 2, 5, 2, 3
    idx = np.zeros((B * T, G, 1), dtype=np.int32)  # only j = 0 ever selected
    dp = oracle.dispatch(idx, B, T, G, M)
    assert dp["counts"].reshape(G, M, B)[:, 1:].sum() == 0
    off = dp["offsets"]
    for e in range(G * M):
        if e % M:
            assert off[e * B] == off[e * B + 1] == off[e * B + 2]


# --------------------------------------------------------------------------
# projections (a6, a7)
# --------------------------------------------------------------------------

def test_kv_layout_one_hot_rows():
    rng = np.random.default_rng(6)
    B, T, G, dh, d = 2, 3, 4, 5, 6
    W = rng.standard_normal((d, G * dh))
    x = np.zeros((B * T, d))
    for row in range(B * T):
        x[row, row % d] = 1.0
    K = oracle.kv_proj(x, W, B, T, G, dh)
    for b in range(B):
        for t in range(T):
            i = (b * T + t) % d
            for g in range(G):
                assert np.array_equal(K[b, g, t], W[i, g * dh:(g + 1) * dh])


def test_q_routed_one_hot_rows():
    rng = np.random.default_rng(7)
    B, T, G, M, k, dh, d = 1, 6, 2, 3, 2, 4, 6
    W = rng.standard_normal((d, G * M * dh))
    x = np.eye(d)
    idx = np.stack([np.sort(rng.choice(M, size=k, replace=False)) for _ in range(T * G)])
    idx = idx.reshape(T, G, k).astype(np.int32)
    Qv = oracle.q_routed(x, W, idx, B, T, G, M, dh)
    for t in range(T):
        for g in range(G):
            for s in range(k):
                e = g * M + idx[t, g, s]
                assert np.array_equal(Qv[0, g, s, t], W[t, e * dh:(e + 1) * dh])


# --------------------------------------------------------------------------
# attention (a8, a9)
# --------------------------------------------------------------------------

def test_attention_closed_forms():
    rng = np.random.default_rng(8)
    T, dh = 33, 16
    q = rng.standard_normal((T, dh))
    K = rng.standard_normal((T, dh))
    V = rng.standard_normal((T, dh))
    o = oracle.causal_attention(q, K, V)
    assert np.array_equal(o[0], V[0])                       # only key 0 is visible
    c = rng.standard_normal(dh)
    oc = oracle.causal_attention(q, K, np.tile(c, (T, 1)))
    np.testing.assert_allclose(oc, np.tile(c, (T, 1)), rtol=0, atol=1e-14)
    oz = oracle.causal_attention(np.zeros((T, dh)), K, V)    # uniform weights
    prefix_mean = np.cumsum(V, axis=0) / np.arange(1, T + 1)[:, None]
    np.testing.assert_allclose(oz, prefix_mean, rtol=0, atol=1e-13)


def test_attention_sharp_scores_pick_own_row():
    T = dh = 16
    K = 40.0 * np.eye(T)
    q = 40.0 * np.eye(T)
    V = np.random.default_rng(9).standard_normal((T, dh))
    o = oracle.causal_attention(q, K, V)
    np.testing.assert_allclose(o, V, rtol=0, atol=1e-12)


def test_attention_matches_torch_sdpa_fp64():
    rng = np.random.default_rng(10)
    T, dh = 70, 32
    q, K, V = (rng.standard_normal((T, dh)) for _ in range(3))
    o = oracle.causal_attention(q, K, V, block=16)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None, None], torch.tensor(K)[None, None], torch.tensor(V)[None, None],
        is_causal=True)[0, 0].numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-13)


def test_attention_sampled_rows_equal_full():
    rng = np.random.default_rng(12)
    T, dh = 90, 8
    q, K, V = (rng.standard_normal((T, dh)) for _ in range(3))
    full = oracle.causal_attention(q, K, V)
    rows = np.array([0, 5, 89, 44])
    part = oracle.causal_attention(q[rows], K, V, rows=rows)
    np.testing.assert_allclose(part, full[rows], rtol=0, atol=1e-14)


# --------------------------------------------------------------------------
# whole layer
# --------------------------------------------------------------------------

def _tiny(B=1, T=16, d=32, G=2, M=2, k=1, dh=8, seed=13, **kw):
    return synth.make_layer_inputs(LayerShape(B, T, d, G, M, k, dh), seed=seed, **kw)


def test_dense_gqa_matches_torch_sdpa():
    inp = _tiny(B=2, T=24, G=2, M=3, dh=8)
    s = inp.shape
    dn = oracle.gqa_dense_layer(inp)
    x = torch.tensor(bf16_to_f64(inp.x)).reshape(s.B, s.T, s.d_model)
    Wq = torch.tensor(bf16_to_f64(inp.W_q))
    Wk = torch.tensor(bf16_to_f64(inp.W_k))
    Wv = torch.tensor(bf16_to_f64(inp.W_v))
    q = (x @ Wq).reshape(s.B, s.T, s.N, s.d_head).transpose(1, 2)
    k = (x @ Wk).reshape(s.B, s.T, s.G, s.d_head).transpose(1, 2).repeat_interleave(s.M, dim=1)
    v = (x @ Wv).reshape(s.B, s.T, s.G, s.d_head).transpose(1, 2).repeat_interleave(s.M, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
    o = o.transpose(1, 2).reshape(s.R, s.N * s.d_head)
    np.testing.assert_allclose(dn["O"], o.numpy(), rtol=0, atol=1e-13)
    y = o @ torch.tensor(bf16_to_f64(inp.W_o_dense))
    np.testing.assert_allclose(dn["y"], y.numpy(), rtol=0, atol=1e-13)


def test_k_equals_m_reproduces_dense_gqa():
    # With k = M every expert is selected, slots (g, s) are the dense heads
    # g*M + s, and W_O = [W_O_dense; 0; 0] gives the dense layer's y.
    inp = _tiny(B=2, T=20, G=2, M=2, k=2, dh=8, seed=14)
    s = inp.shape
    dh = s.d_head
    wo = np.zeros_like(inp.W_o)
    wo[:s.N * dh] = inp.W_o_dense
    inp.W_o = wo
    gq = oracle.gqe_layer(inp)
    dn = oracle.gqa_dense_layer(inp)
    np.testing.assert_allclose(gq["slots"][:, :s.N * dh], dn["O"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(gq["y"], dn["y"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(gq["K"], dn["K"], rtol=0, atol=0)


def test_routed_slots_are_dense_heads_selected():
    # Second formulation, brute force at T <= 16: compute every head densely,
    # then pick for each token the columns of its selected experts.
    inp = _tiny(B=2, T=16, G=3, M=3, k=2, dh=8, seed=15)
    s = inp.shape
    dh = s.d_head
    gq = oracle.gqe_layer(inp)
    dn = oracle.gqa_dense_layer(inp)
    O = dn["O"].reshape(s.R, s.N, dh)
    for row in range(s.R):
        for g in range(s.G):
            for si in range(s.k):
                h = g * s.M + gq["idx"][row, g, si]
                slot = g * s.k + si
                np.testing.assert_allclose(gq["slots"][row, slot * dh:(slot + 1) * dh], O[row, h],
                                           rtol=0, atol=1e-13)
    # the shared head is an extra head on KV group 0
    x = bf16_to_f64(inp.x)
    for b in range(s.B):
        qs = x[b * s.T:(b + 1) * s.T] @ bf16_to_f64(inp.W_qs)
        os_ = oracle.causal_attention(qs, gq["K"][b, 0], gq["V"][b, 0])
        sh = s.k * s.G
        np.testing.assert_allclose(gq["slots"][b * s.T:(b + 1) * s.T, sh * dh:(sh + 1) * dh], os_,
                                   rtol=0, atol=1e-13)


def test_weighted_slot_uniform_router_is_mean():
    inp = _tiny(G=4, M=2, k=1, seed=16)
    inp.W_r = np.zeros_like(inp.W_r)
    s = inp.shape
    dh = s.d_head
    gq = oracle.gqe_layer(inp)
    routed = gq["slots"][:, :s.G * dh].reshape(s.R, s.G, dh)
    w = gq["slots"][:, (s.G + 1) * dh:]
    np.testing.assert_allclose(w, routed.mean(axis=1), rtol=0, atol=1e-14)


def test_weighted_slot_hand_weights():
    # Golden case 1 (omega = 0.6, 0.4) applied to the attention outputs.
    inp = _tiny(G=2, M=2, k=1, seed=17)
    inp.W_r = np.zeros_like(inp.W_r)
    inp.b_r = np.array([math.log(3.0), 0.0, 0.0, 0.0], dtype=np.float64)
    s = inp.shape
    dh = s.d_head
    gq = oracle.gqe_layer(inp)
    o0 = gq["slots"][:, 0:dh]
    o1 = gq["slots"][:, dh:2 * dh]
    np.testing.assert_allclose(gq["slots"][:, 3 * dh:], 0.6 * o0 + 0.4 * o1, rtol=0, atol=1e-14)


def test_causality_whole_layer():
    inp = _tiny(T=16, seed=18)
    a = oracle.gqe_layer(inp)
    inp.x = inp.x.copy()
    inp.x[9:] = synth.normal_bf16(99, 1, inp.x[9:].shape)
    b = oracle.gqe_layer(inp)
    np.testing.assert_array_equal(a["y"][:9], b["y"][:9])
    assert not np.allclose(a["y"][9:], b["y"][9:])


def test_batch_concatenation_invariance():
    inp = _tiny(B=2, T=12, seed=19)
    both = oracle.gqe_layer(inp)
    s = inp.shape
    for b in range(2):
        one = synth.LayerInputs(LayerShape(1, s.T, s.d_model, s.G, s.M, s.k, s.d_head),
                                inp.x[b * s.T:(b + 1) * s.T], inp.W_r, inp.b_r, inp.W_q,
                                inp.W_qs, inp.W_k, inp.W_v, inp.W_o, inp.W_o_dense)
        o = oracle.gqe_layer(one)
        np.testing.assert_allclose(both["y"][b * s.T:(b + 1) * s.T], o["y"], rtol=0, atol=1e-14)


def test_sampled_rows_equal_full_layer():
    inp = _tiny(B=2, T=16, seed=20)
    full = oracle.gqe_layer(inp)
    rows = np.array([0, 7, 16, 31])
    part = oracle.gqe_layer(inp, rows=rows)
    np.testing.assert_allclose(part["y"], full["y"][rows], rtol=0, atol=1e-14)
    np.testing.assert_allclose(part["slots"], full["slots"][rows], rtol=0, atol=1e-14)


def test_row_blocked_sampled_layer_equals_full_layer(monkeypatch):
    # The long-sequence evaluation (x widened 5 rows at a time, each group's
    # K/V built only up to the last evaluated position) gives the full layer's
    # values at the evaluated rows: router, lists, K/V, slots and y.
    s = LayerShape(B=2, T=23, d_model=64, G=3, M=3, k=2, d_head=8)
    inp = synth.make_layer_inputs(s, seed=44, skew=False)
    full = oracle.gqe_layer(inp)
    monkeypatch.setattr(oracle, "_ROW_BLOCK", 5)
    rows = np.array([0, 4, 5, 11, 23, 27, 45])
    part = oracle.gqe_layer(inp, rows=rows, full_kv=False)
    for key in ("idx", "counts", "offsets", "tok", "slot_pos"):
        assert np.array_equal(part[key], full[key]), key
    for key in ("r", "omega", "p", "z"):
        np.testing.assert_allclose(part[key], full[key], rtol=0, atol=1e-14)
    b, t = rows // s.T, rows % s.T
    np.testing.assert_allclose(part["K_rows"], full["K"][b, :, t], rtol=0, atol=1e-14)
    np.testing.assert_allclose(part["V_rows"], full["V"][b, :, t], rtol=0, atol=1e-14)
    np.testing.assert_allclose(part["slots"], full["slots"][rows], rtol=0, atol=1e-13)
    np.testing.assert_allclose(part["y"], full["y"][rows], rtol=0, atol=1e-13)


def test_published_setting_counts():
    g = _golden("published_setting.json")
    ms = g["main_setting"]
    shape = LayerShape(B=1, T=8, d_model=64, G=ms["G"], M=ms["N"] // ms["G"], k=ms["k"], d_head=4)
    assert oracle.active_query_heads(shape) == g["active_query_heads"]["value"]
    assert shape.N == g["active_query_heads"]["of"]
    assert shape.n_slots == g["wo_rows_in_head_units"]["value"]
    inp = synth.make_layer_inputs(shape, seed=22)
    gq = oracle.gqe_layer(inp)
    assert gq["slots"].shape[1] == shape.n_slots * shape.d_head
    assert inp.W_o.shape == (shape.n_slots * shape.d_head, shape.d_model)
    # active (token, query-head) attention rows: one per selected expert + shared
    assert gq["idx"].size + shape.R == oracle.active_query_heads(shape) * shape.R


def _decode_case(seed, B=2, T=9, G=2, M=3, k=2, dh=32):
    s = LayerShape(B=B, T=T, d_model=64, G=G, M=M, k=k, d_head=dh)
    inp = synth.make_layer_inputs(s, seed=seed)
    f = oracle._f64_inputs(inp)
    L = T - 1
    K = oracle.kv_proj(f["x"], f["W_k"], B, T, G, dh)
    V = oracle.kv_proj(f["x"], f["W_v"], B, T, G, dh)
    rows = [b * T + L for b in range(B)]
    return s, inp, f, K[:, :, :L], V[:, :, :L], rows


def test_decode_step_is_the_prefill_layer_at_the_last_position():
    # Decoding token L against the K/V cache of tokens 0..L-1 is the prefill
    # definition evaluated at position L (causality): GQE and dense GQA.
    s, inp, f, Kc, Vc, rows = _decode_case(seed=31)
    ref = oracle.gqe_layer(inp, rows=rows)
    d = oracle.gqe_decode_step(f["x"][rows], Kc, Vc, f["W_r"], f["b_r"], f["W_q"], f["W_qs"],
                               f["W_k"], f["W_v"], f["W_o"], s.G, s.M, s.k, s.d_head)
    np.testing.assert_array_equal(d["idx"], ref["idx"][rows])
    np.testing.assert_allclose(d["slots"], ref["slots"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(d["y"], ref["y"], rtol=0, atol=1e-13)
    dref = oracle.gqa_dense_layer(inp, rows=rows)
    dd = oracle.gqa_dense_decode_step(f["x"][rows], Kc, Vc, f["W_q"], f["W_k"], f["W_v"],
                                      f["W_o_dense"], s.G, s.M, s.d_head)
    np.testing.assert_allclose(dd["y"], dref["y"], rtol=0, atol=1e-13)


def test_decode_step_with_an_empty_cache_returns_the_new_values():
    # L = 0: the only key is the token's own, so every head's output is v_new
    # of its group (the shared head's of group 0), whatever the query.
    s, inp, f, Kc, Vc, rows = _decode_case(seed=32)
    x = f["x"][rows]
    d = oracle.gqe_decode_step(x, Kc[:, :, :0], Vc[:, :, :0], f["W_r"], f["W_r"][0] * 0, f["W_q"],
                               f["W_qs"], f["W_k"], f["W_v"], f["W_o"], s.G, s.M, s.k, s.d_head)
    dh, G, k = s.d_head, s.G, s.k
    v_new = (x @ f["W_v"]).reshape(len(rows), G, dh)
    for g in range(G):
        for si in range(k):
            np.testing.assert_allclose(d["slots"][:, (g * k + si) * dh:(g * k + si + 1) * dh],
                                       v_new[:, g], rtol=0, atol=1e-13)
    np.testing.assert_allclose(d["slots"][:, G * k * dh:(G * k + 1) * dh], v_new[:, 0], rtol=0,
                               atol=1e-13)


# --------------------------------------------------------------------------
# output constructions (the layer and the ablation variants)
# --------------------------------------------------------------------------

def _with_mode_wo(inp, mode):
    """The instance with W_o cut to the mode's slot rows (the first ones)."""
    import dataclasses
    s = inp.shape
    rows = oracle.mode_slots(mode, s.G, s.k) * s.d_head
    return dataclasses.replace(inp, W_o=inp.W_o[:rows].copy())


def test_hard_concat_with_k_equal_m_is_dense_gqa():
    # k = M selects every expert of every group in ascending order, so the hard
    # concatenation is the dense heads in head order; with W_O_dense = W_o it
    # is the dense GQA layer.
    s = LayerShape(B=2, T=9, d_model=32, G=2, M=3, k=3, d_head=8)
    inp = _with_mode_wo(synth.make_layer_inputs(s, seed=90), "hard")
    import dataclasses
    dense = oracle.gqa_dense_layer(dataclasses.replace(inp, W_o_dense=inp.W_o))
    hard = oracle.gqe_layer(inp, mode="hard")
    np.testing.assert_allclose(hard["slots"], dense["O"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(hard["y"], dense["y"], rtol=0, atol=1e-12)


def test_weighted_concat_uniform_router_scales_by_one_over_m():
    # W_r = 0, no bias: every in-group probability is 1/M, so each selected
    # output is scaled by 1/M; with k = M that is the dense layer over M.
    s = LayerShape(B=1, T=11, d_model=32, G=2, M=2, k=2, d_head=8)
    import dataclasses
    inp = _with_mode_wo(synth.make_layer_inputs(s, seed=91), "weighted_concat")
    inp = dataclasses.replace(inp, W_r=np.zeros_like(inp.W_r))
    dense = oracle.gqa_dense_layer(dataclasses.replace(inp, W_o_dense=inp.W_o))
    wc = oracle.gqe_layer(inp, mode="weighted_concat")
    np.testing.assert_allclose(wc["y"], dense["y"] / s.M, rtol=0, atol=1e-13)


def test_weighted_concat_hand_probabilities():
    # Bias ln 3 on expert 0 of each group, W_r = 0: p = (3/4, 1/4), expert 0 is
    # selected with weight 3/4 (k = 1).
    s = LayerShape(B=1, T=7, d_model=32, G=3, M=2, k=1, d_head=8)
    import dataclasses
    base = synth.make_layer_inputs(s, seed=92)
    b = np.zeros(s.N, dtype=np.float32)
    b[0::2] = np.float32(math.log(3.0))
    inp = dataclasses.replace(base, W_r=np.zeros_like(base.W_r), b_r=b)
    hard = oracle.gqe_layer(_with_mode_wo(inp, "hard"), mode="hard")
    wc = oracle.gqe_layer(_with_mode_wo(inp, "weighted_concat"), mode="weighted_concat")
    assert (wc["idx"] == 0).all()
    p0 = 3.0 / 4.0  # the fp32 bias ln 3 moves p by ~1e-8 only
    np.testing.assert_allclose(wc["slots"], p0 * hard["slots"], rtol=1e-7, atol=1e-12)


def test_group_mean_slot_with_k1_is_mean_of_routed_outputs():
    # k = 1: r = 1 for every selection, so the slot is the mean of the G routed
    # outputs whatever the router does.
    s = LayerShape(B=2, T=10, d_model=32, G=4, M=3, k=1, d_head=8)
    inp = synth.make_layer_inputs(s, seed=93)
    gm = oracle.gqe_layer(inp, mode="group_mean")
    dh, G = s.d_head, s.G
    routed = gm["slots"][:, :G * dh].reshape(-1, G, dh)
    np.testing.assert_allclose(gm["slots"][:, (G + 1) * dh:], routed.mean(axis=1), rtol=0, atol=1e-14)


def test_group_mean_slot_hand_weights_k2():
    # p proportional to (5, 3, 2, 1) in every group (bias ln of those, W_r = 0):
    # the top 2 are experts 0 and 1 with r = (5/8, 3/8).
    s = LayerShape(B=1, T=6, d_model=32, G=2, M=4, k=2, d_head=8)
    import dataclasses
    base = synth.make_layer_inputs(s, seed=94)
    b = np.tile(np.log(np.array([5.0, 3.0, 2.0, 1.0])), s.G).astype(np.float32)
    inp = dataclasses.replace(base, W_r=np.zeros_like(base.W_r), b_r=b)
    gm = oracle.gqe_layer(inp, mode="group_mean")
    assert (gm["idx"] == np.array([0, 1])).all()
    dh, G, k = s.d_head, s.G, s.k
    o = gm["slots"][:, :G * k * dh].reshape(-1, G, k, dh)
    want = (5 / 8 * o[:, :, 0] + 3 / 8 * o[:, :, 1]).mean(axis=1)
    np.testing.assert_allclose(gm["slots"][:, (G * k + 1) * dh:], want, rtol=1e-7, atol=1e-12)


def test_group_mean_equals_layer_slot_under_uniform_router():
    # With equal selected mass in every group (W_r = 0), omega = r / G, so the
    # layer's weighted slot and the group mean coincide; the other slots are
    # the same in both constructions.
    s = LayerShape(B=1, T=8, d_model=32, G=3, M=3, k=2, d_head=8)
    import dataclasses
    base = synth.make_layer_inputs(s, seed=95)
    inp = dataclasses.replace(base, W_r=np.zeros_like(base.W_r))
    a = oracle.gqe_layer(inp)
    b = oracle.gqe_layer(inp, mode="group_mean")
    np.testing.assert_allclose(a["slots"], b["slots"], rtol=0, atol=1e-14)
