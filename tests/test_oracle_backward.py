"""Pins of the backward oracle (oracle.backward): every gradient against
central finite differences of the forward, with the router's selection held
fixed, on small fp64 layers. L = sum(dy * y), so dL/dtheta is what the
backward returns for upstream gradient dy."""
import numpy as np
import pytest

import oracle
from oracle import backward as bw


def _layer(seed, B, T, d, G, M, k, dh, bias=True):
    rng = np.random.default_rng(seed)
    N = G * M
    a = {
        "x": rng.standard_normal((B * T, d)),
        "W_r": rng.standard_normal((d, N)) / np.sqrt(d),
        "b_r": rng.standard_normal(N) * 0.1 if bias else None,
        "W_q": rng.standard_normal((d, N * dh)) / np.sqrt(d),
        "W_qs": rng.standard_normal((d, dh)) / np.sqrt(d),
        "W_k": rng.standard_normal((d, G * dh)) / np.sqrt(d),
        "W_v": rng.standard_normal((d, G * dh)) / np.sqrt(d),
        "W_o": rng.standard_normal(((k * G + 2) * dh, d)) / np.sqrt(d),
    }
    idx = oracle.router(a["x"], a["W_r"], a["b_r"], G, M, k)["idx"]
    dy = rng.standard_normal((B * T, d))
    return a, idx, dy


NAMES = ("x", "W_r", "b_r", "W_q", "W_qs", "W_k", "W_v", "W_o")


@pytest.mark.parametrize("case", [
    dict(B=1, T=7, d=12, G=2, M=3, k=2, dh=4),
    dict(B=2, T=5, d=8, G=3, M=2, k=1, dh=4, bias=False),
    dict(B=1, T=6, d=8, G=2, M=2, k=2, dh=4),  # k = M: every expert selected
])
def test_gradients_match_finite_differences(case):
    shape = {kk: case[kk] for kk in ("B", "T", "G", "M", "dh")}
    a, idx, dy = _layer(11, case["B"], case["T"], case["d"], case["G"], case["M"], case["k"], case["dh"],
                        case.get("bias", True))
    grads = bw.backward(*(a[n] for n in NAMES), idx=idx, dy=dy, **shape)

    def loss(arrs):
        y = bw.forward(*(arrs[n] for n in NAMES), idx=idx, **shape)["y"]
        return float((dy * y).sum())

    rng = np.random.default_rng(5)
    eps = 1e-6
    for n in NAMES:
        if a[n] is None:
            continue
        g = grads["d" + n]
        flat = a[n].reshape(-1)
        picks = rng.choice(flat.size, size=min(flat.size, 24), replace=False)
        for i in picks:
            up = {m: (v.copy() if v is not None else None) for m, v in a.items()}
            dn = {m: (v.copy() if v is not None else None) for m, v in a.items()}
            up[n].reshape(-1)[i] += eps
            dn[n].reshape(-1)[i] -= eps
            fd = (loss(up) - loss(dn)) / (2 * eps)
            an = g.reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), f"d{n}[{i}]: fd {fd:.9g} analytic {an:.9g}"


def test_forward_with_the_routers_selection_is_the_layer():
    """The backward's own forward, given the router's selection, is the
    oracle layer (the same y)."""
    from synth import LayerShape
    import synth
    shape = LayerShape(B=1, T=9, d_model=64, G=2, M=3, k=2, d_head=8)
    inp = synth.make_layer_inputs(shape, seed=3)
    f = oracle._f64_inputs(inp)
    ref = oracle.gqe_layer(inp)
    y = bw.forward(f["x"], f["W_r"], f["b_r"], f["W_q"], f["W_qs"], f["W_k"], f["W_v"], f["W_o"],
                   B=1, T=9, G=2, M=3, dh=8, idx=ref["idx"])["y"]
    np.testing.assert_allclose(y, ref["y"], rtol=0, atol=1e-12)


def test_attention_backward_single_key():
    """With one position the softmax is 1: dV = do, dq = dK = 0."""
    rng = np.random.default_rng(2)
    q, K, V, do = (rng.standard_normal((1, 4)) for _ in range(4))
    dq, dK, dV = bw.causal_attention_backward(q, K, V, do)
    np.testing.assert_allclose(dV, do, atol=1e-15)
    np.testing.assert_allclose(dq, 0.0, atol=1e-15)
    np.testing.assert_allclose(dK, 0.0, atol=1e-15)
