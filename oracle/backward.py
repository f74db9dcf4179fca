"""fp64 backward of one GQE prefill layer (the layer's gradients; the survey's
next row f1).

TEST INFRASTRUCTURE, under the same rules as the rest of ``oracle``: only the
tests may call it, the CUDA library never does, and it shares no code with it.

Given the upstream gradient dy = dL/dy of the layer output, it returns dL/dx
and the gradients of every weight, with the router's top-k selection held
fixed: the selection is a discrete choice, and the pages name the weighted
slot as the differentiable path from the loss to the router (gist.science
Technical Summary, "Output Construction"; pptc.cn blog section 4.3). Each
forward step's chain rule is written out below on the plain definitions, in
fp64, with no tiling:

  a11  y = S W_O                      dS = dy W_O^T, dW_O = S^T dy
  a10  S = [o_r | o_s | sum w o_r]    do_r = dS_r + w dS_w, do_s = dS_s,
                                      dw = <o_r, dS_w>
  a4   w = p_sel / sum(p_sel)         (over the token's kG selected experts)
  a2   p = softmax of each group's M logits
  a1   z = x W_r + b                  dW_r = x^T dz, db = sum dz, dx += dz W_r^T
  a8   o = causal softmax(q K^T / sqrt(dh)) V, per stream
  a7   q[t, g, s] = x_t W_q[:, e]     e = g*M + idx[t, g, s];  q_s = x W_qs
  a6   K = x W_k, V = x W_v           (the routed slots of group g and, for
                                      g = 0, the shared head add into dK, dV)

Pinned by ``tests/test_oracle_backward.py``: central finite differences of the
forward below (selection fixed) against every gradient, on small layers.
The load-balancing auxiliary loss is not here: the pages say that one is used
but give no formula for it.
"""
from __future__ import annotations

import math

import numpy as np

from . import causal_attention, kv_proj, q_routed_rows, router_logits


def _group_softmax(z: np.ndarray, G: int, M: int) -> np.ndarray:
    zg = z.reshape(z.shape[0], G, M)
    e = np.exp(zg - zg.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def forward(x, W_r, b_r, W_q, W_qs, W_k, W_v, W_o, B: int, T: int, G: int, M: int, dh: int,
            idx: np.ndarray) -> dict:
    """The GQE layer's forward on fp64 arrays with the selection idx [R, G, k]
    given (the router's choice for these inputs); returns y and the
    intermediates the backward needs."""
    R = B * T
    k = idx.shape[2]
    z = router_logits(x, W_r, b_r)
    p = _group_softmax(z, G, M)
    psel = np.take_along_axis(p, idx.astype(np.int64), axis=-1)       # [R, G, k]
    w = psel / psel.sum(axis=(1, 2), keepdims=True)
    K = kv_proj(x, W_k, B, T, G, dh)                                 # [B, G, T, dh]
    V = kv_proj(x, W_v, B, T, G, dh)
    q = q_routed_rows(x, W_q, idx, G, M, dh)                         # [R, G, k, dh]
    qs = x @ W_qs                                                    # [R, dh]
    o = np.zeros((R, G, k, dh))
    o_s = np.zeros((R, dh))
    for b in range(B):
        rows = slice(b * T, (b + 1) * T)
        for g in range(G):
            for s in range(k):
                o[rows, g, s] = causal_attention(q[rows, g, s], K[b, g], V[b, g])
        o_s[rows] = causal_attention(qs[rows], K[b, 0], V[b, 0])
    weighted = np.einsum("rgs,rgsd->rd", w, o)
    S = np.concatenate([o.reshape(R, G * k * dh), o_s, weighted], axis=1)
    return {"y": S @ W_o, "S": S, "z": z, "p": p, "psel": psel, "w": w, "K": K, "V": V, "q": q,
            "qs": qs, "o": o, "o_s": o_s}


def causal_attention_backward(q: np.ndarray, K: np.ndarray, V: np.ndarray, do: np.ndarray):
    """Gradients of o = softmax_causal(q K^T / sqrt(dh)) V for one head over
    positions 0..n-1: with P the attention weights and dP = do V^T,
    dS = P * (dP - rowsum(dP * P)), dq = dS K / sqrt(dh), dK = dS^T q / sqrt(dh),
    dV = P^T do."""
    n, dh = q.shape
    scale = 1.0 / math.sqrt(dh)
    sc = (q @ K[:n].T) * scale
    sc[np.triu(np.ones((n, n), dtype=bool), 1)] = -np.inf
    P = np.exp(sc - sc.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    dP = do @ V[:n].T
    dS = P * (dP - (dP * P).sum(axis=1, keepdims=True))
    return (dS @ K[:n]) * scale, (dS.T @ q) * scale, P.T @ do


def backward(x, W_r, b_r, W_q, W_qs, W_k, W_v, W_o, B: int, T: int, G: int, M: int, dh: int,
             idx: np.ndarray, dy: np.ndarray) -> dict:
    """dL/d(everything) for L with dL/dy = dy, selection idx held fixed."""
    R = B * T
    k = idx.shape[2]
    f = forward(x, W_r, b_r, W_q, W_qs, W_k, W_v, W_o, B, T, G, M, dh, idx)
    # a11
    dS = dy @ W_o.T
    dW_o = f["S"].T @ dy
    nr = G * k * dh
    dS_r = dS[:, :nr].reshape(R, G, k, dh)
    dS_s = dS[:, nr:nr + dh]
    dS_w = dS[:, nr + dh:]
    # a10
    do = dS_r + f["w"][..., None] * dS_w[:, None, None, :]
    do_s = dS_s
    dw = np.einsum("rgsd,rd->rgs", f["o"], dS_w)
    # a4: w = psel / sum(psel)  ->  dpsel = (dw - sum(w dw)) / sum(psel)
    tot = f["psel"].sum(axis=(1, 2), keepdims=True)
    dpsel = (dw - (f["w"] * dw).sum(axis=(1, 2), keepdims=True)) / tot
    dp = np.zeros_like(f["p"])
    np.put_along_axis(dp, idx.astype(np.int64), dpsel, axis=-1)
    # a2: softmax of each group
    p = f["p"]
    dz = (p * (dp - (dp * p).sum(axis=-1, keepdims=True))).reshape(R, G * M)
    # a1
    dW_r = x.T @ dz
    db_r = dz.sum(axis=0)
    dx = dz @ W_r.T
    # a8: attention, stream by stream
    dq = np.zeros_like(f["q"])
    dqs = np.zeros_like(f["qs"])
    dK = np.zeros_like(f["K"])
    dV = np.zeros_like(f["V"])
    for b in range(B):
        rows = slice(b * T, (b + 1) * T)
        for g in range(G):
            for s in range(k):
                a, kk, vv = causal_attention_backward(f["q"][rows, g, s], f["K"][b, g], f["V"][b, g],
                                                      do[rows, g, s])
                dq[rows, g, s] = a
                dK[b, g] += kk
                dV[b, g] += vv
        a, kk, vv = causal_attention_backward(f["qs"][rows], f["K"][b, 0], f["V"][b, 0], do_s[rows])
        dqs[rows] = a
        dK[b, 0] += kk
        dV[b, 0] += vv
    # a7: routed and shared queries
    dW_q = np.zeros_like(W_q)
    for g in range(G):
        for j in range(M):
            e = g * M + j
            We = W_q[:, e * dh:(e + 1) * dh]
            for s in range(k):
                m = idx[:, g, s] == j
                if m.any():
                    dW_q[:, e * dh:(e + 1) * dh] += x[m].T @ dq[m, g, s]
                    dx[m] += dq[m, g, s] @ We.T
    dW_qs = x.T @ dqs
    dx += dqs @ W_qs.T
    # a6: K and V, back to [R, G*dh]
    dKf = dK.transpose(0, 2, 1, 3).reshape(R, G * dh)
    dVf = dV.transpose(0, 2, 1, 3).reshape(R, G * dh)
    dW_k = x.T @ dKf
    dW_v = x.T @ dVf
    dx += dKf @ W_k.T + dVf @ W_v.T
    return {"y": f["y"], "dx": dx, "dW_r": dW_r, "db_r": db_r, "dW_q": dW_q, "dW_qs": dW_qs,
            "dW_k": dW_k, "dW_v": dW_v, "dW_o": dW_o}
