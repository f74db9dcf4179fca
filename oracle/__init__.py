"""fp64 CPU oracle of one Grouped Query Experts (GQE) prefill layer (and of one
decode step against its dense K/V cache).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference arm of ``bench.py`` may import or call this package. The
CUDA library never calls it, and it shares no code with the CUDA library: the
two meet only in the seeded input generator ``synth`` (which draws numbers and
computes nothing of the layer).

What it computes is the plain definition of the layer, evaluated in fp64 on the
exact values of the bf16 / fp32 inputs, with no tiling, no online softmax and no
rounding to bf16 anywhere. Sources (all pages describe the same paper,
"Grouped Query Experts: Mixture-of-Experts on GQA Self-Attention",
arXiv:2606.20945):

* routed query-head experts inside each fixed GQA group, a per-token router
  choosing k experts per group, K/V projections dense and unchanged
  (gist.science summary, "Technical Summary / Methodology: Architecture and
  Routing"; chatpaper / hotpaper abstract);
* "softmax first, then top-k" inside each group; every group takes part
  (pptc.cn blog, section 7 Conclusion and section 5 Related Work);
* output construction: hard concatenation of the selected experts, one
  renormalised weighted-sum slot, one always-on shared head (gist.science
  summary, "Output Construction");
* W_O of size (kG+2) x d (hotpaper.ai summary, "Core idea" and "Technical
  approach").

Readings where the pages are silent, ambiguous or garbled:

* R1 the shared head attends to KV group 0; R2 it has its own W_qs [d, dh];
* R3 the weighted slot is sum_g sum_{j in S_g} w_gj * o_gj with
  w = p / (sum over all kG selected p) (one slot, renormalised over every
  selected expert of the token);
* R4 the router output r is renormalised per group: r = p / sum_{S_g} p;
* R5 ties go to the lower expert index; R6 routed slots are ordered by group,
  then by ascending expert index inside the group; R7 top-k is taken on the
  logits (equal to top-k on the in-group softmax, which is monotone);
* R8 scale 1/sqrt(dh), no positional encoding, no biases besides the router's;
* R9 W_O is [(kG+2)*dh, d]; R10 expert e = g*M + j; dense head h uses group
  h // M; R11 key u is visible to query t iff u <= t in the same sequence.

Parity is pinned by ``tests/test_oracle_pins.py`` (closed forms, brute force on
tiny inputs, library routines on special cases, the pages' invariants).
"""
from __future__ import annotations

import math

import numpy as np

from synth import LayerInputs, LayerShape, bf16_to_f64

_U64 = 2.0 ** -53  # unit roundoff of fp64


# --------------------------------------------------------------------------
# a1-a4: router
# --------------------------------------------------------------------------

def router_logits(x: np.ndarray, W_r: np.ndarray, b_r: np.ndarray | None) -> np.ndarray:
    """z[t, e] = sum_i x[t, i] * W_r[i, e] + b[e], in fp64.

    Each product of a bf16 value and an fp32 value has at most 8 + 24
    significant bits, so it is exact in fp64; only the summation rounds.
    (Router scores over all experts: gist.science summary, "Conditional
    activation".)
    """
    z = np.asarray(x, np.float64) @ np.asarray(W_r, np.float64)
    if b_r is not None:
        z = z + np.asarray(b_r, np.float64)[None, :]
    return z


def _exact_logit(xrow: np.ndarray, wcol: np.ndarray, b: float) -> float:
    # Products are exact in fp64; math.fsum returns the correctly rounded sum.
    return math.fsum(list(xrow * wcol) + [b])


def _exact_sign_of_difference(xrow: np.ndarray, wa: np.ndarray, wb: np.ndarray, ba: float,
                              bb: float) -> int:
    """Sign of z_a - z_b computed exactly.

    z_a - z_b = sum_i x_i W[i,a] - sum_i x_i W[i,b] + b_a - b_b. Every term is
    an exact fp64 value (bf16 x fp32 products), and math.fsum returns the
    correctly rounded value of their exact sum, which is zero exactly when the
    sum is zero and otherwise has its sign.
    """
    s = math.fsum(list(xrow * wa) + list(-(xrow * wb)) + [ba, -bb])
    return (s > 0) - (s < 0)


def _exact_topk(xrow: np.ndarray, W: np.ndarray, bvec: np.ndarray, g: int, M: int, k: int):
    """The k experts of group g with the largest exact logits, ties to the lower
    index, ascending: expert j precedes i when z_j > z_i exactly, or z_j = z_i
    and j < i."""
    import functools

    def before(j, i):
        s = _exact_sign_of_difference(xrow, W[:, g * M + j], W[:, g * M + i], bvec[g * M + j],
                                      bvec[g * M + i])
        return -1 if s > 0 or (s == 0 and j < i) else 1

    order = sorted(range(M), key=functools.cmp_to_key(before))
    return sorted(order[:k])


def router(x: np.ndarray, W_r: np.ndarray, b_r: np.ndarray | None, G: int, M: int, k: int):
    """Per-group softmax, top-k per group, renormalised weights.

    Returns a dict with
      z     [R, N]    fp64 logits,
      p     [R, G, M] in-group softmax probabilities,
      idx   [R, G, k] int32 selected expert-local indices j, ascending,
      r     [R, G, k] p renormalised inside the group (reading R4),
      omega [R, G, k] p renormalised over all kG selected experts (reading R3).

    The selection is the one exact arithmetic gives: where the fp64 logits of
    a group are closer at the top-k boundary than a certified bound on their
    rounding error, that group's order is decided on the exact logits (the
    exact sign of each difference, ``_exact_topk``) and its logits are
    recomputed correctly rounded (math.fsum of exact products) for the
    softmax.
    """
    if not (1 <= k <= M):
        raise ValueError("need 1 <= k <= M")
    x = np.asarray(x, np.float64)
    W_r = np.asarray(W_r, np.float64)
    R, d = x.shape
    N = G * M
    assert W_r.shape == (d, N)
    bvec = np.zeros(N) if b_r is None else np.asarray(b_r, np.float64)
    z = router_logits(x, W_r, b_r)

    # Certified fp64 error bound of each logit: gamma_{d+1} * (sum |x w| + |b|).
    gam = (d + 1) * _U64 / (1.0 - (d + 1) * _U64)
    bound = gam * (np.abs(x) @ np.abs(W_r) + np.abs(bvec)[None, :]) * 2.0

    zg = z.reshape(R, G, M)
    exact_sel = {}
    if k < M:
        srt = -np.sort(-zg, axis=-1)
        margin = srt[..., k - 1] - srt[..., k]
        bg = bound.reshape(R, G, M).max(axis=-1)
        for t, g in zip(*np.nonzero(margin <= 2.0 * bg)):
            for j in range(M):
                e = g * M + j
                zg[t, g, j] = _exact_logit(x[t], W_r[:, e], bvec[e])
            exact_sel[(int(t), int(g))] = _exact_topk(x[t], W_r, bvec, int(g), M, k)
        z = zg.reshape(R, N)

    # a2: softmax over the M logits of each group (softmax before top-k).
    zmax = zg.max(axis=-1, keepdims=True)
    ez = np.exp(zg - zmax)
    p = ez / ez.sum(axis=-1, keepdims=True)

    # a3: top-k on the logits; a stable sort of -z keeps equal logits in index
    # order, so ties go to the lower j. Selected indices stored ascending.
    # Groups without a certified fp64 margin take their exact selection.
    order = np.argsort(-zg, axis=-1, kind="stable")[..., :k]
    idx = np.sort(order, axis=-1).astype(np.int32)
    for (t, g), sel in exact_sel.items():
        idx[t, g] = sel

    # a4: renormalised weights.
    psel = np.take_along_axis(p, idx.astype(np.int64), axis=-1)
    r = psel / psel.sum(axis=-1, keepdims=True)
    omega = psel / psel.sum(axis=(1, 2), keepdims=True)
    return {"z": z, "p": p, "idx": idx, "r": r, "omega": omega}


# --------------------------------------------------------------------------
# a5: dispatch (token lists per expert)
# --------------------------------------------------------------------------

def dispatch(idx: np.ndarray, B: int, T: int, G: int, M: int):
    """Token lists per (expert, batch element).

    counts[e, b]   number of tokens of sequence b that selected expert e;
    offsets[e*B+b] exclusive prefix sum of counts in (e, b) order, with
                   offsets[N*B] the total (= k*G*B*T);
    tok[...]       for each (e, b), the positions t (0..T-1) that selected e,
                   ascending;
    slot_pos[row, g, s] the index in ``tok`` of the entry for that selection.

    For each (e, b): the positions whose selections in group g contain j
    (e = g*M + j), in increasing order; a selection's entry is the list's
    base plus the number of earlier positions in the same list.
    """
    R, G_, k = idx.shape
    assert G_ == G and R == B * T
    N = G * M
    counts = np.zeros((N, B), dtype=np.int64)
    hits = {}
    for e in range(N):
        g, j = divmod(e, M)
        for b in range(B):
            sel = idx[b * T:(b + 1) * T, g, :] == j      # [T, k]: which slot took j
            hits[(e, b)] = sel
            counts[e, b] = int(sel.sum())
    offsets = np.zeros(N * B + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts.reshape(-1))
    tok = np.zeros(int(offsets[-1]), dtype=np.int32)
    slot_pos = np.full((R, G, k), -1, dtype=np.int64)
    for e in range(N):
        g, j = divmod(e, M)
        for b in range(B):
            sel = hits[(e, b)]
            base = int(offsets[e * B + b])
            t_list = np.nonzero(sel.any(axis=1))[0]       # ascending positions
            tok[base:base + t_list.size] = t_list
            t_s, s_s = np.nonzero(sel)                    # (position, slot) of each hit
            rank = np.searchsorted(t_list, t_s)           # earlier entries of the list
            slot_pos[b * T + t_s, g, s_s] = base + rank
    assert (slot_pos >= 0).all()
    return {"counts": counts.astype(np.int32), "offsets": offsets.astype(np.int32),
            "tok": tok, "slot_pos": slot_pos.astype(np.int32)}


# --------------------------------------------------------------------------
# a6-a7: projections
# --------------------------------------------------------------------------

def kv_proj(x: np.ndarray, W: np.ndarray, B: int, T: int, G: int, dh: int) -> np.ndarray:
    """Dense K (or V) of every group: out[b, g, t, :] = x[b*T+t] @ W[:, g*dh:(g+1)*dh].

    The K/V path is the GQA one, dense and unchanged (gist.science summary,
    "Dense KV path"; pptc.cn blog, section 5).
    """
    y = np.asarray(x, np.float64) @ np.asarray(W, np.float64)  # [R, G*dh]
    return y.reshape(B, T, G, dh).transpose(0, 2, 1, 3).copy()


def q_routed_rows(x_rows: np.ndarray, W_q: np.ndarray, idx_rows: np.ndarray, G: int, M: int,
                  dh: int) -> np.ndarray:
    """Query of every selected expert of the given token rows: q[n, g, s, :].

    Row n's selection (g, s) is expert e = g*M + idx_rows[n, g, s], and its
    query is x_rows[n] @ W_q[:, e*dh:(e+1)*dh]; no other expert computes a
    query for the row (conditional query computation: chatpaper / hotpaper
    abstract).
    """
    x_rows = np.asarray(x_rows, np.float64)
    W_q = np.asarray(W_q, np.float64)
    n, _, k = idx_rows.shape
    q = np.zeros((n, G, k, dh))
    for g in range(G):
        for j in range(M):
            e = g * M + j
            We = W_q[:, e * dh:(e + 1) * dh]
            for s in range(k):
                m = idx_rows[:, g, s] == j
                if m.any():
                    q[m, g, s] = x_rows[m] @ We
    return q


def q_routed(x: np.ndarray, W_q: np.ndarray, idx: np.ndarray, B: int, T: int, G: int,
             M: int, dh: int) -> np.ndarray:
    """The routed queries of every row, slot-major: Qv[b, g, s, t, :]
    (``q_routed_rows`` of all rows, laid out by stream)."""
    k = idx.shape[2]
    q = q_routed_rows(x, W_q, idx, G, M, dh)             # [B*T, G, k, dh]
    return q.reshape(B, T, G, k, dh).transpose(0, 2, 3, 1, 4).copy()


def q_shared(x: np.ndarray, W_qs: np.ndarray, B: int, T: int, dh: int) -> np.ndarray:
    """Always-on shared head query for every token: Qs[b, t, :] (readings R1, R2)."""
    return (np.asarray(x, np.float64) @ np.asarray(W_qs, np.float64)).reshape(B, T, dh)


# --------------------------------------------------------------------------
# a8-a9: causal attention
# --------------------------------------------------------------------------

def causal_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, rows=None,
                     block: int | None = None) -> np.ndarray:
    """o[t] = sum_{u <= t} softmax_u(q[t] . K[u] / sqrt(dh)) V[u] for one head.

    ``q`` holds the queries of the rows ``rows`` (positions in the sequence;
    all positions 0..len(q)-1 when None). Each row is evaluated on its own
    from the definition; ``block`` only groups rows to bound memory (by
    default as many rows as keep one score block near 128 MB).
    """
    q = np.asarray(q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    n, dh = q.shape
    pos = np.arange(n) if rows is None else np.asarray(rows, np.int64)
    scale = 1.0 / math.sqrt(dh)
    out = np.empty((n, V.shape[1]))
    if block is None:
        block = max(1, min(512, (1 << 24) // max(1, int(pos.max(initial=0)) + 1)))
    for s in range(0, n, block):
        ps = pos[s:s + block]
        hi = int(ps.max()) + 1
        sc = (q[s:s + block] @ K[:hi].T) * scale          # [rows, hi]
        mask = np.arange(hi)[None, :] > ps[:, None]
        sc[mask] = -np.inf
        sc -= sc.max(axis=1, keepdims=True)
        w = np.exp(sc)
        w /= w.sum(axis=1, keepdims=True)
        out[s:s + block] = w @ V[:hi]
    return out


# --------------------------------------------------------------------------
# a10-a11: slots and W_O
# --------------------------------------------------------------------------

# Output constructions. "gqe" is the layer (reading R3); the others are the
# ablation variants of the pptc.cn blog's section 4.3 and Table 1 (reading R15:
# that page's labels), and "group_mean" is the alternative weighted slot:
#   gqe              [o_{g,s}] + [o_shared] + [sum_{g,s} omega_{g,s} o_{g,s}]
#   group_mean       [o_{g,s}] + [o_shared] + [(1/G) sum_g sum_s r_{g,s} o_{g,s}]
#                    (each group's selected outputs renormalised inside the
#                    group, then the groups averaged)
#   hard             [o_{g,s}] only: hard concatenation of the selected experts,
#                    with neither the router-supervision slot nor the shared head
#                    ("仅硬拼接")
#   weighted_concat  [p_{g,s} o_{g,s}]: each selected output scaled by its
#                    in-group softmax probability, with neither the supervision
#                    slot nor the shared head ("加权拼接但无重归一化槽"; the page
#                    says the weights are possibly the in-group softmax
#                    probabilities, and that is the reading taken)
OUTPUT_MODES = ("gqe", "group_mean", "hard", "weighted_concat")


def mode_slots(mode: str, G: int, k: int) -> int:
    """Slots per token (W_O has this many d_head-row blocks)."""
    return k * G + 2 if mode in ("gqe", "group_mean") else k * G


def mode_has_shared_head(mode: str) -> bool:
    return mode in ("gqe", "group_mean")


def assemble_slots(o_routed: np.ndarray, o_shared: np.ndarray | None, rt_rows: dict,
                   mode: str = "gqe") -> np.ndarray:
    """Slots per token for an output construction (see OUTPUT_MODES).

    o_routed [R, G, k, dh]; o_shared [R, dh] (None for the modes without the
    shared head); rt_rows holds the router's omega, r, p and idx of the same
    rows -> [R, mode_slots * dh].
    """
    R, G, k, dh = o_routed.shape
    concat = o_routed.reshape(R, G * k * dh)
    if mode == "gqe":
        weighted = np.einsum("rgs,rgsd->rd", rt_rows["omega"], o_routed)
        return np.concatenate([concat, o_shared, weighted], axis=1)
    if mode == "group_mean":
        weighted = np.einsum("rgs,rgsd->rd", rt_rows["r"], o_routed) / G
        return np.concatenate([concat, o_shared, weighted], axis=1)
    if mode == "hard":
        return concat.copy()
    if mode == "weighted_concat":
        psel = np.take_along_axis(rt_rows["p"], rt_rows["idx"].astype(np.int64), axis=-1)
        return (psel[..., None] * o_routed).reshape(R, G * k * dh)
    raise ValueError(f"unknown output mode {mode!r}")


def output_proj(slots: np.ndarray, W_o: np.ndarray) -> np.ndarray:
    """y = slots @ W_O with W_O of shape [slots*dh, d]: [(kG+2)*dh, d] for the
    layer (reading R9)."""
    return np.asarray(slots, np.float64) @ np.asarray(W_o, np.float64)


# --------------------------------------------------------------------------
# whole layers
# --------------------------------------------------------------------------

def _f64_weights(inp: LayerInputs) -> dict:
    """Exact fp64 values of every weight (x is widened row block by row block
    where it is used)."""
    return {
        "W_r": inp.W_r.astype(np.float64),
        "b_r": None if inp.b_r is None else inp.b_r.astype(np.float64),
        "W_q": bf16_to_f64(inp.W_q),
        "W_qs": bf16_to_f64(inp.W_qs),
        "W_k": bf16_to_f64(inp.W_k),
        "W_v": bf16_to_f64(inp.W_v),
        "W_o": bf16_to_f64(inp.W_o),
        "W_o_dense": bf16_to_f64(inp.W_o_dense),
    }


def _f64_inputs(inp: LayerInputs) -> dict:
    f = _f64_weights(inp)
    f["x"] = bf16_to_f64(inp.x)
    return f


# Rows of x widened to fp64 at a time. Every output row of the router and of
# the projections depends on its own x row only, so taking the rows block by
# block changes no arithmetic; it only bounds host memory on long sequences.
_ROW_BLOCK = 16384


def _router_by_rows(inp: LayerInputs, f: dict) -> dict:
    s = inp.shape
    parts = [router(bf16_to_f64(inp.x[lo:lo + _ROW_BLOCK]), f["W_r"], f["b_r"], s.G, s.M, s.k)
             for lo in range(0, s.R, _ROW_BLOCK)]
    return {key: np.concatenate([p_[key] for p_ in parts]) for key in parts[0]}


def _kv_group_prefix(inp: LayerInputs, W_k: np.ndarray, W_v: np.ndarray, b: int, g: int,
                     hi: int):
    """K and V of group g for positions 0..hi-1 of sequence b:
    x[b*T + u] @ W[:, g*dh:(g+1)*dh], as in kv_proj."""
    s = inp.shape
    dh = s.d_head
    Wg = np.concatenate([W_k[:, g * dh:(g + 1) * dh], W_v[:, g * dh:(g + 1) * dh]], axis=1)
    out = np.empty((hi, 2 * dh))
    for lo in range(0, hi, _ROW_BLOCK):
        up = min(hi, lo + _ROW_BLOCK)
        out[lo:up] = bf16_to_f64(inp.x[b * s.T + lo:b * s.T + up]) @ Wg
    return out[:, :dh], out[:, dh:]


def gqe_layer(inp: LayerInputs, rows=None, with_dispatch: bool = True,
              full_kv: bool = True, mode: str = "gqe") -> dict:
    """GQE prefill forward (a1-a11).

    ``mode`` selects the output construction (OUTPUT_MODES; "gqe" is the
    layer); inp.W_o must then have mode_slots(mode, G, k) * d_head rows.

    ``rows`` (optional) is a list of global row indices b*T+t at which the
    queries, attention, slots and y are evaluated; the router and dispatch
    are always computed in full. Without ``rows`` every output is computed in
    full. ``full_kv`` returns K and V for every row ([B, G, T, dh]);
    otherwise only at the evaluated rows (``K_rows``, ``V_rows`` [n, G, dh]),
    and each group's K/V is built only as far as the evaluated rows of a
    sequence reach (long sequences).
    """
    s: LayerShape = inp.shape
    B, T, G, M, k, dh = s.B, s.T, s.G, s.M, s.k, s.d_head
    f = _f64_weights(inp)
    rt = _router_by_rows(inp, f)
    out = dict(rt)
    if with_dispatch:
        out.update(dispatch(rt["idx"], B, T, G, M))
    idx = rt["idx"]
    R = B * T
    sel_rows = np.arange(R) if rows is None else np.asarray(rows, np.int64)
    if full_kv:
        x_all = bf16_to_f64(inp.x)
        K = kv_proj(x_all, f["W_k"], B, T, G, dh)
        V = kv_proj(x_all, f["W_v"], B, T, G, dh)
        out["K"], out["V"] = K, V

    # Queries of the evaluated rows (a7): routed experts and the shared head.
    x_sel = bf16_to_f64(inp.x[sel_rows])
    q_r = q_routed_rows(x_sel, f["W_q"], idx[sel_rows], G, M, dh)
    q_s = q_shared(x_sel, f["W_qs"], 1, sel_rows.size, dh)[0]
    if rows is None:
        out["Qv"] = q_r.reshape(B, T, G, k, dh).transpose(0, 2, 3, 1, 4).copy()
        out["Qs"] = q_s.reshape(B, T, dh)

    # a8-a9: causal attention of each evaluated row against its group's K/V.
    n = sel_rows.size
    o_r = np.zeros((n, G, k, dh))
    o_s = np.zeros((n, dh))
    if not full_kv:
        out["K_rows"] = np.zeros((n, G, dh))
        out["V_rows"] = np.zeros((n, G, dh))
    def attend(b, g):
        # Every evaluated row of sequence b, for every head on group g.
        m = (sel_rows // T) == b
        pos = sel_rows[m] % T
        if full_kv:
            Kg, Vg = K[b, g], V[b, g]
        else:
            Kg, Vg = _kv_group_prefix(inp, f["W_k"], f["W_v"], b, g, int(pos.max()) + 1)
            out["K_rows"][m, g] = Kg[pos]
            out["V_rows"][m, g] = Vg[pos]
        for si in range(k):
            o_r[m, g, si] = causal_attention(q_r[m, g, si], Kg, Vg, rows=pos)
        if g == 0:  # the shared head attends to KV group 0 (reading R1)
            o_s[m] = causal_attention(q_s[m], Kg, Vg, rows=pos)

    work = [(b, g) for b in range(B) if ((sel_rows // T) == b).any() for g in range(G)]
    if full_kv:
        for b, g in work:
            attend(b, g)
    else:
        # Groups are independent: several at a time (numpy's kernels release
        # the GIL); each writes only its own outputs.
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=4) as ex:
            list(ex.map(lambda bg: attend(*bg), work))
    rt_rows = {key: rt[key][sel_rows] for key in ("omega", "r", "p", "idx")}
    slots = assemble_slots(o_r, o_s if mode_has_shared_head(mode) else None, rt_rows, mode)
    assert f["W_o"].shape[0] == slots.shape[1], "W_o rows do not match the output mode"
    out["slots"] = slots
    out["y"] = output_proj(slots, f["W_o"])
    out["rows"] = sel_rows
    return out


def gqa_dense_layer(inp: LayerInputs, rows=None) -> dict:
    """Dense GQA layer with every one of the N = G*M query heads active.

    Head h uses KV group h // M; its output fills slot h of [R, N*dh], and
    y = O @ W_O_dense with W_O_dense [N*dh, d]. This is the all-active
    baseline the speed-up is measured against (gist.science summary,
    "Experimental Results"; pptc.cn blog Table 1 first row).
    """
    s: LayerShape = inp.shape
    B, T, G, M, dh = s.B, s.T, s.G, s.M, s.d_head
    N = G * M
    f = _f64_inputs(inp)
    K = kv_proj(f["x"], f["W_k"], B, T, G, dh)
    V = kv_proj(f["x"], f["W_v"], B, T, G, dh)
    R = B * T
    sel_rows = np.arange(R) if rows is None else np.asarray(rows, np.int64)
    x_sel = f["x"][sel_rows]
    n = sel_rows.size
    O = np.zeros((n, N, dh))
    Q = x_sel @ f["W_q"]  # [n, N*dh]
    for b in range(B):
        m = (sel_rows // T) == b
        if not m.any():
            continue
        pos = sel_rows[m] % T
        for h in range(N):
            O[m, h] = causal_attention(Q[m][:, h * dh:(h + 1) * dh], K[b, h // M], V[b, h // M],
                                       rows=pos)
    O = O.reshape(n, N * dh)
    out = {"K": K, "V": V, "O": O, "y": O @ f["W_o_dense"], "rows": sel_rows}
    if rows is None:
        out["Q"] = Q.reshape(B, T, N, dh).transpose(0, 2, 1, 3).copy()
    return out


def active_query_heads(shape: LayerShape) -> int:
    """Query heads that run attention per token: k per group plus the shared head."""
    return shape.k * shape.G + 1


# ---------------------------------------------------------------- decode step
def _decode_attention(q: np.ndarray, K_cache: np.ndarray, V_cache: np.ndarray,
                      k_new: np.ndarray, v_new: np.ndarray) -> np.ndarray:
    """Attention of one new query against its cache plus its own key: the
    causal definition at position L = len(cache), all L+1 keys visible."""
    K = np.concatenate([K_cache, k_new[None, :]], axis=0)
    V = np.concatenate([V_cache, v_new[None, :]], axis=0)
    L = K_cache.shape[0]
    return causal_attention(q[None, :], K, V, rows=[L])[0]


def gqe_decode_step(x_new: np.ndarray, K_cache: np.ndarray, V_cache: np.ndarray, W_r, b_r,
                    W_q, W_qs, W_k, W_v, W_o, G: int, M: int, k: int, dh: int) -> dict:
    """One GQE decode step (the survey's next row f2): each sequence b appends
    token x_new[b] at position L to its dense, unchanged K/V cache [B, G, L, dh]
    ("the Key-Value projections and the KV cache stay dense and unchanged":
    gist.science Technical Summary, Dense KV path) and the layer's output for
    that token is the prefill definition (a1-a11) at position L: router on the
    new token, only its selected experts' queries plus the shared head attend
    to the cache and the new key, the (kG+2) slots, W_O.

    All inputs are fp64 values of the bf16 / fp32 bits; returns idx, r, omega,
    k_new, v_new [B, G, dh], slots and y.
    """
    B = x_new.shape[0]
    rt = router(x_new, W_r, b_r, G, M, k)
    idx = rt["idx"]
    k_new = (x_new @ W_k).reshape(B, G, dh)
    v_new = (x_new @ W_v).reshape(B, G, dh)
    o_r = np.zeros((B, G, k, dh))
    for b in range(B):
        for g in range(G):
            for s in range(k):
                e = g * M + int(idx[b, g, s])
                q = x_new[b] @ W_q[:, e * dh:(e + 1) * dh]
                o_r[b, g, s] = _decode_attention(q, K_cache[b, g], V_cache[b, g], k_new[b, g],
                                                 v_new[b, g])
    q_s = x_new @ W_qs
    o_s = np.stack([_decode_attention(q_s[b], K_cache[b, 0], V_cache[b, 0], k_new[b, 0], v_new[b, 0])
                    for b in range(B)])
    slots = assemble_slots(o_r, o_s, rt)
    out = dict(rt)
    out.update(k_new=k_new, v_new=v_new, slots=slots, y=output_proj(slots, W_o))
    return out


def gqa_dense_decode_step(x_new: np.ndarray, K_cache: np.ndarray, V_cache: np.ndarray, W_q, W_k,
                          W_v, W_o_dense, G: int, M: int, dh: int) -> dict:
    """Dense GQA decode step: all N = G*M heads, head h on group h // M."""
    B = x_new.shape[0]
    N = G * M
    k_new = (x_new @ W_k).reshape(B, G, dh)
    v_new = (x_new @ W_v).reshape(B, G, dh)
    Q = x_new @ W_q
    O = np.zeros((B, N, dh))
    for b in range(B):
        for h in range(N):
            g = h // M
            O[b, h] = _decode_attention(Q[b, h * dh:(h + 1) * dh], K_cache[b, g], V_cache[b, g],
                                        k_new[b, g], v_new[b, g])
    O = O.reshape(B, N * dh)
    return {"k_new": k_new, "v_new": v_new, "O": O, "y": O @ W_o_dense}
