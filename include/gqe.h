/*
 * gqe.h - C ABI of libgqe.so: the prefill forward of one Grouped Query
 * Experts (GQE) self-attention layer on an NVIDIA B200 (sm_100a), plus the
 * dense GQA layer it is compared against.
 *
 * The method ("Grouped Query Experts: Mixture-of-Experts on GQA
 * Self-Attention", arXiv:2606.20945, as summarised by the gist.science
 * "Technical Summary", the pptc.cn blog and the hotpaper.ai summary):
 * the N = G*M query heads of a GQA layer are split into G fixed groups of M
 * "experts" (the heads sharing one KV head). Per token, a router takes a
 * softmax over each group's M logits and keeps the top k experts of every
 * group; only those experts, plus one always-on shared head, compute a query
 * and run causal attention against their group's dense, unchanged K/V. The
 * outputs fill kG+2 slots (kG routed, the shared head, one renormalised
 * weighted sum of the routed outputs) that feed W_O of size (kG+2) x d.
 *
 * Conventions for every call
 *  - All tensor pointers are DEVICE pointers, allocated and owned by the
 *    caller, 16-byte aligned, densely packed row-major in the layout given.
 *    The library never allocates device memory; scratch comes from the
 *    caller's workspace (size from gqe_workspace_bytes).
 *  - gqe_bf16 is a bf16 bit pattern; float is IEEE fp32.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream). Host-side validation errors return at once and launch
 *    nothing. Device-side failures (a bounded wait that ran out) are recorded
 *    in a per-device status word read by gqe_read_status.
 *  - Inputs are never written, except `slots` in gqe_output_proj (the
 *    weighted slot is filled in place).
 *  - Index conventions: row = b*T + t; expert e = g*M + j (j = 0..M-1 inside
 *    group g); routed slot (g, s) holds the s-th selected expert of group g
 *    in ascending j; the shared head attends to KV group 0; ties in the
 *    top-k go to the lower j. Dense head h uses KV group h / M.
 */
#ifndef GQE_H_
#define GQE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t gqe_bf16;   /* bf16 bit pattern */
typedef void* gqe_stream_t;  /* cudaStream_t */

typedef struct gqe_config {
  int32_t B;       /* sequences (batch) */
  int32_t T;       /* tokens per sequence (prefill length), >= 1 */
  int32_t d_model; /* model width, a multiple of 64 */
  int32_t G;       /* KV groups = KV heads */
  int32_t M;       /* query-head experts per group; N = G*M <= 64 */
  int32_t k;       /* experts selected per group per token, 1 <= k <= M */
  int32_t d_head;  /* head dim: 32 or 64 */
  uint32_t flags;  /* GQE_FLAG_* bits below; other bits must be 0 */
} gqe_config;

/* gqe_attention_fwd, gqe_layer_fwd, gqa_dense_fwd: the caller promises that
 * the workspace holds zeroed split-KV arrival counters -- it was zero-filled
 * before its first use and every earlier call on it completed with GQE_OK and
 * a zero device status (each call leaves the counters zero) -- so the call
 * does not clear them itself. Other entry points ignore the flag. */
#define GQE_FLAG_WS_CLEAN 1u

/* Expert-major routed queries: gqe_dispatch writes Qv in token-list order
 * ([k*G*B*T, d_head], row r = entry r of tok, i.e. (expert, sequence) lists
 * one after another, positions ascending) instead of slot-major; the layer
 * (gqe_layer_fwd) then runs gqe_attention_fwd_compact. Results are the same;
 * only the layout of Qv and the attention's tiling differ. */
#define GQE_FLAG_EXPERT_MAJOR 2u

/* Output construction (at most one of the three; none = the GQE layer). The
 * layer builds S slots per token from its routed outputs o[g, s]:
 *   default      S = kG+2: o[g, s] (hard concatenation), the shared head,
 *                and the weighted slot sum_{g,s} omega[g, s] o[g, s] with
 *                omega = p / (selected p of all groups);
 *   GROUP_MEAN   S = kG+2, as the default but omega = r / G: each group's
 *                selected outputs renormalised inside the group, the groups
 *                averaged (the other reading of the weighted slot);
 *   OUT_HARD     S = kG: the routed outputs only -- no weighted slot, no
 *                shared head ("hard concatenation only": pptc.cn blog, section
 *                4.3 and Table 1);
 *   OUT_WEIGHTED_CONCAT
 *                S = kG: p[g, s] * o[g, s] with p the in-group softmax
 *                probability -- no weighted slot, no shared head ("weighted
 *                concatenation without the renormalised slot": same section).
 * The flag changes what gqe_router_topk writes to omega (the weights the
 * output uses), the slot buffer ([B*T, S*d_head]), W_o ([S*d_head, d_model])
 * and, for the last two, drops the shared head (Qs may be NULL). The decode
 * step supports the default construction only. */
#define GQE_FLAG_SLOT_GROUP_MEAN 4u
#define GQE_FLAG_OUT_HARD 8u
#define GQE_FLAG_OUT_WEIGHTED_CONCAT 16u

/* A shard of the layer split over KV groups: the same construction without
 * the shared head, S = kG+1 (routed slots, then the weighted slot); combines
 * with the default or GROUP_MEAN. Each rank of a split runs its groups (G =
 * its group count, W_q/W_k/W_v columns and W_o rows of those groups) on the
 * routing of the whole layer; the rank holding group 0 keeps the shared head
 * (no flag), the others set this one, and the partial y of the ranks sum to
 * the layer's y (the weighted slot enters W_O linearly). */
#define GQE_FLAG_NO_SHARED_HEAD 32u

typedef enum gqe_status {
  GQE_OK = 0,
  GQE_ERR_INVALID = 1,      /* bad shape, k > M, null or misaligned pointer */
  GQE_ERR_UNSUPPORTED = 2,  /* valid but not built (e.g. d_head not 32/64) */
  GQE_ERR_WORKSPACE = 3,    /* workspace smaller than gqe_workspace_bytes */
  GQE_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed */
  GQE_ERR_TIMEOUT = 5,      /* a device-side bounded wait ran out */
  GQE_ERR_DEVICE_CHECK = 6  /* a device-side consistency check failed */
} gqe_status;

/* Workspace kinds for gqe_workspace_bytes / gqe_workspace_offset. */
enum {
  GQE_WS_DISPATCH = 1, /* scratch of gqe_dispatch */
  GQE_WS_LAYER = 2,    /* everything gqe_layer_fwd keeps between its steps */
  GQE_WS_DENSE = 3,    /* everything gqa_dense_fwd keeps between its steps */
  GQE_WS_ATTENTION = 4, /* scratch of gqe_attention_fwd (split-KV partials) */
  GQE_WS_DECODE = 5,    /* scratch of gqe_decode_step */
  GQE_WS_DENSE_DECODE = 6, /* scratch of gqa_dense_decode_step */
  GQE_WS_BACKWARD = 7      /* scratch of gqe_layer_bwd */
};

/* Items inside the GQE_WS_LAYER / GQE_WS_DENSE workspaces (for inspection). */
enum {
  GQE_ITEM_IDX = 1, GQE_ITEM_R, GQE_ITEM_OMEGA, GQE_ITEM_COUNTS, GQE_ITEM_OFFSETS,
  GQE_ITEM_TOK, GQE_ITEM_SLOT_POS, GQE_ITEM_QV, GQE_ITEM_QS, GQE_ITEM_K, GQE_ITEM_V,
  GQE_ITEM_SLOTS, GQE_ITEM_DISPATCH_WS, GQE_ITEM_ATTENTION_WS,
  GQE_ITEM_DENSE_Q = 32, GQE_ITEM_DENSE_O
};

/* Bytes of workspace the given call needs for `cfg` (0 if cfg is invalid;
 * at least 256 otherwise). */
size_t gqe_workspace_bytes(const gqe_config* cfg, int which);

/* Byte offset of `item` inside workspace `which`, or (size_t)-1. Items of
 * GQE_WS_LAYER: all above; of GQE_WS_DENSE: DENSE_Q, K, V, DENSE_O; of
 * GQE_WS_DECODE (one row per sequence): IDX, R, OMEGA, SLOTS. */
size_t gqe_workspace_offset(const gqe_config* cfg, int which, int item);

/*
 * Router: logits, per-group softmax, top-k per group, renormalised weights
 * (steps a1-a4). Router scores over the query-head experts and selection of
 * k experts inside every group: gist.science "Technical Summary", Methodology
 * ("Conditional activation"); softmax before top-k inside each group: pptc.cn
 * blog section 7; every group takes part: pptc.cn blog section 5.
 *
 *   z[row, e]  = sum_i x[row, i] * W_r[i, e] + b_r[e]      (fp32, with a
 *                certified error bound; a top-k decision whose margin is
 *                below the bound is re-taken from fp64 logits under their
 *                own certified bound, and one that bound does not settle
 *                either from the exact logits (integer sums of the exact
 *                products), so idx is the exact-arithmetic selection, ties
 *                included)
 *   p          = softmax over the M logits of each group
 *   idx[row, g, s] = the k largest j of group g, ascending, ties to lower j
 *   r[row, g, s]     = p / sum of the selected p of group g
 *   omega[row, g, s] = p / sum of the selected p of all G groups (the
 *                      weighted slot's weights; with GQE_FLAG_SLOT_GROUP_MEAN
 *                      r / G, with GQE_FLAG_OUT_WEIGHTED_CONCAT p itself)
 *
 * x [B*T, d_model] bf16; W_r [d_model, N] fp32; b_r [N] fp32 or NULL;
 * idx [B*T, G, k] int32; r, omega [B*T, G, k] fp32.
 */
gqe_status gqe_router_topk(const gqe_config* cfg, const gqe_bf16* x, const float* W_r,
                           const float* b_r, int32_t* idx, float* r, float* omega,
                           gqe_stream_t stream);

/*
 * Dispatch (step a5) and the grouped query projection over the active rows
 * only (step a7): only the selected experts compute a query ("reduces only
 * the active query-head computation": chatpaper / hotpaper abstract).
 *
 *   counts[e*B + b]  tokens of sequence b that selected expert e
 *   offsets[e*B + b] exclusive prefix sum of counts in (e, b) order;
 *                    offsets[N*B] = k*G*B*T
 *   tok[offsets[e*B+b] + i] = i-th smallest position t of sequence b that
 *                    selected e (stable, bit-exact)
 *   slot_pos[row, g, s] = index in tok of the entry of that selection
 *   Qv[b, g, s, t, :] = x[row] @ W_q[:, e*dh:(e+1)*dh] for e = g*M + idx[row,g,s]
 *   Qs[b, t, :]       = x[row] @ W_qs   (the always-on shared head)
 *
 * idx [B*T, G, k] int32 (from gqe_router_topk); x [B*T, d_model];
 * W_q [d_model, N*d_head]; W_qs [d_model, d_head]; counts [N*B];
 * offsets [N*B + 1]; tok [k*G*B*T]; slot_pos [B*T, G, k];
 * Qv [B, G, k, T, d_head]; Qs [B, T, d_head] (NULL allowed, and not
 * written, when the output construction has no shared head).
 * ws: >= gqe_workspace_bytes(cfg, GQE_WS_DISPATCH) bytes.
 */
gqe_status gqe_dispatch(const gqe_config* cfg, const int32_t* idx, const gqe_bf16* x,
                        const gqe_bf16* W_q, const gqe_bf16* W_qs, int32_t* counts,
                        int32_t* offsets, int32_t* tok, int32_t* slot_pos, gqe_bf16* Qv,
                        gqe_bf16* Qs, void* ws, size_t ws_bytes, gqe_stream_t stream);

/*
 * gqe_dispatch without a workspace argument (the paper has no counterpart:
 * this is a calling convention of this library). For callers that cannot
 * allocate device memory per call -- their memory belongs to another
 * allocator, e.g. a serving runtime that reserves the GPU at start-up or a
 * plugin interface that passes only input and output buffers. The scratch
 * lives in a 4 MiB static device array of the library (held by every GPU that
 * loads it, until exit); arguments and results are those of gqe_dispatch.
 *  - The first call on a device looks up the array's address on that device;
 *    make it before any stream capture. The address is kept for the life of
 *    the process: do not use this entry point after cudaDeviceReset (or any
 *    other teardown of the device's primary context) in the same process.
 *  - All calls on a device share the array: calls that overlap on the GPU
 *    race. Each call writes every scratch word before reading it.
 *  - Configurations needing more than 4 MiB of dispatch scratch
 *    (gqe_workspace_bytes(cfg, GQE_WS_DISPATCH)) return GQE_ERR_WORKSPACE.
 */
gqe_status gqe_dispatch_noalloc(const gqe_config* cfg, const int32_t* idx, const gqe_bf16* x,
                                const gqe_bf16* W_q, const gqe_bf16* W_qs, int32_t* counts,
                                int32_t* offsets, int32_t* tok, int32_t* slot_pos,
                                gqe_bf16* Qv, gqe_bf16* Qs, gqe_stream_t stream);

/*
 * Dense, unchanged K/V projection of every group (step a6; "the Key-Value
 * projections and the KV cache stay dense and unchanged": gist.science
 * "Technical Summary", Dense KV path). The dense GQA path uses this same call.
 *   K[b, g, t, :] = x[row] @ W_k[:, g*dh:(g+1)*dh], V likewise with W_v.
 * x [B*T, d_model]; W_k, W_v [d_model, G*d_head]; K, V [B, G, T, d_head].
 */
gqe_status gqe_kv_proj(const gqe_config* cfg, const gqe_bf16* x, const gqe_bf16* W_k,
                       const gqe_bf16* W_v, gqe_bf16* K, gqe_bf16* V, gqe_stream_t stream);

/*
 * Routed and shared causal attention (steps a8, a9): every routed slot stream
 * (g, s) attends causally to K/V of group g; the shared head to K/V of group
 * 0. o[t] = sum_{u<=t} softmax_u(q[t].K[u] / sqrt(dh)) V[u], fp32 softmax and
 * accumulation, bf16 output written straight into the slot buffer:
 *   slots[row, (g*k+s)*dh ...] routed, slots[row, k*G*dh ...] shared.
 * Slot kG+1 (weighted) is not touched.
 * Short sequences are split along the keys (each CTA takes a chunk of KV
 * tiles; the last CTA of a query-tile pair merges the chunks' unnormalised
 * rows), which needs scratch from ws: >= gqe_workspace_bytes(cfg,
 * GQE_WS_ATTENTION). Calls sharing one ws must not overlap on the GPU. The
 * call clears the scratch's arrival counters first unless cfg->flags has
 * GQE_FLAG_WS_CLEAN.
 * Qv [B, G, k, T, d_head]; Qs [B, T, d_head] (unused, NULL allowed, when
 * the output construction has no shared head); K, V [B, G, T, d_head];
 * slots [B*T, S*d_head] (S of the output construction: kG+2 by default).
 */
gqe_status gqe_attention_fwd(const gqe_config* cfg, const gqe_bf16* Qv, const gqe_bf16* Qs,
                             const gqe_bf16* K, const gqe_bf16* V, gqe_bf16* slots, void* ws,
                             size_t ws_bytes, gqe_stream_t stream);

/*
 * The same attention (steps a8, a9) over compacted, expert-major query
 * tiles: the routed causal attention streams tiles of 128 consecutive entries
 * of one (expert, sequence) token list against the group's dense K/V, masks
 * each row causally by its original position tok[r], and never loads a K/V
 * tile that lies entirely after a tile's last position; empty lists take no
 * work ("only the selected query experts, plus one always-on shared head,
 * run causal attention against their group's dense, unchanged KV head":
 * gist.science "Technical Summary", Conditional activation and Dense KV
 * path). The shared head runs as in gqe_attention_fwd.
 *   slots[b*T + tok[r], (g*k+s)*dh ...] = o of list entry r, where the entry
 *   belongs to expert e = g*M + j of sequence b and s is the rank of j among
 *   the token's k selections in group g (from idx).
 * Qe [k*G*B*T, d_head] in list order (gqe_dispatch with GQE_FLAG_EXPERT_MAJOR);
 * Qs [B, T, d_head]; K, V [B, G, T, d_head]; idx, offsets, tok as written by
 * gqe_router_topk and gqe_dispatch; slots [B*T, (k*G+2)*d_head]. No
 * workspace. Slot kG+1 is not touched.
 */
gqe_status gqe_attention_fwd_compact(const gqe_config* cfg, const gqe_bf16* Qe, const gqe_bf16* Qs,
                                     const gqe_bf16* K, const gqe_bf16* V, const int32_t* idx,
                                     const int32_t* offsets, const int32_t* tok, gqe_bf16* slots,
                                     gqe_stream_t stream);

/*
 * Weighted slot and output projection (steps a10, a11): the renormalised
 * weighted sum of the selected experts' outputs ("Output Construction":
 * gist.science "Technical Summary"), then y = slots @ W_O with W_O of size
 * (kG+2) x d (hotpaper.ai summary, Technical approach).
 *   slots[row, (kG+1)*dh ...] = sum_{g,s} omega[row,g,s] * slots[row, (g*k+s)*dh ...]
 *   y = slots @ W_o
 * slots [B*T, (k*G+2)*d_head] (updated in place); omega [B*T, G, k] fp32;
 * W_o [(k*G+2)*d_head, d_model]; y [B*T, d_model].
 * With GQE_FLAG_OUT_HARD: y = slots @ W_o over the kG routed slots
 * (slots [B*T, kG*d_head], W_o [kG*d_head, d_model]); with
 * GQE_FLAG_OUT_WEIGHTED_CONCAT each routed slot is first scaled in place by
 * omega (= its in-group probability, rounded to bf16 once).
 */
gqe_status gqe_output_proj(const gqe_config* cfg, gqe_bf16* slots, const float* omega,
                           const gqe_bf16* W_o, gqe_bf16* y, gqe_stream_t stream);

/*
 * The whole GQE layer (a1-a11), ordered on `stream`; every intermediate
 * lives in `ws` (>= gqe_workspace_bytes(cfg, GQE_WS_LAYER); see
 * gqe_workspace_offset). The K/V and shared-head query projections run on a
 * side stream owned by the library (one per device) that forks from `stream`
 * after the router and joins it before the attention, so the call is still
 * stream-ordered as a whole (and captures into a CUDA graph as a fork/join).
 * The results are bitwise those of the step calls. Batches of at most 4096
 * rows with d_head 64 (slot-major) take every expert's queries from one dense
 * GEMM that stores only the routed rows: the token lists (COUNTS, OFFSETS,
 * TOK, SLOT_POS) of the workspace are then not written. Arguments as in the
 * calls above.
 */
gqe_status gqe_layer_fwd(const gqe_config* cfg, const gqe_bf16* x, const float* W_r,
                         const float* b_r, const gqe_bf16* W_q, const gqe_bf16* W_qs,
                         const gqe_bf16* W_k, const gqe_bf16* W_v, const gqe_bf16* W_o,
                         gqe_bf16* y, void* ws, size_t ws_bytes, gqe_stream_t stream);

/*
 * Dense GQA layer with all N query heads active: the all-active baseline of
 * the speed-up (gist.science "Technical Summary", Experimental Results;
 * pptc.cn blog Table 1, first row). Q = x @ W_q [d_model, N*d_head]; K/V via
 * gqe_kv_proj; head h attends to group h / M; O [B*T, N*d_head];
 * y = O @ W_o_dense [N*d_head, d_model]. ws >= gqe_workspace_bytes(cfg,
 * GQE_WS_DENSE). `k` of cfg is ignored.
 */
gqe_status gqa_dense_fwd(const gqe_config* cfg, const gqe_bf16* x, const gqe_bf16* W_q,
                         const gqe_bf16* W_k, const gqe_bf16* W_v, const gqe_bf16* W_o_dense,
                         gqe_bf16* y, void* ws, size_t ws_bytes, gqe_stream_t stream);

/*
 * Synchronises the current device, returns its status word in
 * *device_status_out (a gqe_status value; 0 = no device-side failure since
 * the last read) and clears it. Returns GQE_ERR_CUDA if the device cannot
 * be synchronised.
 */
gqe_status gqe_read_status(int32_t* device_status_out);

/* Launches one CTA that waits, with the given bound, on a barrier nothing
 * completes; exercises the device-side timeout path (status GQE_ERR_TIMEOUT)
 * without hanging the GPU. limit_ns must be in [1e3, 5e9]. */
gqe_status gqe_selftest_wait_timeout(uint64_t limit_ns, gqe_stream_t stream);

const char* gqe_status_string(gqe_status s);

/* Library ABI version (major*100 + minor). */
int gqe_version(void);

/*
 * Decode step (one new token per sequence against its K/V cache). The K/V
 * cache stays dense and unchanged ("the Key-Value projections and the KV
 * cache stay dense and unchanged": gist.science "Technical Summary", Dense KV
 * path); the new token's output is the prefill definition (steps a1-a11) at
 * its position: the router picks k experts per group for it, only those
 * experts' queries and the shared head attend to the cache and the token's
 * own key, then the (kG+2) slots and W_O.
 *   cfg->B   sequences, one new token each;
 *   cfg->T   keys after the step: the new token is at position T - 1 and
 *            the cache holds positions 0 .. T-2 on entry (T >= 1);
 *   x        [B, d_model] the new tokens;
 *   K_cache, V_cache [B, G, cache_capacity, d_head], cache_capacity >= T;
 *            the call writes the new token's K and V at position T - 1;
 *   y        [B, d_model].
 * Scratch: >= gqe_workspace_bytes(cfg, GQE_WS_DECODE) (0 when unsupported:
 * more than 16 query heads per group). GQE_ERR_UNSUPPORTED also for B >
 * 65535. The extent limits of the other calls apply to the B new rows, not
 * to the cache length. Weights as in gqe_layer_fwd.
 */
gqe_status gqe_decode_step(const gqe_config* cfg, const gqe_bf16* x, const float* W_r,
                           const float* b_r, const gqe_bf16* W_q, const gqe_bf16* W_qs,
                           const gqe_bf16* W_k, const gqe_bf16* W_v, const gqe_bf16* W_o,
                           gqe_bf16* K_cache, gqe_bf16* V_cache, int32_t cache_capacity, gqe_bf16* y,
                           void* ws, size_t ws_bytes, gqe_stream_t stream);

/* Dense-GQA decode step: every one of the N heads (head h on group h / M)
 * against the same cache; W_o_dense [N*d_head, d_model]. cfg->k is ignored.
 * Scratch: gqe_workspace_bytes(cfg, GQE_WS_DENSE_DECODE). */
gqe_status gqa_dense_decode_step(const gqe_config* cfg, const gqe_bf16* x, const gqe_bf16* W_q,
                                 const gqe_bf16* W_k, const gqe_bf16* W_v,
                                 const gqe_bf16* W_o_dense, gqe_bf16* K_cache, gqe_bf16* V_cache,
                                 int32_t cache_capacity, gqe_bf16* y, void* ws, size_t ws_bytes,
                                 gqe_stream_t stream);

/*
 * Backward of the layer (the default output construction; cfg->flags may
 * hold GQE_FLAG_WS_CLEAN only, else GQE_ERR_UNSUPPORTED): given
 * dy = dL/dy [B*T, d_model] (fp32), the gradients of L with the router's
 * top-k selection held fixed -- the selection is a discrete choice, and the
 * weighted slot is the layer's differentiable path from the loss to the
 * router ("a differentiable path for the language-modelling loss to reach the
 * router": gist.science Technical Summary, Output Construction). Through the
 * weighted slot the router gets d(omega) = <o, dS_w>, the quotient rule of
 * omega = p_sel / sum(p_sel) and each group's softmax Jacobian. The forward
 * is recomputed first (as gqe_layer_fwd, into the scratch; the attention also
 * keeps each row's log-sum-exp) and the gradients use its bf16 intermediates
 * (routing, Q, K, V, slots). The products run on the tensor cores with bf16
 * operands (dy, dO, P, dS and the gradients of Q, K, V and the router logits
 * each rounded once) and fp32 accumulation; the result is deterministic.
 * Outputs (fp32, overwritten): dx [B*T, d_model], dW_r [d_model, N],
 * db_r [N] (NULL: not computed), dW_q [d_model, N*d_head],
 * dW_qs [d_model, d_head], dW_k, dW_v [d_model, G*d_head],
 * dW_o [(kG+2)*d_head, d_model]. Inputs as in gqe_layer_fwd.
 * Scratch: >= gqe_workspace_bytes(cfg, GQE_WS_BACKWARD).
 */
gqe_status gqe_layer_bwd(const gqe_config* cfg, const gqe_bf16* x, const float* W_r, const float* b_r,
                         const gqe_bf16* W_q, const gqe_bf16* W_qs, const gqe_bf16* W_k, const gqe_bf16* W_v,
                         const gqe_bf16* W_o, const float* dy, float* dx, float* dW_r, float* db_r,
                         float* dW_q, float* dW_qs, float* dW_k, float* dW_v, float* dW_o, void* ws,
                         size_t ws_bytes, gqe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GQE_H_ */
