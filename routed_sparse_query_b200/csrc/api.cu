// C ABI of libgqe.so: argument validation, workspace layout and the order of
// the kernel launches. Every call is asynchronous on the caller's stream and
// launches nothing when validation fails.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "gqe_internal.h"
#include "ptx.cuh"

namespace gqe {

namespace api_impl {

size_t round256(size_t v) { return (v + 255) / 256 * 256; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <typename... P>
bool all_aligned(const P*... ps) {
  bool ok = true;
  ((ok = ok && ps != nullptr && aligned16(ps)), ...);
  return ok;
}

gqe_status check_cfg(const gqe_config* c) {
  if (c == nullptr) return GQE_ERR_INVALID;
  if (c->B < 1 || c->T < 1 || c->G < 1 || c->M < 1 || c->k < 1 || c->k > c->M) return GQE_ERR_INVALID;
  if (c->d_model < 64 || c->d_model % 64 != 0 ||
      (c->flags & ~(GQE_FLAG_WS_CLEAN | GQE_FLAG_EXPERT_MAJOR | kOutFlags | GQE_FLAG_NO_SHARED_HEAD)) != 0u)
    return GQE_ERR_INVALID;
  const uint32_t out = c->flags & kOutFlags;
  if ((out & (out - 1u)) != 0u) return GQE_ERR_INVALID;  // at most one output construction
  // A shard without the shared head keeps the weighted slot.
  if ((c->flags & GQE_FLAG_NO_SHARED_HEAD) && (out & (GQE_FLAG_OUT_HARD | GQE_FLAG_OUT_WEIGHTED_CONCAT)))
    return GQE_ERR_INVALID;
  if (c->G * c->M > kMaxExperts || c->G > 32) return GQE_ERR_UNSUPPORTED;
  if (c->d_head != 32 && c->d_head != 64) return GQE_ERR_UNSUPPORTED;
  // Index arithmetic of the kernels stays within int32 for these extents.
  const long long R = static_cast<long long>(c->B) * c->T;
  const long long N = static_cast<long long>(c->G) * c->M;
  if (R * c->d_model >= (1ll << 31) * 4 || R * (N + 2) * c->d_head >= (1ll << 31) ||
      R * c->G * c->k * 4 >= (1ll << 31))
    return GQE_ERR_UNSUPPORTED;
  if (router_smem_bytes(*c) > kRouterSmemLimit) return GQE_ERR_UNSUPPORTED;
  return GQE_OK;
}

gqe_status cuda_status(int e) { return e == cudaSuccess ? GQE_OK : GQE_ERR_CUDA; }

struct LayerWs {
  size_t idx, r, omega, counts, offsets, tok, slot_pos, Qv, Qs, K, V, slots, dws, aws, total;
};

// Short batches (at most this many rows, d_head 64, slot-major attention):
// the queries of every expert come from one dense GEMM whose epilogue stores
// only the routed rows, straight into the slot-major streams, so the dispatch
// lists and the gathered routed Q GEMM leave the critical path (at the price
// of the unselected experts' projection FLOPs). The routed Q rows are the
// same values either way.
constexpr long long kShortBatchRows = 4096;
bool short_batch_path(const gqe_config& c) {
  return c.d_head == 64 && (c.flags & GQE_FLAG_EXPERT_MAJOR) == 0u &&
         static_cast<long long>(c.B) * c.T <= kShortBatchRows;
}

LayerWs layer_ws(const gqe_config& c) {
  const size_t R = static_cast<size_t>(c.B) * c.T;
  const size_t N = static_cast<size_t>(c.G) * c.M;
  const size_t sel = R * c.G * c.k;
  const size_t dh = c.d_head;
  LayerWs L{};
  size_t o = 0;
  auto put = [&](size_t& field, size_t bytes) {
    field = o;
    o = round256(o + bytes);
  };
  put(L.idx, sel * 4);
  put(L.r, sel * 4);
  put(L.omega, sel * 4);
  put(L.counts, N * c.B * 4);
  put(L.offsets, (N * c.B + 1) * 4);
  put(L.tok, sel * 4);
  put(L.slot_pos, sel * 4);
  put(L.Qv, sel * dh * 2);
  put(L.Qs, R * dh * 2);
  put(L.K, R * c.G * dh * 2);
  put(L.V, R * c.G * dh * 2);
  put(L.slots, R * n_slots(c) * dh * 2);
  put(L.dws, dispatch_ws_layout(c).total);
  put(L.aws, attention_plan(c, n_streams(c)).total);
  L.total = o;
  return L;
}

// Backward: the layer's workspace (the recomputed forward), y of the
// recomputation, then the fp32 gradients in flight.
struct BwdWs {
  LayerWs L;
  size_t y, dS, dOr, dOs, dz, stats, dQr, dQs, dKp, dVp;  // fp32
  size_t dy16, WoT, sT, xT, WcT, Y, dO16;                 // bf16 operands of the tensor-core GEMMs
  size_t lse, zl, Drow;                                   // the forward attention's row statistics; logits; dO . O
  long long ldR, ldS, Kcat, zoff;
  size_t total;
};

BwdWs bwd_ws(const gqe_config& c) {
  BwdWs W{};
  W.L = layer_ws(c);
  const size_t R = static_cast<size_t>(c.B) * c.T, dh = c.d_head, d = c.d_model;
  const size_t gk = static_cast<size_t>(c.G) * c.k, N = static_cast<size_t>(c.G) * c.M;
  const size_t Sdh = (gk + 2) * dh;
  W.ldR = static_cast<long long>((R + 7) / 8 * 8);
  W.ldS = static_cast<long long>((Sdh + 63) / 64 * 64);
  W.zoff = static_cast<long long>(N * dh + dh + 2 * c.G * dh);
  W.Kcat = W.zoff + static_cast<long long>((N + 63) / 64 * 64);
  size_t o = W.L.total;
  auto put = [&](size_t& field, size_t bytes) {
    field = o;
    o = round256(o + bytes);
  };
  put(W.y, R * d * 2);
  put(W.dS, R * Sdh * 4);
  put(W.dOr, R * gk * dh * 4);
  put(W.dOs, R * dh * 4);
  put(W.dz, R * N * 4);
  put(W.stats, static_cast<size_t>(c.B) * (gk + 1) * ((c.T + 63) / 64 * 64) * 8);
  put(W.dQr, 2 * R * gk * dh * 4);
  put(W.dQs, 2 * R * dh * 4);
  put(W.dKp, 2 * R * (gk + 1) * dh * 4);
  put(W.dVp, 2 * R * (gk + 1) * dh * 4);
  put(W.dy16, R * d * 2);
  put(W.WoT, d * W.ldS * 2);
  put(W.sT, Sdh * W.ldR * 2);
  put(W.xT, d * W.ldR * 2);
  put(W.WcT, static_cast<size_t>(W.Kcat) * d * 2);
  put(W.Y, R * W.Kcat * 2);
  put(W.dO16, R * (gk + 1) * dh * 2);
  put(W.lse, static_cast<size_t>(c.B) * (gk + 1) * ((c.T + 63) / 64 * 64) * 4);
  put(W.zl, R * N * 4);
  put(W.Drow, static_cast<size_t>(c.B) * (gk + 1) * ((c.T + 63) / 64 * 64) * 4);
  W.total = o;
  return W;
}

// Decode step: the layer's per-token buffers for B rows (one new token per
// sequence; K/V go to the caller's cache), then the decode attention scratch.
gqe_config decode_rows_cfg(const gqe_config& c) {
  gqe_config c1 = c;
  c1.T = 1;
  return c1;
}

struct DecodeWs {
  LayerWs L1;
  size_t daws, total;
};

DecodeWs decode_ws(const gqe_config& c) {
  DecodeWs D{};
  D.L1 = layer_ws(decode_rows_cfg(c));
  D.daws = round256(D.L1.total);
  D.total = D.daws + decode_attention_ws_bytes(c, false);
  return D;
}

struct DenseDecodeWs {
  size_t Q, O, daws, total;
};

DenseDecodeWs dense_decode_ws(const gqe_config& c) {
  const size_t N = static_cast<size_t>(c.G) * c.M;
  DenseDecodeWs D{};
  D.Q = 0;
  D.O = round256(static_cast<size_t>(c.B) * N * c.d_head * 2);
  D.daws = round256(D.O + static_cast<size_t>(c.B) * N * c.d_head * 2);
  D.total = D.daws + decode_attention_ws_bytes(c, true);
  return D;
}

struct DenseWs {
  size_t Q, K, V, O, aws, total;
};

DenseWs dense_ws(const gqe_config& c) {
  const size_t R = static_cast<size_t>(c.B) * c.T;
  const size_t N = static_cast<size_t>(c.G) * c.M;
  const size_t dh = c.d_head;
  DenseWs L{};
  size_t o = 0;
  auto put = [&](size_t& field, size_t bytes) {
    field = o;
    o = round256(o + bytes);
  };
  put(L.Q, R * N * dh * 2);
  put(L.K, R * c.G * dh * 2);
  put(L.V, R * c.G * dh * 2);
  put(L.O, R * N * dh * 2);
  put(L.aws, attention_plan(c, static_cast<int>(N)).total);
  L.total = o;
  return L;
}

// One warp waits, with a bound, on a barrier that nothing completes: the
// wait gives up after limit_ns and records GQE_ERR_TIMEOUT.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, limit_ns);
  __syncwarp();
}

// Per-device side stream for the K/V (and shared-head Q) projections of
// gqe_layer_fwd: they read only x and the weights, so they run beside the
// dispatch and the routed Q projection (fork on the caller's stream after the router, join before the
// attention). Created on first use; the enqueue sequence is serialised by
// the mutex so that concurrent callers on one device do not interleave
// their event records. Captured into CUDA graphs like any fork/join.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  bool ok = false;
};
std::mutex g_side_mu;
SideStream g_side[64];

SideStream* side_stream_locked() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  SideStream& ss = g_side[dev];
  if (!ss.ok) {
    if (cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    if (cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess)
      return nullptr;
    ss.ok = true;
  }
  return &ss;
}

// Token lists and the routed query projection (plus the shared head unless
// Qs is null), after the caller's checks.
gqe_status dispatch_and_project(const gqe_config& c, const int32_t* idx, const gqe_bf16* x,
                                const gqe_bf16* W_q, const gqe_bf16* W_qs, int32_t* counts,
                                int32_t* offsets, int32_t* tok, int32_t* slot_pos, gqe_bf16* Qv,
                                gqe_bf16* Qs, void* ws, size_t ws_bytes, gqe_stream_t stream) {
  const DispatchWs L = dispatch_ws_layout(c);
  if (ws_bytes < L.total) return GQE_ERR_WORKSPACE;
  int e = launch_dispatch_lists(c, idx, counts, offsets, tok, slot_pos, ws, L, stream);
  if (e != cudaSuccess) return GQE_ERR_CUDA;
  char* w = static_cast<char*>(ws);
  return cuda_status(gemm_q_routed(c, x, W_q, W_qs, idx, tok, w + L.qtiles,
                                   reinterpret_cast<const int32_t*>(w + L.n_qtiles), L.max_qtiles,
                                   Qv, Qs, (c.flags & GQE_FLAG_EXPERT_MAJOR) != 0u, stream));
}

}  // namespace api_impl
using namespace api_impl;

}  // namespace gqe

using namespace gqe;

extern "C" {

size_t gqe_workspace_bytes(const gqe_config* cfg, int which) {
  if (cfg != nullptr && (which == GQE_WS_DECODE || which == GQE_WS_DENSE_DECODE)) {
    // Decode: the per-token buffers have B rows; T is the cache length.
    gqe_config c1 = decode_rows_cfg(*cfg);
    if (which == GQE_WS_DENSE_DECODE) c1.k = 1;
    if (cfg->T < 1 || check_cfg(&c1) != GQE_OK || (cfg->flags & (kOutFlags | GQE_FLAG_NO_SHARED_HEAD)) != 0u)
      return 0;
    if (which == GQE_WS_DECODE) return decode_heads(*cfg, false) > 16 ? 0 : decode_ws(*cfg).total;
    gqe_config cd = *cfg;
    cd.k = 1;
    return decode_heads(cd, true) > 16 ? 0 : dense_decode_ws(cd).total;
  }
  if (check_cfg(cfg) != GQE_OK) return 0;
  switch (which) {
    case GQE_WS_DISPATCH: return dispatch_ws_layout(*cfg).total;
    case GQE_WS_LAYER: return layer_ws(*cfg).total;
    case GQE_WS_BACKWARD:
      return (cfg->flags & ~GQE_FLAG_WS_CLEAN) != 0u ? 0 : bwd_ws(*cfg).total;
    case GQE_WS_DENSE: return dense_ws(*cfg).total;
    case GQE_WS_ATTENTION: {
      const size_t t = attention_plan(*cfg, n_streams(*cfg)).total;
      return t > 256 ? t : 256;
    }
    default: return 0;
  }
}

size_t gqe_workspace_offset(const gqe_config* cfg, int which, int item) {
  const size_t bad = static_cast<size_t>(-1);
  if (cfg != nullptr && which == GQE_WS_DECODE) {
    // The decode step's per-token buffers (one row per sequence).
    if (gqe_workspace_bytes(cfg, GQE_WS_DECODE) == 0) return bad;
    const LayerWs& L = decode_ws(*cfg).L1;
    switch (item) {
      case GQE_ITEM_IDX: return L.idx;
      case GQE_ITEM_R: return L.r;
      case GQE_ITEM_OMEGA: return L.omega;
      case GQE_ITEM_SLOTS: return L.slots;
      default: return bad;
    }
  }
  if (check_cfg(cfg) != GQE_OK) return bad;
  if (which == GQE_WS_LAYER) {
    const LayerWs L = layer_ws(*cfg);
    switch (item) {
      case GQE_ITEM_IDX: return L.idx;
      case GQE_ITEM_R: return L.r;
      case GQE_ITEM_OMEGA: return L.omega;
      case GQE_ITEM_COUNTS: return L.counts;
      case GQE_ITEM_OFFSETS: return L.offsets;
      case GQE_ITEM_TOK: return L.tok;
      case GQE_ITEM_SLOT_POS: return L.slot_pos;
      case GQE_ITEM_QV: return L.Qv;
      case GQE_ITEM_QS: return L.Qs;
      case GQE_ITEM_K: return L.K;
      case GQE_ITEM_V: return L.V;
      case GQE_ITEM_SLOTS: return L.slots;
      case GQE_ITEM_DISPATCH_WS: return L.dws;
      case GQE_ITEM_ATTENTION_WS: return L.aws;
      default: return bad;
    }
  }
  if (which == GQE_WS_DENSE) {
    const DenseWs L = dense_ws(*cfg);
    switch (item) {
      case GQE_ITEM_DENSE_Q: return L.Q;
      case GQE_ITEM_K: return L.K;
      case GQE_ITEM_V: return L.V;
      case GQE_ITEM_DENSE_O: return L.O;
      default: return bad;
    }
  }
  return bad;
}

gqe_status gqe_router_topk(const gqe_config* cfg, const gqe_bf16* x, const float* W_r,
                           const float* b_r, int32_t* idx, float* r, float* omega,
                           gqe_stream_t stream) {
  const gqe_status s = check_cfg(cfg);
  if (s != GQE_OK) return s;
  if (!all_aligned(x, W_r, idx, r, omega)) return GQE_ERR_INVALID;
  if (b_r != nullptr && (reinterpret_cast<uintptr_t>(b_r) & 3u)) return GQE_ERR_INVALID;
  return cuda_status(launch_router(*cfg, x, W_r, b_r, idx, r, omega, stream));
}

gqe_status gqe_dispatch(const gqe_config* cfg, const int32_t* idx, const gqe_bf16* x,
                        const gqe_bf16* W_q, const gqe_bf16* W_qs, int32_t* counts,
                        int32_t* offsets, int32_t* tok, int32_t* slot_pos, gqe_bf16* Qv,
                        gqe_bf16* Qs, void* ws, size_t ws_bytes, gqe_stream_t stream) {
  const gqe_status s = check_cfg(cfg);
  if (s != GQE_OK) return s;
  const bool shared = has_shared_head(*cfg);
  if (!all_aligned(idx, x, W_q, counts, offsets, tok, slot_pos, Qv) || ws == nullptr || !aligned16(ws) ||
      (shared && !all_aligned(W_qs, Qs)))
    return GQE_ERR_INVALID;
  return dispatch_and_project(*cfg, idx, x, W_q, W_qs, counts, offsets, tok, slot_pos, Qv,
                              shared ? Qs : nullptr, ws, ws_bytes, stream);
}

gqe_status gqe_kv_proj(const gqe_config* cfg, const gqe_bf16* x, const gqe_bf16* W_k,
                       const gqe_bf16* W_v, gqe_bf16* K, gqe_bf16* V, gqe_stream_t stream) {
  const gqe_status s = check_cfg(cfg);
  if (s != GQE_OK) return s;
  if (!all_aligned(x, W_k, W_v, K, V)) return GQE_ERR_INVALID;
  return cuda_status(gemm_kv(*cfg, x, W_k, W_v, K, V, stream));
}

gqe_status gqe_attention_fwd(const gqe_config* cfg, const gqe_bf16* Qv, const gqe_bf16* Qs,
                             const gqe_bf16* K, const gqe_bf16* V, gqe_bf16* slots, void* ws,
                             size_t ws_bytes, gqe_stream_t stream) {
  const gqe_status s = check_cfg(cfg);
  if (s != GQE_OK) return s;
  if (!all_aligned(Qv, K, V, slots) || (has_shared_head(*cfg) && !all_aligned(Qs))) return GQE_ERR_INVALID;
  const size_t need = attention_plan(*cfg, n_streams(*cfg)).total;
  if (need > 0 && (ws == nullptr || !aligned16(ws))) return GQE_ERR_INVALID;
  if (ws_bytes < need) return GQE_ERR_WORKSPACE;
  const bool clean = (cfg->flags & GQE_FLAG_WS_CLEAN) != 0u;
  return cuda_status(attention_gqe(*cfg, Qv, Qs, K, V, slots, ws, ws_bytes, clean, stream));
}

gqe_status gqe_attention_fwd_compact(const gqe_config* cfg, const gqe_bf16* Qe, const gqe_bf16* Qs,
                                     const gqe_bf16* K, const gqe_bf16* V, const int32_t* idx,
                                     const int32_t* offsets, const int32_t* tok, gqe_bf16* slots,
                                     gqe_stream_t stream) {
  const gqe_status s = check_cfg(cfg);
  if (s != GQE_OK) return s;
  if (!all_aligned(Qe, K, V, idx, offsets, tok, slots) || (has_shared_head(*cfg) && !all_aligned(Qs)))
    return GQE_ERR_INVALID;
  return cuda_status(attention_gqe_em(*cfg, Qe, Qs, K, V, idx, offsets, tok, slots, stream));
}

gqe_status gqe_output_proj(const gqe_config* cfg, gqe_bf16* slots, const float* omega,
                           const gqe_bf16* W_o, gqe_bf16* y, gqe_stream_t stream) {
  const gqe_status s = check_cfg(cfg);
  if (s != GQE_OK) return s;
  if (!all_aligned(slots, omega, W_o, y)) return GQE_ERR_INVALID;
  return cuda_status(gemm_output(*cfg, slots, omega, W_o, y, stream));
}

// The layer forward; lse (optional, slot-major attention only) receives the
// attention rows' log-sum-exp for the backward.
static gqe_status layer_fwd(const gqe_config* cfg, const gqe_bf16* x, const float* W_r, const float* b_r,
                            const gqe_bf16* W_q, const gqe_bf16* W_qs, const gqe_bf16* W_k, const gqe_bf16* W_v,
                            const gqe_bf16* W_o, gqe_bf16* y, void* ws, size_t ws_bytes, gqe_stream_t stream,
                            float* lse, bool allow_short) {
  const gqe_status s = check_cfg(cfg);
  if (s != GQE_OK) return s;
  const bool shared = has_shared_head(*cfg);
  if (!all_aligned(x, W_r, W_q, W_k, W_v, W_o, y) || ws == nullptr || !aligned16(ws) ||
      (shared && !all_aligned(W_qs)))
    return GQE_ERR_INVALID;
  const LayerWs L = layer_ws(*cfg);
  if (ws_bytes < L.total) return GQE_ERR_WORKSPACE;
  char* w = static_cast<char*>(ws);
  auto I = [&](size_t o) { return reinterpret_cast<int32_t*>(w + o); };
  auto F = [&](size_t o) { return reinterpret_cast<float*>(w + o); };
  auto H = [&](size_t o) { return reinterpret_cast<gqe_bf16*>(w + o); };
  // The split-KV counters are zeroed first (unless the caller vouches that
  // they are), so that the kernels of the layer follow each other directly
  // (programmatic dependent launch).
  if ((cfg->flags & (GQE_FLAG_WS_CLEAN | GQE_FLAG_EXPERT_MAJOR)) == 0u &&
      zero_attention_counters(*cfg, n_streams(*cfg), w + L.aws, stream) != cudaSuccess)
    return GQE_ERR_CUDA;
  // K/V projection on the side stream (falls back to the caller's stream).
  cudaStream_t main_st = static_cast<cudaStream_t>(stream);
  const bool short_batch = allow_short && short_batch_path(*cfg);
  {
    std::lock_guard<std::mutex> guard(g_side_mu);
    // The router goes first (it heads the critical path); the K/V projection
    // forks after it and runs beside the dispatch and the Q projection.
    gqe_status st = gqe_router_topk(cfg, x, W_r, b_r, I(L.idx), F(L.r), F(L.omega), stream);
    if (st != GQE_OK) return st;
    SideStream* side = side_stream_locked();
    if (side != nullptr && (cudaEventRecord(side->fork, main_st) != cudaSuccess ||
                            cudaStreamWaitEvent(side->s, side->fork, 0) != cudaSuccess))
      return GQE_ERR_CUDA;
    // The side stream also takes the shared-head query projection (it reads
    // only x), so the routed Q projection on the critical path has only the
    // routed tiles.
    if (short_batch && cfg->M == 2) {
      // Short batch, two experts per group: K, V and every expert's queries
      // (the routed rows stored straight into the slot-major streams) in one
      // launch of four outputs; the shared head's queries on the side stream.
      if (shared && gemm_q_shared(*cfg, x, W_qs, H(L.Qs), side ? side->s : stream) != cudaSuccess)
        return GQE_ERR_CUDA;
      if (side != nullptr && cudaEventRecord(side->join, side->s) != cudaSuccess) return GQE_ERR_CUDA;
      if (gemm_kvq(*cfg, x, W_k, W_v, W_q, I(L.idx), H(L.K), H(L.V), H(L.Qv), stream) != cudaSuccess)
        return GQE_ERR_CUDA;
    } else if (short_batch) {
      // Short batch: the shared head's queries first (they join before the
      // attention), then K/V on the side stream; every expert's queries in
      // one dense GEMM on this stream, the routed rows stored straight into
      // the slot-major streams (no token lists).
      if (shared && gemm_q_shared(*cfg, x, W_qs, H(L.Qs), side ? side->s : stream) != cudaSuccess)
        return GQE_ERR_CUDA;
      const gqe_status kv = gqe_kv_proj(cfg, x, W_k, W_v, H(L.K), H(L.V), side ? side->s : stream);
      if (kv != GQE_OK) return kv;
      if (side != nullptr && cudaEventRecord(side->join, side->s) != cudaSuccess) return GQE_ERR_CUDA;
      if (gemm_q_all_routed(*cfg, x, W_q, I(L.idx), H(L.Qv), stream) != cudaSuccess) return GQE_ERR_CUDA;
    } else {
      const gqe_status kv = gqe_kv_proj(cfg, x, W_k, W_v, H(L.K), H(L.V), side ? side->s : stream);
      if (kv != GQE_OK) return kv;
      if (shared && gemm_q_shared(*cfg, x, W_qs, H(L.Qs), side ? side->s : stream) != cudaSuccess)
        return GQE_ERR_CUDA;
      if (side != nullptr && cudaEventRecord(side->join, side->s) != cudaSuccess) return GQE_ERR_CUDA;
      st = dispatch_and_project(*cfg, I(L.idx), x, W_q, W_qs, I(L.counts), I(L.offsets), I(L.tok),
                                I(L.slot_pos), H(L.Qv), nullptr, w + L.dws, L.total - L.dws, stream);
      if (st != GQE_OK) return st;
    }
    if (side != nullptr && cudaStreamWaitEvent(main_st, side->join, 0) != cudaSuccess)
      return GQE_ERR_CUDA;
  }
  const int ea = (cfg->flags & GQE_FLAG_EXPERT_MAJOR) != 0u
                     ? attention_gqe_em(*cfg, H(L.Qv), H(L.Qs), H(L.K), H(L.V), I(L.idx), I(L.offsets),
                                        I(L.tok), H(L.slots), stream)
                     : attention_gqe(*cfg, H(L.Qv), H(L.Qs), H(L.K), H(L.V), H(L.slots), w + L.aws,
                                     L.total - L.aws, true, stream, lse);
  if (ea != cudaSuccess) return GQE_ERR_CUDA;
  return gqe_output_proj(cfg, H(L.slots), F(L.omega), W_o, y, stream);
}

gqe_status gqe_layer_fwd(const gqe_config* cfg, const gqe_bf16* x, const float* W_r,
                         const float* b_r, const gqe_bf16* W_q, const gqe_bf16* W_qs,
                         const gqe_bf16* W_k, const gqe_bf16* W_v, const gqe_bf16* W_o,
                         gqe_bf16* y, void* ws, size_t ws_bytes, gqe_stream_t stream) {
  return layer_fwd(cfg, x, W_r, b_r, W_q, W_qs, W_k, W_v, W_o, y, ws, ws_bytes, stream, nullptr, true);
}

gqe_status gqe_layer_bwd(const gqe_config* cfg, const gqe_bf16* x, const float* W_r, const float* b_r,
                         const gqe_bf16* W_q, const gqe_bf16* W_qs, const gqe_bf16* W_k, const gqe_bf16* W_v,
                         const gqe_bf16* W_o, const float* dy, float* dx, float* dW_r, float* db_r,
                         float* dW_q, float* dW_qs, float* dW_k, float* dW_v, float* dW_o, void* ws,
                         size_t ws_bytes, gqe_stream_t stream) {
  const gqe_status s = check_cfg(cfg);
  if (s != GQE_OK) return s;
  if ((cfg->flags & ~GQE_FLAG_WS_CLEAN) != 0u) return GQE_ERR_UNSUPPORTED;  // the default construction only
  if (!all_aligned(x, W_r, W_q, W_qs, W_k, W_v, W_o, dy, dx, dW_r, dW_q, dW_qs, dW_k, dW_v, dW_o) ||
      ws == nullptr || !aligned16(ws) || (b_r != nullptr && (reinterpret_cast<uintptr_t>(b_r) & 3u)) ||
      (db_r != nullptr && (reinterpret_cast<uintptr_t>(db_r) & 3u)))
    return GQE_ERR_INVALID;
  const gqe_config& c = *cfg;
  const BwdWs W = bwd_ws(c);
  if (ws_bytes < W.total) return GQE_ERR_WORKSPACE;
  char* w = static_cast<char*>(ws);
  auto Fp = [&](size_t o) { return reinterpret_cast<float*>(w + o); };
  auto Hp = [&](size_t o) { return reinterpret_cast<uint16_t*>(w + o); };
  // The forward, into the layer part of the workspace (routing, Q, K, V, slots).
  gqe_status st = layer_fwd(cfg, x, W_r, b_r, W_q, W_qs, W_k, W_v, W_o, reinterpret_cast<gqe_bf16*>(w + W.y), ws,
                            W.L.total, stream, Fp(W.lse), true);
  if (st != GQE_OK) return st;
  const LayerWs& L = W.L;
  const long long R = static_cast<long long>(c.B) * c.T;
  const int d = c.d_model, dh = c.d_head, gk = c.G * c.k, N = c.G * c.M, Sdh = (gk + 2) * dh;
  const uint16_t* xb = reinterpret_cast<const uint16_t*>(x);
  const uint16_t* slots = Hp(L.slots);
  const int Ri = static_cast<int>(R);
  const long long c1 = static_cast<long long>(N) * dh, c2 = c1 + dh, c3 = c2 + static_cast<long long>(c.G) * dh,
                  c4 = W.zoff, Kc = W.Kcat;
  const int Gdh = c.G * dh;
  uint16_t* dy16 = Hp(W.dy16);
  uint16_t* WcT = Hp(W.WcT);
  uint16_t* Y = Hp(W.Y);
  auto U = [](const gqe_bf16* p) { return reinterpret_cast<const uint16_t*>(p); };
  int e = cudaSuccess;
  auto ok = [&](int r) { e = r; return r == cudaSuccess; };
  // a11: dS = dy W_O^T; dW_O = S^T dy (tensor cores, bf16 operands).
  ok(bwd_cast(dy, d, R, d, dy16, d, stream)) && ok(bwd_transpose(U(W_o), d, Sdh, d, Hp(W.WoT), W.ldS, stream)) &&
      ok(gemm_f32out(dy16, d, Ri, d, Hp(W.WoT), W.ldS, Sdh, Fp(W.dS), Sdh, stream)) &&
      ok(bwd_transpose(slots, Sdh, Ri, Sdh, Hp(W.sT), W.ldR, stream)) &&
      ok(gemm_f32out(Hp(W.sT), W.ldR, Sdh, Ri, dy16, d, d, dW_o, d, stream)) &&
      // a10, a4, a2: slots and router -> dO, dz; db = sum dz.
      ok(bwd_slots_router(c, xb, W_r, b_r, Fp(W.zl), reinterpret_cast<const int32_t*>(w + L.idx), Fp(L.omega), slots,
                          Fp(W.dS), Fp(W.dOr), Fp(W.dOs), Fp(W.dz), Hp(W.dO16), Fp(W.Drow), stream)) &&
      (db_r == nullptr || ok(bwd_colsum(Fp(W.dz), db_r, R, N, stream))) &&
      // a8: attention -> dq, dK, dV.
      ok(bwd_attention_tc(c, Hp(L.Qv), Hp(L.Qs), Hp(L.K), Hp(L.V), Hp(W.dO16), Fp(W.Drow), Fp(W.lse), Fp(W.stats),
                          Fp(W.dQr), Fp(W.dQs), Fp(W.dKp), Fp(W.dVp), stream)) &&
      // a7, a6, a1: Y = [dQ (routed, scattered to their experts) | dQs | dK | dV | dz];
      // dx = Y [W_q | W_qs | W_k | W_v | W_r]^T; each weight gradient = x^T (its columns of Y).
      ok(bwd_pack(c, Fp(W.dQr), Fp(W.dQs), Fp(W.dKp), Fp(W.dVp), Fp(W.dz), reinterpret_cast<const int32_t*>(w + L.idx),
                  Y, static_cast<int>(Kc), stream)) &&
      ok(bwd_transpose(U(W_q), c1, d, static_cast<int>(c1), WcT, d, stream)) &&
      ok(bwd_transpose(U(W_qs), dh, d, dh, WcT + c1 * d, d, stream)) &&
      ok(bwd_transpose(U(W_k), Gdh, d, Gdh, WcT + c2 * d, d, stream)) &&
      ok(bwd_transpose(U(W_v), Gdh, d, Gdh, WcT + c3 * d, d, stream)) &&
      ok(bwd_transpose(W_r, N, d, N, WcT + c4 * d, d, stream)) &&
      ok(gemm_f32out(Y, Kc, Ri, static_cast<int>(c4 + N), WcT, d, d, dx, d, stream)) &&
      ok(bwd_transpose(xb, d, Ri, d, Hp(W.xT), W.ldR, stream)) &&
      ok(gemm_f32out(Hp(W.xT), W.ldR, d, Ri, Y, Kc, static_cast<int>(c1), dW_q, c1, stream)) &&
      ok(gemm_f32out(Hp(W.xT), W.ldR, d, Ri, Y + c1, Kc, dh, dW_qs, dh, stream)) &&
      ok(gemm_f32out(Hp(W.xT), W.ldR, d, Ri, Y + c2, Kc, Gdh, dW_k, Gdh, stream)) &&
      ok(gemm_f32out(Hp(W.xT), W.ldR, d, Ri, Y + c3, Kc, Gdh, dW_v, Gdh, stream)) &&
      ok(gemm_f32out(Hp(W.xT), W.ldR, d, Ri, Y + c4, Kc, N, dW_r, N, stream));
  return cuda_status(e);
}

gqe_status gqa_dense_fwd(const gqe_config* cfg, const gqe_bf16* x, const gqe_bf16* W_q,
                         const gqe_bf16* W_k, const gqe_bf16* W_v, const gqe_bf16* W_o_dense,
                         gqe_bf16* y, void* ws, size_t ws_bytes, gqe_stream_t stream) {
  if (cfg == nullptr) return GQE_ERR_INVALID;
  gqe_config c = *cfg;
  c.k = 1;  // not used by the dense layer
  const gqe_status s = check_cfg(&c);
  if (s != GQE_OK) return s;
  if (!all_aligned(x, W_q, W_k, W_v, W_o_dense, y) || ws == nullptr || !aligned16(ws))
    return GQE_ERR_INVALID;
  const DenseWs L = dense_ws(c);
  if (ws_bytes < L.total) return GQE_ERR_WORKSPACE;
  char* w = static_cast<char*>(ws);
  auto H = [&](size_t o) { return reinterpret_cast<gqe_bf16*>(w + o); };
  int e = (c.flags & GQE_FLAG_WS_CLEAN) != 0u ? cudaSuccess
                                                : zero_attention_counters(c, c.G * c.M, w + L.aws, stream);
  if (e != cudaSuccess) return GQE_ERR_CUDA;
  if (short_batch_path(c) && c.M == 2) {
    // Short batches, two heads per group: K, V and Q in one launch of four
    // outputs (the same fusion as the GQE layer's short path).
    e = gemm_kvq(c, x, W_k, W_v, W_q, nullptr, H(L.K), H(L.V), H(L.Q), stream);
    if (e != cudaSuccess) return GQE_ERR_CUDA;
  } else {
    // K/V projection beside the Q projection (side stream, as in gqe_layer_fwd).
    std::lock_guard<std::mutex> guard(g_side_mu);
    cudaStream_t main_st = static_cast<cudaStream_t>(stream);
    SideStream* side = side_stream_locked();
    if (side != nullptr && (cudaEventRecord(side->fork, main_st) != cudaSuccess ||
                            cudaStreamWaitEvent(side->s, side->fork, 0) != cudaSuccess))
      return GQE_ERR_CUDA;
    e = gemm_kv(c, x, W_k, W_v, H(L.K), H(L.V), side ? side->s : stream);
    if (e == cudaSuccess && side != nullptr) e = cudaEventRecord(side->join, side->s);
    if (e == cudaSuccess) e = gemm_q_dense(c, x, W_q, H(L.Q), stream);
    if (e == cudaSuccess && side != nullptr) e = cudaStreamWaitEvent(main_st, side->join, 0);
    if (e != cudaSuccess) return GQE_ERR_CUDA;
  }
  e = attention_dense(c, H(L.Q), H(L.K), H(L.V), H(L.O), w + L.aws, L.total - L.aws, true, stream);
  if (e != cudaSuccess) return GQE_ERR_CUDA;
  const int N = c.G * c.M;
  return cuda_status(gemm_rowmajor(H(L.O), c.B * c.T, N * c.d_head, W_o_dense, c.d_model, y, stream));
}

gqe_status gqe_read_status(int32_t* device_status_out) {
  if (device_status_out == nullptr) return GQE_ERR_INVALID;
  if (cudaDeviceSynchronize() != cudaSuccess) return GQE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return GQE_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return GQE_ERR_CUDA;
  *device_status_out = v;
  return GQE_OK;
}

gqe_status gqe_selftest_wait_timeout(uint64_t limit_ns, gqe_stream_t stream) {
  if (limit_ns < 1000ull || limit_ns > 5000000000ull) return GQE_ERR_INVALID;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  return cuda_status(cudaGetLastError());
}

const char* gqe_status_string(gqe_status s) {
  switch (s) {
    case GQE_OK: return "ok";
    case GQE_ERR_INVALID: return "invalid argument";
    case GQE_ERR_UNSUPPORTED: return "unsupported configuration";
    case GQE_ERR_WORKSPACE: return "workspace too small";
    case GQE_ERR_CUDA: return "CUDA error";
    case GQE_ERR_TIMEOUT: return "device-side wait timed out";
    case GQE_ERR_DEVICE_CHECK: return "device-side check failed";
    default: return "unknown status";
  }
}

int gqe_version(void) { return 100; }

}  // extern "C"

gqe_status gqe_decode_step(const gqe_config* cfg, const gqe_bf16* x, const float* W_r,
                           const float* b_r, const gqe_bf16* W_q, const gqe_bf16* W_qs,
                           const gqe_bf16* W_k, const gqe_bf16* W_v, const gqe_bf16* W_o,
                           gqe_bf16* K_cache, gqe_bf16* V_cache, int32_t cache_capacity, gqe_bf16* y,
                           void* ws, size_t ws_bytes, gqe_stream_t stream) {
  if (cfg == nullptr || cfg->T < 1) return GQE_ERR_INVALID;
  const gqe_config c1 = decode_rows_cfg(*cfg);
  const gqe_status s = check_cfg(&c1);  // B rows; the long extent is the cache
  if (s != GQE_OK) return s;
  if ((cfg->flags & (kOutFlags | GQE_FLAG_NO_SHARED_HEAD)) != 0u)
    return GQE_ERR_UNSUPPORTED;  // default construction only
  if (cache_capacity < cfg->T) return GQE_ERR_INVALID;
  if (!all_aligned(x, W_r, W_q, W_qs, W_k, W_v, W_o, K_cache, V_cache, y) || ws == nullptr ||
      !aligned16(ws))
    return GQE_ERR_INVALID;
  if (b_r != nullptr && (reinterpret_cast<uintptr_t>(b_r) & 3u)) return GQE_ERR_INVALID;
  if (decode_heads(*cfg, false) > 16 || cfg->B > 65535) return GQE_ERR_UNSUPPORTED;
  const DecodeWs D = decode_ws(*cfg);
  if (ws_bytes < D.total) return GQE_ERR_WORKSPACE;
  const LayerWs& L = D.L1;
  char* w = static_cast<char*>(ws);
  auto I = [&](size_t o) { return reinterpret_cast<int32_t*>(w + o); };
  auto F = [&](size_t o) { return reinterpret_cast<float*>(w + o); };
  auto H = [&](size_t o) { return reinterpret_cast<gqe_bf16*>(w + o); };
  gqe_status st = gqe_router_topk(&c1, x, W_r, b_r, I(L.idx), F(L.r), F(L.omega), stream);
  if (st != GQE_OK) return st;
  st = gqe_dispatch(&c1, I(L.idx), x, W_q, W_qs, I(L.counts), I(L.offsets), I(L.tok),
                    I(L.slot_pos), H(L.Qv), H(L.Qs), w + L.dws, L.aws - L.dws, stream);
  if (st != GQE_OK) return st;
  if (gemm_kv_at(c1, x, W_k, W_v, K_cache, V_cache, cache_capacity, cfg->T - 1, stream) != cudaSuccess)
    return GQE_ERR_CUDA;
  if (decode_attention(*cfg, false, H(L.Qv), H(L.Qs), K_cache, V_cache, cache_capacity, H(L.slots),
                       (cfg->G * cfg->k + 2) * cfg->d_head, w + D.daws, stream) != cudaSuccess)
    return GQE_ERR_CUDA;
  return gqe_output_proj(&c1, H(L.slots), F(L.omega), W_o, y, stream);
}

gqe_status gqa_dense_decode_step(const gqe_config* cfg, const gqe_bf16* x, const gqe_bf16* W_q,
                                 const gqe_bf16* W_k, const gqe_bf16* W_v,
                                 const gqe_bf16* W_o_dense, gqe_bf16* K_cache, gqe_bf16* V_cache,
                                 int32_t cache_capacity, gqe_bf16* y, void* ws, size_t ws_bytes,
                                 gqe_stream_t stream) {
  if (cfg == nullptr) return GQE_ERR_INVALID;
  gqe_config c = *cfg;
  c.k = 1;  // not used by the dense layer
  if (c.T < 1) return GQE_ERR_INVALID;
  const gqe_config c1 = decode_rows_cfg(c);
  const gqe_status s = check_cfg(&c1);  // B rows; the long extent is the cache
  if (s != GQE_OK) return s;
  if (cache_capacity < c.T) return GQE_ERR_INVALID;
  if (!all_aligned(x, W_q, W_k, W_v, W_o_dense, K_cache, V_cache, y) || ws == nullptr ||
      !aligned16(ws))
    return GQE_ERR_INVALID;
  if (decode_heads(c, true) > 16 || c.B > 65535) return GQE_ERR_UNSUPPORTED;
  const DenseDecodeWs D = dense_decode_ws(c);
  if (ws_bytes < D.total) return GQE_ERR_WORKSPACE;
  char* w = static_cast<char*>(ws);
  auto H = [&](size_t o) { return reinterpret_cast<gqe_bf16*>(w + o); };
  const int N = c.G * c.M;
  int e = gemm_q_dense(c1, x, W_q, H(D.Q), stream);
  if (e == cudaSuccess) e = gemm_kv_at(c1, x, W_k, W_v, K_cache, V_cache, cache_capacity, c.T - 1, stream);
  if (e == cudaSuccess)
    e = decode_attention(c, true, H(D.Q), nullptr, K_cache, V_cache, cache_capacity, H(D.O),
                         N * c.d_head, w + D.daws, stream);
  if (e != cudaSuccess) return GQE_ERR_CUDA;
  return cuda_status(gemm_rowmajor(H(D.O), c.B, N * c.d_head, W_o_dense, c.d_model, y, stream));
}
