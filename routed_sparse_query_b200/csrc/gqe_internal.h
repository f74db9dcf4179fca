// Internal declarations shared by the .cu files of libgqe.so.
#pragma once
#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include <atomic>
#include <utility>

#include "gqe.h"

namespace gqe {

// Wall-time bound of every device-side wait (2 s).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Router limits: N = G*M experts (<= 64, G <= 32). The logits are reduced
// over NP = max(4, next power of two >= N) columns (W_r is staged in shared
// memory zero-padded to NP columns); a configuration is supported when the
// router's narrowest block (2 tokens per thread) fits in kRouterSmemLimit.
constexpr int kMaxExperts = 64;
__host__ __device__ constexpr int router_np(int N) {
  return N <= 4 ? 4 : N <= 8 ? 8 : N <= 16 ? 16 : N <= 32 ? 32 : 64;
}
constexpr size_t kRouterSmemLimit = 200 * 1024;

// Output construction (gqe.h, GQE_FLAG_OUT_* / GQE_FLAG_SLOT_GROUP_MEAN):
// whether the layer has the shared head, its query streams (kG routed, plus
// the shared head) and its slots per token (plus the weighted slot).
constexpr uint32_t kOutFlags = GQE_FLAG_SLOT_GROUP_MEAN | GQE_FLAG_OUT_HARD | GQE_FLAG_OUT_WEIGHTED_CONCAT;
inline bool has_weighted_slot(const gqe_config& c) {
  return (c.flags & (GQE_FLAG_OUT_HARD | GQE_FLAG_OUT_WEIGHTED_CONCAT)) == 0u;
}
inline bool has_shared_head(const gqe_config& c) {
  return has_weighted_slot(c) && (c.flags & GQE_FLAG_NO_SHARED_HEAD) == 0u;
}
inline int n_streams(const gqe_config& c) { return c.G * c.k + (has_shared_head(c) ? 1 : 0); }
inline int n_slots(const gqe_config& c) {
  return c.G * c.k + (has_shared_head(c) ? 1 : 0) + (has_weighted_slot(c) ? 1 : 0);
}
// What gqe_router_topk writes to omega: 0 = p over all selected, 1 = r / G,
// 2 = p (the in-group probability).
inline int omega_mode(const gqe_config& c) {
  return (c.flags & GQE_FLAG_SLOT_GROUP_MEAN) ? 1 : (c.flags & GQE_FLAG_OUT_WEIGHTED_CONCAT) ? 2 : 0;
}

// Dispatch tiling: tokens of one sequence are cut into tiles of this size.
constexpr int kDispatchTile = 256;  // == dispatch CTA size: one token per thread
constexpr int kQTileRows = 128;  // rows of one grouped-GEMM tile

struct DispatchWs {
  // Byte offsets inside the dispatch workspace.
  size_t masks;        // uint64 [R]: selection bitmask per token
  size_t tile_counts;  // int32 [N][num_tiles]
  size_t tile_base;    // int32 [N][num_tiles]
  size_t qtiles;       // int4  [max_qtiles]: (e, b, first list entry, rows)
  size_t n_qtiles;     // int32 [1]
  size_t total;
  int num_tiles;
  int tiles_per_seq;
  int max_qtiles;
};
DispatchWs dispatch_ws_layout(const gqe_config& c);

size_t router_smem_bytes(const gqe_config& c);

// Launches `kern` with programmatic dependent launch allowed (the kernel
// overlaps the tail of the previous kernel on the stream; see pdl_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              void* stream, Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Raises the dynamic shared-memory limit of kernel K to `bytes`, once per
// device (the attribute is per device; re-setting it on every launch costs
// host time on short layers).
// Safe to call from several host threads (the attribute may be set twice).
template <auto K>
inline int ensure_smem(int bytes) {
  static std::atomic<int> done[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return cudaFuncSetAttribute(K, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (done[dev].load(std::memory_order_relaxed) >= bytes) return 0;
  const cudaError_t e = cudaFuncSetAttribute(K, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done[dev].store(bytes, std::memory_order_relaxed);
  return e;
}

// Launchers (return cudaError_t as int).
int launch_router(const gqe_config& c, const uint16_t* x, const float* W_r, const float* b_r,
                  int32_t* idx, float* r, float* omega, void* stream);
int launch_dispatch_lists(const gqe_config& c, const int32_t* idx, int32_t* counts,
                          int32_t* offsets, int32_t* tok, int32_t* slot_pos, void* ws,
                          const DispatchWs& L, void* stream);
int launch_weighted_slot(const gqe_config& c, uint16_t* slots, const float* omega, void* stream);
// Weighted concatenation: routed slot (g, s) of every row times omega[row, g, s].
int launch_scale_slots(const gqe_config& c, uint16_t* slots, const float* omega, void* stream);

// GEMM front ends (tcgen05). out layouts are described in gemm.cu.
int gemm_kv(const gqe_config& c, const uint16_t* x, const uint16_t* W_k, const uint16_t* W_v,
            uint16_t* K, uint16_t* V, void* stream);
// Routed query projection over the token lists plus the shared-head query
// projection, in one launch (Qs == nullptr: routed tiles only).
// expert_major: Qv is written in token-list order ([k*G*B*T, dh], row = list
// entry) instead of slot-major [B, G, k, T, dh].
int gemm_q_routed(const gqe_config& c, const uint16_t* x, const uint16_t* W_q, const uint16_t* W_qs,
                  const int32_t* idx, const int32_t* tok, const void* qtiles,
                  const int32_t* n_qtiles, int max_qtiles, uint16_t* Qv, uint16_t* Qs,
                  bool expert_major, void* stream);
// The shared-head query projection alone (Qs [B, T, dh]); the same tiles and
// accumulation order as the shared tiles of gemm_q_routed, so the same bits.
int gemm_q_shared(const gqe_config& c, const uint16_t* x, const uint16_t* W_qs, uint16_t* Qs,
                  void* stream);
int gemm_q_dense(const gqe_config& c, const uint16_t* x, const uint16_t* W_q, uint16_t* Q,
                 void* stream);
int gemm_rowmajor(const uint16_t* A, int rows, int K, const uint16_t* W, int N, uint16_t* out,
                  void* stream);
// Weighted slot + W_O projection (steps a10, a11): y = slots @ W_o, with
// the weighted slot written into slots first (fused into the GEMM when
// d_head is one K block).
int gemm_output(const gqe_config& c, uint16_t* slots, const float* omega, const uint16_t* W_o,
                uint16_t* y, void* stream);

// Attention front ends (tcgen05). Split-KV plan: small problems cut each
// query-tile pair's KV range into chunks; the scratch (partial rows and
// per-pair counters) comes from the workspace (total == 0: no scratch).
struct AttnPlan {
  int n_qt, n_pairs, chunk, items;
  size_t part, ml, counters, counter_bytes, total;
};
AttnPlan attention_plan(const gqe_config& c, int H);
// counters_zeroed: the caller has zeroed the split-KV arrival counters of ws
// earlier on the stream (zero_attention_counters); otherwise the call does.
// lse (optional): each stream's rows' log-sum-exp, base 2 of s log2(e)/sqrt(dh),
// [B*(G*k+1)][T rounded up to 64].
int attention_gqe(const gqe_config& c, const uint16_t* Qv, const uint16_t* Qs, const uint16_t* K,
                  const uint16_t* V, uint16_t* slots, void* ws, size_t ws_bytes,
                  bool counters_zeroed, void* stream, float* lse = nullptr);
// Every expert's queries in one dense GEMM, only the routed rows stored:
// Qv[b][g][s][t] = x[b T + t] W_q[:, e], e = g M + idx[b T + t][g][s].
int gemm_q_all_routed(const gqe_config& c, const uint16_t* x, const uint16_t* W_q, const int32_t* idx,
                      uint16_t* Qv, void* stream);
// K, V and every head's queries in one launch of four outputs (needs
// G*M*dh = 2*G*dh, M = 2). idx non-null: only the routed rows are stored, into
// the slot-major streams Q = Qv (as gemm_q_all_routed); null: every head's
// queries, Q [B][G*M][T][dh] (as gemm_q_dense).
int gemm_kvq(const gqe_config& c, const uint16_t* x, const uint16_t* W_k, const uint16_t* W_v,
             const uint16_t* W_q, const int32_t* idx, uint16_t* K, uint16_t* V, uint16_t* Q, void* stream);
// Expert-major routed attention (Qe in token-list order, rows masked by
// their positions tok[]) plus the shared head, one launch, no scratch.
int attention_gqe_em(const gqe_config& c, const uint16_t* Qe, const uint16_t* Qs, const uint16_t* K,
                     const uint16_t* V, const int32_t* idx, const int32_t* offsets, const int32_t* tok,
                     uint16_t* slots, void* stream);
int attention_dense(const gqe_config& c, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                    uint16_t* O, void* ws, size_t ws_bytes, bool counters_zeroed, void* stream);
int zero_attention_counters(const gqe_config& c, int H, void* ws, void* stream);

// fp32-output tensor-core GEMM (gemm.cu): C[M, N] = A[M, K] B[K, N], A bf16
// K-contiguous (row stride lda), B bf16 N-contiguous (row stride ldb, rows at
// least N rounded up to 64 long); lda, ldb multiples of 8.
int gemm_f32out(const uint16_t* A, long long lda, int M, int K, const uint16_t* B, long long ldb, int N,
                float* C, long long ldc, void* stream);

// Backward of the layer (backward.cu).
template <typename TI>
int bwd_transpose(const TI* in, long long ldi, int rows, int cols, uint16_t* out, long long ldo, void* stream);
int bwd_cast(const float* in, long long ldi, long long rows, int cols, uint16_t* out, long long ldo, void* stream);
int bwd_pack(const gqe_config& c, const float* dQr, const float* dQs, const float* dKp, const float* dVp,
             const float* dz, const int32_t* idx, uint16_t* Y, int ld, void* stream);
// zl: [B*T, G*M] fp32 scratch for the router logits.
int bwd_slots_router(const gqe_config& c, const uint16_t* x, const float* W_r, const float* b_r, float* zl,
                     const int32_t* idx, const float* omega, const uint16_t* slots, const float* dS, float* dOr,
                     float* dOs, float* dz, uint16_t* dO16, float* Drow, void* stream);
// Attention backward on tcgen05 (attn_bwd.cu): dq of every stream, dK and dV
// of every stream (dKp, dVp [B, G*k+1, T, dh]; summed per group by bwd_pack),
// each output in two parts [2][...] (summed by bwd_pack); Drow: D = dO . O;
// lse: the forward attention's row statistics; stats: [B, G*k+1, T rounded
// up to 64] float2 scratch.
int bwd_attention_tc(const gqe_config& c, const uint16_t* Qv, const uint16_t* Qs, const uint16_t* K,
                     const uint16_t* V, const uint16_t* dO16, const float* Drow, const float* lse, float* stats,
                     float* dQr, float* dQs, float* dKp, float* dVp, void* stream);
int bwd_colsum(const float* dz, float* db, long long R, int N, void* stream);

// Decode step. cfg.T = keys after the step (the new token sits at T - 1),
// cap = cache capacity per (sequence, group). K/V projection of the new
// tokens (rows B, one per sequence) written into the cache at position pos.
int gemm_kv_at(const gqe_config& c1, const uint16_t* x, const uint16_t* W_k, const uint16_t* W_v,
               uint16_t* Kc, uint16_t* Vc, int cap, int pos, void* stream);
// Heads per group of the decode attention: k + 1 (GQE, the shared head in
// group 0) or M (dense).
int decode_heads(const gqe_config& c, bool dense);
size_t decode_attention_ws_bytes(const gqe_config& c, bool dense);
// Q: GQE routed queries [B][G][k][dh] (Qs [B][dh]) or dense [B][G*M][dh].
int decode_attention(const gqe_config& c, bool dense, const uint16_t* Q, const uint16_t* Qs,
                     const uint16_t* Kc, const uint16_t* Vc, int cap, uint16_t* out, int ldo,
                     void* ws, void* stream);

}  // namespace gqe
