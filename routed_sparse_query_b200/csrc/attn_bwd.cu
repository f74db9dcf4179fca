// Causal attention backward on tcgen05 for the routed and shared streams of
// the GQE layer (the gradient of steps a8, a9). For one stream with queries
// q_t, the group's keys k_u and values v_u (u <= t), scores
// s_tu = q_t . k_u / sqrt(dh), P = softmax_u(s), O = P V, and the upstream
// gradient dO:
//   dP_tu = dO_t . v_u,  D_t = dO_t . O_t,  dS_tu = P_tu (dP_tu - D_t),
//   dq_t = sum_u dS_tu k_u / sqrt(dh),  dk_u = sum_t dS_tu q_t / sqrt(dh),
//   dv_u = sum_t P_tu dO_t
// (the plain derivative of softmax attention; the pages state the forward,
// "every selected query expert attends to its group's keys and values":
// gist.science Technical Summary, "Grouped Attention").
//
// Two kernels, each CTA 16 compute warps and one issuing warp. Compute warp w
// serves TMEM lanes 32 (w % 4) .. (one row each) and column quarter w / 4 of
// every 64-column tile; the issuing warp (one elected thread) runs the TMA
// loads and the UMMAs and waits on the compute warps only through mbarriers,
// so no tile's math waits for an issue. The S / dP products of tiles n + 1
// and n + 2 go into two more of three TMEM buffers while the compute warps
// work on tile n.
//   attn_bwd_q_kernel, two CTAs per 128 query rows of a stream (each half
//     of the 64-key tiles up to the diagonal): S = Q K^T and dP = dO V^T, P
//     from the row's log-sum-exp (kept by the forward), dS in bf16 over S,
//     and dQ += dS K (A from TMEM). The rows' (lse, D) go to a stats buffer
//     for the second kernel.
//   attn_bwd_kv_kernel, two CTAs per 128 keys of one stream (each half of the
//     64-query tiles from the diagonal on): S^T = K Q^T and dP^T = V dO^T,
//     P^T and dS^T written back in bf16, then dV += P^T dO and dK += dS^T Q.
// Each CTA writes its own part of dQ, dK, dV; the parts, and dK, dV over a
// group's streams, are summed later in a fixed order, so the result is
// deterministic.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cmath>

#include "gqe_internal.h"
#include "ptx.cuh"
#include "tmap.h"

namespace gqe {

namespace attn_bwd_impl {

constexpr int kBufs = 3;      // TMEM S / dP buffers: products issued kBufs - 1 tiles ahead of their use
constexpr int kStages = 6;    // ring of 64-row tiles
constexpr int kAhead = 3;     // loads issued this many tiles ahead of their use; a stage is reloaded
                              // only after the tile kStages - kAhead before it, whose UMMAs precede
                              // the products the threads have just waited for
constexpr int kCompute = 512;             // 16 compute warps: 4 column quarters x 4 lane quarters
constexpr int kIssuer = kCompute / 32;     // warp 16: TMA loads and UMMA issue
constexpr int kThreads = kCompute + 32;

template <int DH>
struct Cfg {
  static constexpr int SWB = DH * 2;  // bytes per row = swizzle width
  static constexpr uint32_t LAYOUT = SWB == 128 ? kLayoutSW128 : kLayoutSW64;
  static constexpr int ROWS128 = 128 * DH * 2;
  static constexpr int ROWS64 = 64 * DH * 2;
  // Ring stage of the key kernel: Q and dO tiles of 64 rows, then the 64
  // rows' (lse, D) (512 bytes, padded to keep the next stage 1024-aligned).
  static constexpr int KV_STAGE = 2 * ROWS64 + 1024;
  static constexpr size_t SMEM_Q = 1024 + 2 * static_cast<size_t>(ROWS128) + 2 * kStages * ROWS64 + 256;
  static constexpr size_t SMEM_KV = 1024 + 2 * static_cast<size_t>(ROWS128) + kStages * KV_STAGE + 256;
};

struct Params {
  int B, T, Tp, G, k, H;  // Tp: T rounded up to 64 (row stride of stats); H = G k + 1 streams
  float scale;            // 1 / sqrt(dh)
  float scale_log2;       // log2(e) / sqrt(dh)
  const float* Drow;      // [B, H, Tp]: D = dO . O of each row
  const float* lse;       // [B, H, Tp]: each row's log-sum-exp (base 2 of s log2(e)/sqrt(dh)), from the forward
  float2* stats;          // [B, H, Tp]: (lse, D) for the key kernel
  // Outputs in two parts [2][...], one per half of a CTA pair's tiles.
  float* dQr;             // [2][B*T, G*k, dh]
  float* dQs;             // [2][B*T, dh]
  float* dKp;             // [2][B, H, T, dh]: dK of each stream
  float* dVp;
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float bf16f(uint16_t v) { return __uint_as_float(static_cast<uint32_t>(v) << 16); }

// Waits (bounded) for the last loads issued into the ring (at most kAhead
// are ever ahead of their use), so that no copy lands in the shared memory of
// an exited CTA.
__device__ __forceinline__ void drain_loads(uint64_t* full, int issued) {
  volatile int none = 0;
  for (int n = issued > kAhead ? issued - kAhead : 0; n < issued; ++n)
    mbar_wait(&full[n % kStages], (n / kStages) & 1, &none, 500000000ull);
}

// Named barriers over the compute warps only (the issuing warp never waits
// on them): a plain barrier, and one that returns whether pred held in every
// thread.
__device__ __forceinline__ void compute_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kCompute) : "memory"); }
__device__ __forceinline__ bool compute_all(bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred p, 2, %2, p;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(out)
      : "r"(static_cast<uint32_t>(pred)), "n"(kCompute)
      : "memory");
  return out != 0u;
}

template <int DH>
__device__ __forceinline__ void store_rows32(float* dst, const uint32_t (&v)[32], float scale) {
#pragma unroll
  for (int c4 = 0; c4 < 8; ++c4)
    reinterpret_cast<float4*>(dst)[c4] =
        make_float4(__uint_as_float(v[4 * c4]) * scale, __uint_as_float(v[4 * c4 + 1]) * scale,
                    __uint_as_float(v[4 * c4 + 2]) * scale, __uint_as_float(v[4 * c4 + 3]) * scale);
}

template <int DH>
__global__ void __launch_bounds__(kThreads, 1) attn_bwd_q_kernel(const __grid_constant__ CUtensorMap tmQv,
                                                                 const __grid_constant__ CUtensorMap tmQs,
                                                                 const __grid_constant__ CUtensorMap tmK,
                                                                 const __grid_constant__ CUtensorMap tmV,
                                                                 const __grid_constant__ CUtensorMap tmdO,
                                                                 const Params p) {
  using C = Cfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sQ = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sdO = sQ + C::ROWS128;
  uint8_t* sK = sdO + C::ROWS128;
  uint8_t* sV = sK + kStages * C::ROWS64;
  uint64_t* q_full = reinterpret_cast<uint64_t*>(sV + kStages * C::ROWS64);
  uint64_t* kv_full = q_full + 1;
  uint64_t* kv_empty = kv_full + kStages;
  uint64_t* s_full = kv_empty + kStages;  // [kBufs]: S, dP of a tile in TMEM
  uint64_t* p_ready = s_full + kBufs;     // [kBufs]: its dS in TMEM (one arrival per compute warp)
  uint64_t* done = p_ready + kBufs;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int gk = p.G * p.k, H = p.H;
  const int nq = (p.T + 127) / 128;
  // Two CTAs per (stream, query tile), each taking half of its key tiles.
  const int part = static_cast<int>(blockIdx.x & 1);
  const int rest = static_cast<int>(blockIdx.x >> 1);
  const int qt = nq - 1 - rest % nq;  // longest rows first
  const int h = (rest / nq) % H;
  const int b = rest / (nq * H);
  const int g = h < gk ? h / p.k : 0;
  const int t0 = qt * 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = min(2 * qt + 2, (p.T + 63) / 64);  // 64-key tiles up to the diagonal
  const int mid = (ntiles + 1) / 2;
  const int j0 = part ? mid : 0;
  const int total = part ? ntiles - mid : mid;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1u);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kv_full[s], 1u);
      mbar_init(&kv_empty[s], 1u);
    }
    for (int i = 0; i < kBufs; ++i) {
      mbar_init(&s_full[i], 1u);
      mbar_init(&p_ready[i], kCompute / 32);
    }
    mbar_init(done, 1u);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tA = tmem + 384;  // dQ accumulator; S / dP buffers at 128 (n % kBufs), +64
  int issued = 0;                  // issuer lane 0: ring loads issued
  bool ok = true;

  if (warp == kIssuer) {
    // ---------------------------------------------------------------- issuer
    auto load = [&](int n) -> bool {
      const int s = n % kStages;
      if (!mbar_wait(&kv_empty[s], ((n / kStages) & 1) ^ 1u, abort_flag)) return false;
      mbar_arrive_expect_tx(&kv_full[s], 2u * C::ROWS64);
      tma_load_3d(sK + s * C::ROWS64, &tmK, &kv_full[s], 0, 64 * (j0 + n), b * p.G + g);
      tma_load_3d(sV + s * C::ROWS64, &tmV, &kv_full[s], 0, 64 * (j0 + n), b * p.G + g);
      issued = n + 1;
      return true;
    };
    constexpr uint32_t idS = idesc_bf16_f32(128, 64, 0, 0);
    constexpr uint32_t idQ = idesc_bf16_f32(128, DH, 0, 1);
    const uint64_t dQd = smem_desc(smem_u32(sQ), 16, 8 * C::SWB, C::LAYOUT);
    const uint64_t ddO = smem_desc(smem_u32(sdO), 16, 8 * C::SWB, C::LAYOUT);
    const uint64_t dKk = smem_desc(smem_u32(sK), 16, 8 * C::SWB, C::LAYOUT);
    const uint64_t dVk = smem_desc(smem_u32(sV), 16, 8 * C::SWB, C::LAYOUT);
    const uint64_t dKn = smem_desc(smem_u32(sK), C::ROWS64, 8 * C::SWB, C::LAYOUT);  // K as an MN-major B
    // S and dP of key tile n into buffer n % kBufs. Its previous tile's
    // readers are done: the compute warps signalled p_ready for it, and its
    // dQ UMMA was issued before this one.
    auto issue_sdp = [&](int n) -> bool {
      const int s = n % kStages;
      if (!__all_sync(0xffffffffu, (n > 0 || mbar_wait(q_full, 0, abort_flag)) &&
                                       mbar_wait(&kv_full[s], (n / kStages) & 1, abort_flag)))
        return false;
      tc_fence_after();
      const uint32_t tS = tmem + 128 * (n % kBufs);
      const uint64_t ko = static_cast<uint64_t>((s * C::ROWS64) >> 4);
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk) umma_bf16_ss_elect(tS, dQd + 2 * kk, dKk + ko + 2 * kk, idS, kk > 0);
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk)
        umma_bf16_ss_elect(tS + 64, ddO + 2 * kk, dVk + ko + 2 * kk, idS, kk > 0);
      umma_commit_elect(&s_full[n % kBufs]);
      return true;
    };
    if (lane == 0) {
      prefetch_tmap(h < gk ? &tmQv : &tmQs);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmdO);
      if (total > 0) {  // an empty half loads nothing (no copy may outlive the CTA)
        mbar_arrive_expect_tx(q_full, 2u * C::ROWS128);
        if (h < gk) tma_load_3d(sQ, &tmQv, q_full, 0, t0, b * gk + h);
        else tma_load_3d(sQ, &tmQs, q_full, 0, t0, b);
        tma_load_3d(sdO, &tmdO, q_full, 0, t0, b * H + h);
      }
      for (int n = 0; n < kAhead && n < total; ++n)
        if (!load(n)) break;
    }
    __syncwarp();
    for (int n = 0; ok && n < kBufs - 1 && n < total; ++n) ok = issue_sdp(n);
    for (int n = 0; ok && n < total; ++n) {
      // The stage of tile n + kAhead last held tile n + kAhead - kStages,
      // whose dQ UMMA was issued kStages - kAhead iterations ago.
      if (lane == 0 && n + kAhead < total) load(n + kAhead);
      __syncwarp();
      if (!__all_sync(0xffffffffu, mbar_wait(&p_ready[n % kBufs], (n / kBufs) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tS = tmem + 128 * (n % kBufs);
      const uint64_t ko = static_cast<uint64_t>(((n % kStages) * C::ROWS64) >> 4);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        umma_bf16_ts_elect(tA, tS + kk * 8, dKn + ko + (kk * 16 * C::SWB) / 16, idQ, (n > 0 || kk > 0) ? 1u : 0u);
      umma_commit_elect(&kv_empty[n % kStages]);
      if (n + kBufs - 1 < total) ok = issue_sdp(n + kBufs - 1);
    }
    umma_commit_elect(done);
  } else {
    // ---------------------------------------------------------- compute warps
    const int cq = warp >> 2;                // column quarter (16 of the tile's 64 columns)
    const int row = (warp & 3) * 32 + lane;  // TMEM lane = query row in the tile
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int t = t0 + row;
    const bool row_ok = t < p.T;
    const size_t srow = (static_cast<size_t>(b) * H + h) * p.Tp + t;
    const float sl = p.scale_log2;
    const float lse = row_ok ? p.lse[srow] : 0.0f;
    const float D = row_ok ? p.Drow[srow] : 0.0f;
    for (int n = 0; n < total; ++n) {
      if (!compute_all(mbar_wait(&s_full[n % kBufs], (n / kBufs) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tS = tmem + 128 * (n % kBufs);
      const int ub = 64 * (j0 + n) + 16 * cq;  // first key of this thread's columns
      uint32_t va[16], pa[16], w[8];
      tmem_ld16_nowait(tS + lane_base + 16 * cq, va);
      tmem_ld16_nowait(tS + 64 + lane_base + 16 * cq, pa);
      tmem_ld_wait2_16(va, pa);
#pragma unroll
      for (int c = 0; c < 16; c += 2) {
        float ds[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float P = (ub + c + e <= t) ? ex2f(__uint_as_float(va[c + e]) * sl - lse) : 0.0f;
          ds[e] = P * (__uint_as_float(pa[c + e]) - D);
        }
        w[c / 2] = pack_bf16x2(ds[0], ds[1]);
      }
      tc_fence_before();
      compute_sync();  // every read of S and dP done before dS goes over S
      tc_fence_after();
      tmem_st8(tS + lane_base + 8 * cq, w);  // keys 16cq.. -> columns 8cq..
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready[n % kBufs]);
    }
  }
  const bool have = __syncthreads_and(ok && mbar_wait(done, 0, abort_flag));
  tc_fence_after();
  if (warp < kIssuer) {
    const int cq = warp >> 2, row = (warp & 3) * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int t = t0 + row;
    const bool row_ok = t < p.T;
    const size_t r = static_cast<size_t>(b) * p.T + t;
    const size_t srow = (static_cast<size_t>(b) * H + h) * p.Tp + t;
    if (have && cq * 32 < DH) {  // the first DH / 32 column quarters drain 32 dQ columns each
      const size_t R = static_cast<size_t>(p.B) * p.T;
      float* dq = h < gk ? p.dQr + part * R * gk * DH + (r * gk + h) * DH : p.dQs + part * R * DH + r * DH;
      uint32_t v[32];
      if (total > 0) {
        tmem_ld32(tA + lane_base + 32 * cq, v);
      } else {  // no key tiles in this half: its part is zero
#pragma unroll
        for (int c = 0; c < 32; ++c) v[c] = 0u;
      }
      if (row_ok) store_rows32<DH>(dq + 32 * cq, v, p.scale);
    }
    if (have && part == 0 && cq == 0 && row_ok) p.stats[srow] = make_float2(p.lse[srow], p.Drow[srow]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kIssuer && lane == 0 && !have) {
    volatile int none = 0;
    if (total > 0) mbar_wait(q_full, 0, &none, 500000000ull);
    drain_loads(kv_full, issued);
  }
  if (warp == 0) {
    if (!have) {
      volatile int none = 0;
      mbar_wait(done, 0, &none, 500000000ull);
    }
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int DH>
__global__ void __launch_bounds__(kThreads, 1) attn_bwd_kv_kernel(const __grid_constant__ CUtensorMap tmQv,
                                                                  const __grid_constant__ CUtensorMap tmQs,
                                                                  const __grid_constant__ CUtensorMap tmK,
                                                                  const __grid_constant__ CUtensorMap tmV,
                                                                  const __grid_constant__ CUtensorMap tmdO,
                                                                  const Params p) {
  using C = Cfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sK = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sV = sK + C::ROWS128;
  uint8_t* ring = sV + C::ROWS128;  // [kStages] x (Q | dO | (lse, D) x 64)
  uint64_t* kv_full = reinterpret_cast<uint64_t*>(ring + kStages * C::KV_STAGE);
  uint64_t* q_full = kv_full + 1;
  uint64_t* q_empty = q_full + kStages;
  uint64_t* s_full = q_empty + kStages;  // [kBufs]: S^T, dP^T of a tile in TMEM
  uint64_t* p_ready = s_full + kBufs;    // [kBufs]: its P^T, dS^T in TMEM (one arrival per compute warp)
  uint64_t* done = p_ready + kBufs;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int gk = p.G * p.k, H = p.H;
  const int nk = (p.T + 127) / 128;
  // Two CTAs per (stream, key tile), each taking half of its query tiles.
  const int part = static_cast<int>(blockIdx.x & 1);
  const int rest = static_cast<int>(blockIdx.x >> 1);
  const int kb = rest % nk;  // longest query ranges first
  const int h = (rest / nk) % H;
  const int b = rest / (nk * H);
  const int g = h < gk ? h / p.k : 0;
  const int u0 = kb * 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = (p.T + 63) / 64 - 2 * kb;  // 64-query tiles from the diagonal on
  const int mid = (ntiles + 1) / 2;
  const int jq0 = 2 * kb + (part ? mid : 0);  // first query tile of this CTA
  const int total = part ? ntiles - mid : mid;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1u);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&q_full[s], 1u);
      mbar_init(&q_empty[s], 1u);
    }
    for (int i = 0; i < kBufs; ++i) {
      mbar_init(&s_full[i], 1u);
      mbar_init(&p_ready[i], kCompute / 32);
    }
    mbar_init(done, 1u);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tK = tmem + 384, tV = tmem + 448;  // S^T / dP^T buffers at 128 (n % kBufs), +64
  const float2* st_row = p.stats + (static_cast<size_t>(b) * H + h) * p.Tp;
  int issued = 0;  // issuer lane 0: ring loads issued
  bool ok = true;

  if (warp == kIssuer) {
    // ---------------------------------------------------------------- issuer
    auto load = [&](int n) -> bool {
      const int s = n % kStages;
      if (!mbar_wait(&q_empty[s], ((n / kStages) & 1) ^ 1u, abort_flag)) return false;
      const int j = jq0 + n;
      uint8_t* st = ring + s * C::KV_STAGE;
      mbar_arrive_expect_tx(&q_full[s], 2u * C::ROWS64 + 512u);
      if (h < gk) tma_load_3d(st, &tmQv, &q_full[s], 0, 64 * j, b * gk + h);
      else tma_load_3d(st, &tmQs, &q_full[s], 0, 64 * j, b);
      tma_load_3d(st + C::ROWS64, &tmdO, &q_full[s], 0, 64 * j, b * H + h);
      bulk_load(st + 2 * C::ROWS64, st_row + 64 * j, 512u, &q_full[s]);
      issued = n + 1;
      return true;
    };
    constexpr uint32_t idS = idesc_bf16_f32(128, 64, 0, 0);
    constexpr uint32_t idO = idesc_bf16_f32(128, DH, 0, 1);
    const uint64_t dKk = smem_desc(smem_u32(sK), 16, 8 * C::SWB, C::LAYOUT);
    const uint64_t dVk = smem_desc(smem_u32(sV), 16, 8 * C::SWB, C::LAYOUT);
    const uint64_t dRk = smem_desc(smem_u32(ring), 16, 8 * C::SWB, C::LAYOUT);         // Q, dO as K-major B
    const uint64_t dRn = smem_desc(smem_u32(ring), C::ROWS64, 8 * C::SWB, C::LAYOUT);  // Q, dO as MN-major B
    constexpr uint64_t kO = static_cast<uint64_t>(C::ROWS64 >> 4);                      // dO after Q in a stage
    // S^T and dP^T of query tile n into buffer n % kBufs (its previous
    // tile's readers are done, as in the query kernel).
    auto issue_sdp = [&](int n) -> bool {
      const int s = n % kStages;
      if (!__all_sync(0xffffffffu, (n > 0 || mbar_wait(kv_full, 0, abort_flag)) &&
                                       mbar_wait(&q_full[s], (n / kStages) & 1, abort_flag)))
        return false;
      tc_fence_after();
      const uint32_t tS = tmem + 128 * (n % kBufs);
      const uint64_t qo = static_cast<uint64_t>((s * C::KV_STAGE) >> 4);
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk) umma_bf16_ss_elect(tS, dKk + 2 * kk, dRk + qo + 2 * kk, idS, kk > 0);
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk)
        umma_bf16_ss_elect(tS + 64, dVk + 2 * kk, dRk + qo + kO + 2 * kk, idS, kk > 0);
      umma_commit_elect(&s_full[n % kBufs]);
      return true;
    };
    if (lane == 0) {
      prefetch_tmap(h < gk ? &tmQv : &tmQs);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmdO);
      if (total > 0) {  // an empty half loads nothing (no copy may outlive the CTA)
        mbar_arrive_expect_tx(kv_full, 2u * C::ROWS128);
        tma_load_3d(sK, &tmK, kv_full, 0, u0, b * p.G + g);
        tma_load_3d(sV, &tmV, kv_full, 0, u0, b * p.G + g);
      }
      for (int n = 0; n < kAhead && n < total; ++n)
        if (!load(n)) break;
    }
    __syncwarp();
    for (int n = 0; ok && n < kBufs - 1 && n < total; ++n) ok = issue_sdp(n);
    for (int n = 0; ok && n < total; ++n) {
      if (lane == 0 && n + kAhead < total) load(n + kAhead);
      __syncwarp();
      if (!__all_sync(0xffffffffu, mbar_wait(&p_ready[n % kBufs], (n / kBufs) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tS = tmem + 128 * (n % kBufs);
      const uint64_t qo = static_cast<uint64_t>(((n % kStages) * C::KV_STAGE) >> 4);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        umma_bf16_ts_elect(tV, tS + kk * 8, dRn + qo + kO + (kk * 16 * C::SWB) / 16, idO, (n > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        umma_bf16_ts_elect(tK, tS + 64 + kk * 8, dRn + qo + (kk * 16 * C::SWB) / 16, idO, (n > 0 || kk > 0) ? 1u : 0u);
      umma_commit_elect(&q_empty[n % kStages]);
      if (n + kBufs - 1 < total) ok = issue_sdp(n + kBufs - 1);
    }
    umma_commit_elect(done);
  } else {
    // ---------------------------------------------------------- compute warps
    const int cq = warp >> 2;                // column quarter (16 of the tile's 64 columns)
    const int row = (warp & 3) * 32 + lane;  // TMEM lane = key row in the tile
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int u = u0 + row;                  // key of this thread
    const float sl = p.scale_log2;
    for (int n = 0; n < total; ++n) {
      const int s = n % kStages;
      // The stage's (lse, D) are read here too, so its load is waited for as
      // well (complete by now: the products of this tile read the same stage).
      if (!compute_all(mbar_wait(&s_full[n % kBufs], (n / kBufs) & 1, abort_flag) &&
                       mbar_wait(&q_full[s], (n / kStages) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tS = tmem + 128 * (n % kBufs);
      const float2* sst = reinterpret_cast<const float2*>(ring + s * C::KV_STAGE + 2 * C::ROWS64) + 16 * cq;
      const int tq0 = 64 * (jq0 + n) + 16 * cq;  // first query of this thread's columns
      uint32_t va[16], pa[16], pw[8], dw[8];
      tmem_ld16_nowait(tS + lane_base + 16 * cq, va);
      tmem_ld16_nowait(tS + 64 + lane_base + 16 * cq, pa);
      tmem_ld_wait2_16(va, pa);
#pragma unroll
      for (int c = 0; c < 16; c += 2) {
        float pv[2], dv[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int tq = tq0 + c + e;
          float P = 0.0f, dS = 0.0f;
          if (u <= tq && tq < p.T) {  // the stats past T are not written
            const float2 ld = sst[c + e];
            P = ex2f(__uint_as_float(va[c + e]) * sl - ld.x);
            dS = P * (__uint_as_float(pa[c + e]) - ld.y);
          }
          pv[e] = P;
          dv[e] = dS;
        }
        pw[c / 2] = pack_bf16x2(pv[0], pv[1]);
        dw[c / 2] = pack_bf16x2(dv[0], dv[1]);
      }
      tc_fence_before();
      compute_sync();  // every read of S^T and dP^T done before P^T, dS^T go over them
      tc_fence_after();
      tmem_st8(tS + lane_base + 8 * cq, pw);  // queries 16cq.. -> columns 8cq..
      tmem_st8(tS + 64 + lane_base + 8 * cq, dw);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_ready[n % kBufs]);
    }
  }
  const bool have = __syncthreads_and(ok && mbar_wait(done, 0, abort_flag));
  tc_fence_after();
  if (have && warp < 8) {
    // Column quarter 0 drains dK, quarter 1 dV.
    const int cq = warp >> 2, u = u0 + (warp & 3) * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const size_t o = static_cast<size_t>(part) * p.B * H * p.T * DH + ((static_cast<size_t>(b) * H + h) * p.T + u) * DH;
#pragma unroll
    for (int cc = 0; cc < DH / 32; ++cc) {
      uint32_t v[32];
      if (total > 0) {
        tmem_ld32((cq == 0 ? tK : tV) + lane_base + 32 * cc, v);
      } else {  // no query tiles in this half: its part is zero
#pragma unroll
        for (int c = 0; c < 32; ++c) v[c] = 0u;
      }
      if (u < p.T) store_rows32<DH>((cq == 0 ? p.dKp : p.dVp) + o + 32 * cc, v, cq == 0 ? p.scale : 1.0f);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kIssuer && lane == 0 && !have) {
    volatile int none = 0;
    if (total > 0) mbar_wait(kv_full, 0, &none, 500000000ull);
    drain_loads(q_full, issued);
  }
  if (warp == 0) {
    if (!have) {
      volatile int none = 0;
      mbar_wait(done, 0, &none, 500000000ull);
    }
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int DH>
int launch_bwd(const gqe_config& c, const uint16_t* Qv, const uint16_t* Qs, const uint16_t* K, const uint16_t* V,
               const uint16_t* dO16, const Params& p, void* stream) {
  using Cf = Cfg<DH>;
  const int gk = c.G * c.k, H = gk + 1;
  CUtensorMap q128, s128, k64, v64, o128, q64, s64, k128, v128, o64;
  const uint64_t nqv = static_cast<uint64_t>(c.B) * gk, nkv = static_cast<uint64_t>(c.B) * c.G,
                 nst = static_cast<uint64_t>(c.B) * H;
  const bool maps = make_tmap_bf16_3d(&q128, Qv, DH, c.T, nqv, DH, 128) &&
                    make_tmap_bf16_3d(&s128, Qs, DH, c.T, c.B, DH, 128) &&
                    make_tmap_bf16_3d(&k64, K, DH, c.T, nkv, DH, 64) &&
                    make_tmap_bf16_3d(&v64, V, DH, c.T, nkv, DH, 64) &&
                    make_tmap_bf16_3d(&o128, dO16, DH, c.T, nst, DH, 128) &&
                    make_tmap_bf16_3d(&q64, Qv, DH, c.T, nqv, DH, 64) &&
                    make_tmap_bf16_3d(&s64, Qs, DH, c.T, c.B, DH, 64) &&
                    make_tmap_bf16_3d(&k128, K, DH, c.T, nkv, DH, 128) &&
                    make_tmap_bf16_3d(&v128, V, DH, c.T, nkv, DH, 128) &&
                    make_tmap_bf16_3d(&o64, dO16, DH, c.T, nst, DH, 64);
  if (!maps) return cudaErrorInvalidValue;
  // Each CTA allocates all 512 TMEM columns: ask for enough shared memory that
  // no second CTA shares the SM (it would wait in its allocation).
  constexpr int kOneCtaSmem = 120 * 1024;
  const int smem_q = static_cast<int>(Cf::SMEM_Q) > kOneCtaSmem ? static_cast<int>(Cf::SMEM_Q) : kOneCtaSmem;
  const int smem_kv = static_cast<int>(Cf::SMEM_KV) > kOneCtaSmem ? static_cast<int>(Cf::SMEM_KV) : kOneCtaSmem;
  const long long ctas = 2ll * c.B * H * ((c.T + 127) / 128);
  if (ctas > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  int e = ensure_smem<attn_bwd_q_kernel<DH>>(smem_q);
  if (e == cudaSuccess) e = ensure_smem<attn_bwd_kv_kernel<DH>>(smem_kv);
  if (e != cudaSuccess) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  attn_bwd_q_kernel<DH><<<static_cast<unsigned>(ctas), kThreads, smem_q, st>>>(q128, s128, k64, v64, o128, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_bwd_kv_kernel<DH><<<static_cast<unsigned>(ctas), kThreads, smem_kv, st>>>(q64, s64, k128, v128, o64, p);
  return cudaGetLastError();
}

}  // namespace attn_bwd_impl

int bwd_attention_tc(const gqe_config& c, const uint16_t* Qv, const uint16_t* Qs, const uint16_t* K,
                     const uint16_t* V, const uint16_t* dO16, const float* Drow, const float* lse, float* stats,
                     float* dQr, float* dQs, float* dKp, float* dVp, void* stream) {
  using namespace attn_bwd_impl;
  const int gk = c.G * c.k;
  Params p{c.B, c.T, (c.T + 63) / 64 * 64, c.G, c.k, gk + 1,
           static_cast<float>(1.0 / std::sqrt(static_cast<double>(c.d_head))),
           static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(c.d_head))),
           Drow, lse, reinterpret_cast<float2*>(stats), dQr, dQs, dKp, dVp};
  switch (c.d_head) {
    case 64: return launch_bwd<64>(c, Qv, Qs, K, V, dO16, p, stream);
    case 32: return launch_bwd<32>(c, Qv, Qs, K, V, dO16, p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gqe
