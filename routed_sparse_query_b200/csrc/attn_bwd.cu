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
// Two kernels, each CTA 128 threads (thread i = TMEM lane i), one elected
// thread of warp 0 issuing TMA loads and UMMAs:
//   attn_bwd_q_kernel, one CTA per 128 query rows of a stream: pass 1 walks
//     the 64-key tiles up to the diagonal, S = Q K^T in TMEM, and takes each
//     row's log-sum-exp (base 2); pass 2 recomputes S, computes dP = dO V^T,
//     writes dS as bf16 over S in TMEM and accumulates dQ += dS K in TMEM.
//     The rows' (lse, D) go to a stats buffer for the second kernel.
//   attn_bwd_kv_kernel, one CTA per 128 keys of a group: for every stream of
//     the group and every 64-query tile from the diagonal on, S^T = K Q^T and
//     dP^T = V dO^T in TMEM, P^T and dS^T written back as bf16, then
//     dV += P^T dO and dK += dS^T Q with the A operand read from TMEM.
// Every output row has one writer and a fixed summation order, so the result
// is deterministic.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cmath>

#include "gqe_internal.h"
#include "ptx.cuh"
#include "tmap.h"

namespace gqe {

namespace attn_bwd_impl {

constexpr int kStages = 3;

template <int DH>
struct Cfg {
  static constexpr int SWB = DH * 2;  // bytes per row = swizzle width
  static constexpr uint32_t LAYOUT = SWB == 128 ? kLayoutSW128 : kLayoutSW64;
  static constexpr int ROWS128 = 128 * DH * 2;
  static constexpr int ROWS64 = 64 * DH * 2;
  static constexpr size_t SMEM = 1024 + 2 * static_cast<size_t>(ROWS128) + 2 * kStages * ROWS64 + 256;
};

struct Params {
  int B, T, G, k, H;     // H = G k + 1 streams per sequence (the shared one last)
  float scale;           // 1 / sqrt(dh)
  float scale_log2;      // log2(e) / sqrt(dh)
  const float* dOr;      // [B*T, G*k, dh] fp32
  const float* dOs;      // [B*T, dh]
  const uint16_t* slots; // [B*T, Sdh]: the forward's attention outputs (stream h = slot h)
  int Sdh;
  float2* stats;         // [B, H, T]: (lse base 2 of s log2(e)/sqrt(dh), D)
  float* dQr;            // [B*T, G*k, dh]
  float* dQs;            // [B*T, dh]
  float* dKf;            // [B*T, G*dh]
  float* dVf;
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float bf16f(uint16_t v) { return __uint_as_float(static_cast<uint32_t>(v) << 16); }

// Waits (bounded) for every TMA load issued into the ring but not consumed,
// so that no copy lands in the shared memory of an exited CTA.
__device__ __forceinline__ void drain_loads(uint64_t* full, int consumed, int issued) {
  volatile int none = 0;
  for (int n = consumed; n < issued; ++n)
    mbar_wait(&full[n % kStages], (n / kStages) & 1, &none, 500000000ull);
}

template <int DH>
__global__ void __launch_bounds__(128) attn_bwd_q_kernel(const __grid_constant__ CUtensorMap tmQv,
                                                         const __grid_constant__ CUtensorMap tmQs,
                                                         const __grid_constant__ CUtensorMap tmK,
                                                         const __grid_constant__ CUtensorMap tmV,
                                                         const __grid_constant__ CUtensorMap tmdO, const Params p) {
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
  uint64_t* s_full = kv_empty + kStages;
  uint64_t* done = s_full + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int gk = p.G * p.k, H = p.H;
  const int nq = (p.T + 127) / 128;
  const int qt = nq - 1 - static_cast<int>(blockIdx.x % nq);  // longest rows first
  const int h = static_cast<int>((blockIdx.x / nq) % H);
  const int b = static_cast<int>(blockIdx.x / (nq * H));
  const int g = h < gk ? h / p.k : 0;
  const int t0 = qt * 128;
  const int warp = threadIdx.x >> 5;
  const int nkv = min(2 * qt + 2, (p.T + 63) / 64);  // 64-key tiles up to the diagonal
  const int total = 2 * nkv;                          // pass 1, then pass 2

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1u);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kv_full[s], 1u);
      mbar_init(&kv_empty[s], 1u);
    }
    mbar_init(s_full, 1u);
    mbar_init(done, 1u);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tslot, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tS = tmem, tP = tmem + 64, tA = tmem + 128;

  int issued = 0;  // thread 0: ring loads issued
  auto load = [&](int n) -> bool {
    const int s = n % kStages;
    if (!mbar_wait(&kv_empty[s], ((n / kStages) & 1) ^ 1u, abort_flag)) return false;
    const bool second = n >= nkv;
    const int j = second ? n - nkv : n;
    mbar_arrive_expect_tx(&kv_full[s], static_cast<uint32_t>(C::ROWS64 * (second ? 2 : 1)));
    tma_load_3d(sK + s * C::ROWS64, &tmK, &kv_full[s], 0, 64 * j, b * p.G + g);
    if (second) tma_load_3d(sV + s * C::ROWS64, &tmV, &kv_full[s], 0, 64 * j, b * p.G + g);
    issued = n + 1;
    return true;
  };
  if (threadIdx.x == 0) {
    prefetch_tmap(h < gk ? &tmQv : &tmQs);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmdO);
    mbar_arrive_expect_tx(q_full, 2u * C::ROWS128);
    if (h < gk) tma_load_3d(sQ, &tmQv, q_full, 0, t0, b * gk + h);
    else tma_load_3d(sQ, &tmQs, q_full, 0, t0, b);
    tma_load_3d(sdO, &tmdO, q_full, 0, t0, b * H + h);
    for (int n = 0; n < kStages - 1 && n < total; ++n)
      if (!load(n)) break;
  }
  __syncwarp();

  // Row of this thread; D = dO . O from the fp32 gradient and the forward's output.
  const int t = t0 + static_cast<int>(threadIdx.x);
  const bool row_ok = t < p.T;
  const size_t r = static_cast<size_t>(b) * p.T + t;
  float D = 0.0f;
  if (row_ok) {
    const float* dO = h < gk ? p.dOr + (r * gk + h) * DH : p.dOs + r * DH;
    const uint16_t* O = p.slots + r * p.Sdh + static_cast<size_t>(h) * DH;
#pragma unroll 8
    for (int c = 0; c < DH; ++c) D = fmaf(dO[c], bf16f(O[c]), D);
  }
  const float sl = p.scale_log2;
  float m2 = -INFINITY, l = 0.0f, lse = 0.0f;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;

  constexpr uint32_t idS = idesc_bf16_f32(128, 64, 0, 0);
  constexpr uint32_t idQ = idesc_bf16_f32(128, DH, 0, 1);
  const uint64_t dQd = smem_desc(smem_u32(sQ), 16, 8 * C::SWB, C::LAYOUT);
  const uint64_t ddO = smem_desc(smem_u32(sdO), 16, 8 * C::SWB, C::LAYOUT);
  const uint64_t dKk = smem_desc(smem_u32(sK), 16, 8 * C::SWB, C::LAYOUT);
  const uint64_t dVk = smem_desc(smem_u32(sV), 16, 8 * C::SWB, C::LAYOUT);
  const uint64_t dKn = smem_desc(smem_u32(sK), C::ROWS64, 8 * C::SWB, C::LAYOUT);  // K as an MN-major B

  bool ok = true;
  int n = 0;
  for (; n < total; ++n) {
    const bool second = n >= nkv;
    const int j = second ? n - nkv : n;
    const int s = n % kStages;
    const uint64_t ko = static_cast<uint64_t>((s * C::ROWS64) >> 4);
    if (warp == 0) {
      const bool w = __all_sync(0xffffffffu, (n > 0 || mbar_wait(q_full, 0, abort_flag)) &&
                                                 mbar_wait(&kv_full[s], (n / kStages) & 1, abort_flag));
      if (w) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) umma_bf16_ss_elect(tS, dQd + 2 * kk, dKk + ko + 2 * kk, idS, kk > 0);
        if (second) {
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk)
            umma_bf16_ss_elect(tP, ddO + 2 * kk, dVk + ko + 2 * kk, idS, kk > 0);
        } else {
          umma_commit_elect(&kv_empty[s]);
        }
        umma_commit_elect(s_full);
      }
    }
    if (!__syncthreads_and(mbar_wait(s_full, n & 1, abort_flag))) {
      ok = false;
      break;
    }
    tc_fence_after();
    if (threadIdx.x == 0 && n + kStages - 1 < total) load(n + kStages - 1);
    __syncwarp();
    const int u0 = 64 * j;
    // Two halves of 32 keys; in pass 2 the bf16 dS of a half goes over S
    // columns that half has already read.
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      uint32_t va[32];
      tmem_ld32(tS + lane_base + 32 * hf, va);
      const int ub = u0 + 32 * hf;
      if (!second) {
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (ub + c <= t) mx = fmaxf(mx, __uint_as_float(va[c]) * sl);
        if (mx > -INFINITY) {
          const float mn = fmaxf(m2, mx);
          float sum = 0.0f;
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (ub + c <= t) sum += ex2f(__uint_as_float(va[c]) * sl - mn);
          l = (m2 == -INFINITY ? 0.0f : l * ex2f(m2 - mn)) + sum;
          m2 = mn;
        }
      } else {
        uint32_t pa[32], w[16];
        tmem_ld32(tP + lane_base + 32 * hf, pa);
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          float ds[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float P = (ub + c + e <= t) ? ex2f(__uint_as_float(va[c + e]) * sl - lse) : 0.0f;
            ds[e] = P * (__uint_as_float(pa[c + e]) - D);
          }
          w[c / 2] = pack_bf16x2(ds[0], ds[1]);
        }
        tmem_st16(tS + lane_base + 16 * hf, w);  // keys 32hf..32hf+31 -> columns 16hf..16hf+15
      }
    }
    if (!second && j == nkv - 1) lse = m2 + log2f(l);
    if (second) tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == 0 && second) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        umma_bf16_ts_elect(tA, tS + kk * 8, dKn + ko + (kk * 16 * C::SWB) / 16, idQ, (j > 0 || kk > 0) ? 1u : 0u);
      umma_commit_elect(&kv_empty[s]);
    }
  }
  if (warp == 0) umma_commit_elect(done);
  const bool have = __syncthreads_and(ok && mbar_wait(done, 0, abort_flag));
  tc_fence_after();
  if (have) {
#pragma unroll
    for (int cc = 0; cc < DH / 32; ++cc) {
      uint32_t v[32];
      tmem_ld32(tA + lane_base + cc * 32, v);
      if (row_ok) {
        float* dq = h < gk ? p.dQr + (r * gk + h) * DH : p.dQs + r * DH;
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4)
          reinterpret_cast<float4*>(dq + cc * 32)[c4] =
              make_float4(__uint_as_float(v[4 * c4]) * p.scale, __uint_as_float(v[4 * c4 + 1]) * p.scale,
                          __uint_as_float(v[4 * c4 + 2]) * p.scale, __uint_as_float(v[4 * c4 + 3]) * p.scale);
      }
    }
    if (row_ok) p.stats[(static_cast<size_t>(b) * H + h) * p.T + t] = make_float2(lse, D);
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && !have) {
    volatile int none = 0;
    mbar_wait(q_full, 0, &none, 500000000ull);
    drain_loads(kv_full, n, issued);
  }
  if (warp == 0) {
    if (!have) {
      volatile int none = 0;
      mbar_wait(done, 0, &none, 500000000ull);
    }
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int DH>
__global__ void __launch_bounds__(128) attn_bwd_kv_kernel(const __grid_constant__ CUtensorMap tmQv,
                                                          const __grid_constant__ CUtensorMap tmQs,
                                                          const __grid_constant__ CUtensorMap tmK,
                                                          const __grid_constant__ CUtensorMap tmV,
                                                          const __grid_constant__ CUtensorMap tmdO, const Params p) {
  using C = Cfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sK = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sV = sK + C::ROWS128;
  uint8_t* sQ = sV + C::ROWS128;
  uint8_t* sdO = sQ + kStages * C::ROWS64;
  uint64_t* kv_full = reinterpret_cast<uint64_t*>(sdO + kStages * C::ROWS64);
  uint64_t* q_full = kv_full + 1;
  uint64_t* q_empty = q_full + kStages;
  uint64_t* s_full = q_empty + kStages;
  uint64_t* done = s_full + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int gk = p.G * p.k, H = p.H;
  const int nk = (p.T + 127) / 128;
  const int kb = static_cast<int>(blockIdx.x % nk);  // longest key ranges first
  const int g = static_cast<int>((blockIdx.x / nk) % p.G);
  const int b = static_cast<int>(blockIdx.x / (nk * p.G));
  const int u0 = kb * 128;
  const int warp = threadIdx.x >> 5;
  const int nq64 = (p.T + 63) / 64;
  const int per = nq64 - 2 * kb;                 // 64-query tiles from the diagonal on
  const int nstreams = p.k + (g == 0 ? 1 : 0);   // the group's routed slots, and the shared head in group 0
  const int total = nstreams * per;
  auto stream_of = [&](int si) { return si < p.k ? g * p.k + si : gk; };

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1u);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&q_full[s], 1u);
      mbar_init(&q_empty[s], 1u);
    }
    mbar_init(s_full, 1u);
    mbar_init(done, 1u);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tslot, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tS = tmem, tP = tmem + 64, tK = tmem + 128, tV = tmem + 192;

  int issued = 0;
  auto load = [&](int n) -> bool {
    const int s = n % kStages;
    if (!mbar_wait(&q_empty[s], ((n / kStages) & 1) ^ 1u, abort_flag)) return false;
    const int hh = stream_of(n / per);
    const int j = 2 * kb + n % per;
    mbar_arrive_expect_tx(&q_full[s], 2u * C::ROWS64);
    if (hh < gk) tma_load_3d(sQ + s * C::ROWS64, &tmQv, &q_full[s], 0, 64 * j, b * gk + hh);
    else tma_load_3d(sQ + s * C::ROWS64, &tmQs, &q_full[s], 0, 64 * j, b);
    tma_load_3d(sdO + s * C::ROWS64, &tmdO, &q_full[s], 0, 64 * j, b * H + hh);
    issued = n + 1;
    return true;
  };
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmQv);
    prefetch_tmap(&tmQs);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmdO);
    mbar_arrive_expect_tx(kv_full, 2u * C::ROWS128);
    tma_load_3d(sK, &tmK, kv_full, 0, u0, b * p.G + g);
    tma_load_3d(sV, &tmV, kv_full, 0, u0, b * p.G + g);
    for (int n = 0; n < kStages - 1 && n < total; ++n)
      if (!load(n)) break;
  }
  __syncwarp();

  const int u = u0 + static_cast<int>(threadIdx.x);  // key row of this thread
  const float sl = p.scale_log2;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  constexpr uint32_t idS = idesc_bf16_f32(128, 64, 0, 0);
  constexpr uint32_t idO = idesc_bf16_f32(128, DH, 0, 1);
  const uint64_t dKk = smem_desc(smem_u32(sK), 16, 8 * C::SWB, C::LAYOUT);
  const uint64_t dVk = smem_desc(smem_u32(sV), 16, 8 * C::SWB, C::LAYOUT);
  const uint64_t dQk = smem_desc(smem_u32(sQ), 16, 8 * C::SWB, C::LAYOUT);
  const uint64_t ddOk = smem_desc(smem_u32(sdO), 16, 8 * C::SWB, C::LAYOUT);
  const uint64_t dQn = smem_desc(smem_u32(sQ), C::ROWS64, 8 * C::SWB, C::LAYOUT);   // Q as an MN-major B
  const uint64_t ddOn = smem_desc(smem_u32(sdO), C::ROWS64, 8 * C::SWB, C::LAYOUT);

  bool ok = true;
  int n = 0;
  for (; n < total; ++n) {
    const int hh = stream_of(n / per);
    const int j = 2 * kb + n % per;
    const int s = n % kStages;
    const uint64_t qo = static_cast<uint64_t>((s * C::ROWS64) >> 4);
    if (warp == 0) {
      const bool w = __all_sync(0xffffffffu, (n > 0 || mbar_wait(kv_full, 0, abort_flag)) &&
                                                 mbar_wait(&q_full[s], (n / kStages) & 1, abort_flag));
      if (w) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) umma_bf16_ss_elect(tS, dKk + 2 * kk, dQk + qo + 2 * kk, idS, kk > 0);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) umma_bf16_ss_elect(tP, dVk + 2 * kk, ddOk + qo + 2 * kk, idS, kk > 0);
        umma_commit_elect(s_full);
      }
    }
    if (!__syncthreads_and(mbar_wait(s_full, n & 1, abort_flag))) {
      ok = false;
      break;
    }
    tc_fence_after();
    if (threadIdx.x == 0 && n + kStages - 1 < total) load(n + kStages - 1);
    __syncwarp();
    const float2* st = p.stats + (static_cast<size_t>(b) * H + hh) * p.T + 64 * j;
    const int tq0 = 64 * j;
    // Two halves of 32 queries: P^T over S^T and dS^T over dP^T, each half
    // written over columns it has already read.
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      uint32_t va[32], pa[32], pw[16], dw[16];
      tmem_ld32(tS + lane_base + 32 * hf, va);
      tmem_ld32(tP + lane_base + 32 * hf, pa);
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        float pv[2], dv[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int cc = 32 * hf + c + e;
          const int tq = tq0 + cc;
          float P = 0.0f, dS = 0.0f;
          if (u <= tq && tq < p.T) {
            const float2 ld = __ldg(st + cc);
            P = ex2f(__uint_as_float(va[c + e]) * sl - ld.x);
            dS = P * (__uint_as_float(pa[c + e]) - ld.y);
          }
          pv[e] = P;
          dv[e] = dS;
        }
        pw[c / 2] = pack_bf16x2(pv[0], pv[1]);
        dw[c / 2] = pack_bf16x2(dv[0], dv[1]);
      }
      tmem_st16(tS + lane_base + 16 * hf, pw);  // queries 32hf.. -> columns 16hf..
      tmem_st16(tP + lane_base + 16 * hf, dw);
    }
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        umma_bf16_ts_elect(tV, tS + kk * 8, ddOn + qo + (kk * 16 * C::SWB) / 16, idO, (n > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        umma_bf16_ts_elect(tK, tP + kk * 8, dQn + qo + (kk * 16 * C::SWB) / 16, idO, (n > 0 || kk > 0) ? 1u : 0u);
      umma_commit_elect(&q_empty[s]);
    }
  }
  if (warp == 0) umma_commit_elect(done);
  const bool have = __syncthreads_and(ok && total > 0 && mbar_wait(done, 0, abort_flag));
  tc_fence_after();
  if (have) {
    const bool row_ok = u < p.T;
    const size_t o = (static_cast<size_t>(b) * p.T + u) * p.G * DH + static_cast<size_t>(g) * DH;
#pragma unroll
    for (int cc = 0; cc < DH / 32; ++cc) {
      uint32_t vk[32], vv[32];
      tmem_ld32(tK + lane_base + cc * 32, vk);
      tmem_ld32(tV + lane_base + cc * 32, vv);
      if (row_ok) {
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          reinterpret_cast<float4*>(p.dKf + o + cc * 32)[c4] =
              make_float4(__uint_as_float(vk[4 * c4]) * p.scale, __uint_as_float(vk[4 * c4 + 1]) * p.scale,
                          __uint_as_float(vk[4 * c4 + 2]) * p.scale, __uint_as_float(vk[4 * c4 + 3]) * p.scale);
          reinterpret_cast<float4*>(p.dVf + o + cc * 32)[c4] =
              make_float4(__uint_as_float(vv[4 * c4]), __uint_as_float(vv[4 * c4 + 1]),
                          __uint_as_float(vv[4 * c4 + 2]), __uint_as_float(vv[4 * c4 + 3]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && !have) {
    volatile int none = 0;
    mbar_wait(kv_full, 0, &none, 500000000ull);
    drain_loads(q_full, n, issued);
  }
  if (warp == 0) {
    if (!have) {
      volatile int none = 0;
      mbar_wait(done, 0, &none, 500000000ull);
    }
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int DH>
int launch_bwd(const gqe_config& c, const uint16_t* Qv, const uint16_t* Qs, const uint16_t* K, const uint16_t* V,
               const uint16_t* dO16, const Params& p, void* stream) {
  using Cf = Cfg<DH>;
  const int gk = c.G * c.k, H = gk + 1;
  CUtensorMap q128, s128, k64, v64, o128, q64, s64, k128, v128, o64;
  const bool maps = make_tmap_bf16_3d(&q128, Qv, DH, c.T, static_cast<uint64_t>(c.B) * gk, DH, 128) &&
                    make_tmap_bf16_3d(&s128, Qs, DH, c.T, c.B, DH, 128) &&
                    make_tmap_bf16_3d(&k64, K, DH, c.T, static_cast<uint64_t>(c.B) * c.G, DH, 64) &&
                    make_tmap_bf16_3d(&v64, V, DH, c.T, static_cast<uint64_t>(c.B) * c.G, DH, 64) &&
                    make_tmap_bf16_3d(&o128, dO16, DH, c.T, static_cast<uint64_t>(c.B) * H, DH, 128) &&
                    make_tmap_bf16_3d(&q64, Qv, DH, c.T, static_cast<uint64_t>(c.B) * gk, DH, 64) &&
                    make_tmap_bf16_3d(&s64, Qs, DH, c.T, c.B, DH, 64) &&
                    make_tmap_bf16_3d(&k128, K, DH, c.T, static_cast<uint64_t>(c.B) * c.G, DH, 128) &&
                    make_tmap_bf16_3d(&v128, V, DH, c.T, static_cast<uint64_t>(c.B) * c.G, DH, 128) &&
                    make_tmap_bf16_3d(&o64, dO16, DH, c.T, static_cast<uint64_t>(c.B) * H, DH, 64);
  if (!maps) return cudaErrorInvalidValue;
  const long long nq = (c.T + 127) / 128;
  const long long q_ctas = static_cast<long long>(c.B) * H * nq;
  const long long kv_ctas = static_cast<long long>(c.B) * c.G * nq;
  if (q_ctas > 0x7fffffffll || kv_ctas > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  int e = ensure_smem<attn_bwd_q_kernel<DH>>(static_cast<int>(Cf::SMEM));
  if (e == cudaSuccess) e = ensure_smem<attn_bwd_kv_kernel<DH>>(static_cast<int>(Cf::SMEM));
  if (e != cudaSuccess) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  attn_bwd_q_kernel<DH><<<static_cast<unsigned>(q_ctas), 128, Cf::SMEM, st>>>(q128, s128, k64, v64, o128, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_bwd_kv_kernel<DH><<<static_cast<unsigned>(kv_ctas), 128, Cf::SMEM, st>>>(q64, s64, k128, v128, o64, p);
  return cudaGetLastError();
}

}  // namespace attn_bwd_impl

int bwd_attention_tc(const gqe_config& c, const uint16_t* Qv, const uint16_t* Qs, const uint16_t* K,
                     const uint16_t* V, const uint16_t* dO16, const float* dOr, const float* dOs,
                     const uint16_t* slots, float* stats, float* dQr, float* dQs, float* dKf, float* dVf,
                     void* stream) {
  using namespace attn_bwd_impl;
  const int gk = c.G * c.k;
  Params p{c.B, c.T, c.G, c.k, gk + 1,
           static_cast<float>(1.0 / std::sqrt(static_cast<double>(c.d_head))),
           static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(c.d_head))),
           dOr, dOs, slots, (gk + 2) * c.d_head, reinterpret_cast<float2*>(stats), dQr, dQs, dKf, dVf};
  switch (c.d_head) {
    case 64: return launch_bwd<64>(c, Qv, Qs, K, V, dO16, p, stream);
    case 32: return launch_bwd<32>(c, Qv, Qs, K, V, dO16, p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gqe
