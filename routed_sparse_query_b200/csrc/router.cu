// Router (steps a1-a4 of the GQE layer): per-token logits x . W_r + b in
// fp32, softmax inside each of the G groups, top-k per group with ties to the
// lower expert index, and the two renormalisations of the selected
// probabilities. ("Grouped Query Experts: Mixture-of-Experts on GQA
// Self-Attention": router choosing k query-head experts in every GQA group,
// gist.science Technical Summary, Methodology; softmax before top-k inside
// the group, pptc.cn blog section 7.)
//
// One warp per token row. W_r is staged once per CTA in shared memory.
// Lane l owns rows l, l+32, l+64, ... of the dot products and keeps NP
// partial sums; a shuffle reduce-scatter leaves every logit complete on one
// or more lanes, in a fixed order (the result is deterministic).
//
// Exact selection: each fp32 logit carries the bound
//   |z_fp32 - z| <= gamma_h * (||x||_1 * max_i |W_r[i,e]| + |b_e|),
// h = d/32 + 6 roundings on its longest path (d/32 FMAs per lane, 5 shuffle
// adds, the bias add), gamma_h = h u / (1 - h u), u = 2^-24 (Higham,
// "Accuracy and Stability of Numerical Algorithms", 2nd ed., sec. 3.1). A
// group whose top-k decision is not certain under these intervals (computed
// with directed rounding) recomputes its logits in fp64 (products of a bf16
// and an fp32 value are exact in fp64) and decides on those, so the selection
// equals the exact-arithmetic one.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "gqe_internal.h"
#include "ptx.cuh"

namespace gqe {

namespace router_impl {

constexpr int kRouterWarps = 8;

__device__ __forceinline__ float bf16_to_f32(uint16_t v) {
  return __uint_as_float(static_cast<uint32_t>(v) << 16);
}

template <int NP>
__device__ __forceinline__ void reduce_scatter(float (&v)[NP], int lane) {
#pragma unroll
  for (int lvl = 0; lvl < 5; ++lvl) {
    const int off = 16 >> lvl;
    const int cnt = NP >> lvl;
    if (cnt > 1) {
      const int h = cnt / 2;
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < NP / 2; ++i) {
        if (i < h) {
          const float keep = upper ? v[i + h] : v[i];
          const float send = upper ? v[i] : v[i + h];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
    }
  }
}

struct RouterArgs {
  const uint16_t* x;
  const float* W_r;
  const float* b_r;
  int32_t* idx;
  float* r;
  float* omega;
  int R, d, G, M, k, N;
};

template <int NP>
__global__ void __launch_bounds__(kRouterWarps * 32) router_kernel(RouterArgs a) {
  constexpr int S = router_row_floats(NP);
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* Wsm = reinterpret_cast<float*>(smem_raw);                 // [d][S]
  float* wmax = Wsm + static_cast<size_t>(a.d) * S;                 // [NP]
  float* bsm = wmax + NP;                                           // [NP]
  double* zd_all = reinterpret_cast<double*>(bsm + NP);             // [warps][NP]
  float* zf_all = reinterpret_cast<float*>(zd_all + kRouterWarps * NP);  // [max(warps*NP, 256)]

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  pdl_wait();
  pdl_launch_dependents();

  // Stage W_r (zero padded to S columns) and the bias. Rows of 4k floats are
  // copied with 16-byte cp.async so that all loads are in flight at once.
  if ((a.N & 3) == 0) {
    const int cpr = a.N >> 2;  // 16-byte chunks per row
    for (int i = tid; i < a.d * cpr; i += blockDim.x) {
      const int row = i / cpr, c = i - row * cpr;
      cp_async_16(smem_u32(Wsm + row * S + 4 * c), a.W_r + static_cast<size_t>(row) * a.N + 4 * c, 16u);
    }
    cp_async_commit();
  } else {
    for (int i = tid; i < a.d * a.N; i += blockDim.x) {
      const int row = i / a.N, col = i - row * a.N;
      Wsm[row * S + col] = a.W_r[i];
    }
  }
  for (int i = tid; i < a.d * (S - a.N); i += blockDim.x) {
    const int row = i / (S - a.N), col = a.N + i % (S - a.N);
    Wsm[row * S + col] = 0.0f;
  }
  cp_async_wait<0>();
  for (int e = tid; e < NP; e += blockDim.x) bsm[e] = (e < a.N && a.b_r != nullptr) ? a.b_r[e] : 0.0f;
  __syncthreads();
  // max_i |W_r[i, e]|: thread t scans column t % NP over rows t / NP (mod
  // the number of parts), then one thread per column combines the parts.
  {
    constexpr int parts = kRouterWarps * 32 / NP;
    float mx = 0.0f;
    const int col = tid % NP, part = tid / NP;
    for (int row = part; row < a.d; row += parts) mx = fmaxf(mx, fabsf(Wsm[row * S + col]));
    zf_all[tid] = mx;  // zf_all has room for kRouterWarps * 32 floats
    __syncthreads();
    if (tid < NP) {
      float m2 = 0.0f;
      for (int p = 0; p < parts; ++p) m2 = fmaxf(m2, zf_all[p * NP + tid]);
      wmax[tid] = m2;
    }
    __syncthreads();
  }

  double* zd = zd_all + warp * NP;
  float* zf = zf_all + warp * NP;
  const int h = a.d / 32 + 6;
  const float u = 5.9604644775390625e-08f;  // 2^-24
  const float gam = (h * u) / (1.0f - h * u);
  const float gam_ru = __fmul_ru(gam, 1.01f);

  const int nwarps_total = gridDim.x * kRouterWarps;
  for (int row = blockIdx.x * kRouterWarps + warp; row < a.R; row += nwarps_total) {
    const uint16_t* xr = a.x + static_cast<size_t>(row) * a.d;
    float acc[NP];
#pragma unroll
    for (int e = 0; e < NP; ++e) acc[e] = 0.0f;
    float nx = 0.0f;
#pragma unroll 8
    for (int m = lane; m < a.d; m += 32) {
      const float xi = bf16_to_f32(xr[m]);
      nx += fabsf(xi);
      const float4* w4 = reinterpret_cast<const float4*>(Wsm + m * S);
#pragma unroll
      for (int q = 0; q < NP / 4; ++q) {
        const float4 w = w4[q];
        acc[4 * q + 0] = fmaf(xi, w.x, acc[4 * q + 0]);
        acc[4 * q + 1] = fmaf(xi, w.y, acc[4 * q + 1]);
        acc[4 * q + 2] = fmaf(xi, w.z, acc[4 * q + 2]);
        acc[4 * q + 3] = fmaf(xi, w.w, acc[4 * q + 3]);
      }
    }
    reduce_scatter<NP>(acc, lane);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) nx += __shfl_xor_sync(0xffffffffu, nx, off);

    // Owner lanes write the logits (+ bias) to the warp's scratch.
    if constexpr (NP >= 32) {
#pragma unroll
      for (int i = 0; i < NP / 32; ++i) {
        const int e = lane * (NP / 32) + i;
        zf[e] = acc[i] + bsm[e];
      }
    } else {
      constexpr int per = 32 / NP;
      if (lane % per == 0) {
        const int e = lane / per;
        zf[e] = acc[0] + bsm[e];
      }
    }
    __syncwarp();

    // Lane g decides group g.
    const int g = lane;
    bool certain = true;
    uint64_t selmask = 0;
    if (g < a.G) {
      const float* zg = zf + g * a.M;
      for (int s = 0; s < a.k; ++s) {
        float best = -INFINITY;
        int bj = -1;
        for (int j = 0; j < a.M; ++j) {
          if (!((selmask >> j) & 1ull) && (bj < 0 || zg[j] > best)) {
            best = zg[j];
            bj = j;
          }
        }
        selmask |= 1ull << bj;
      }
      if (a.k < a.M) {
        float lo = INFINITY, hi = -INFINITY;
        for (int j = 0; j < a.M; ++j) {
          const int e = g * a.M + j;
          const float bd = __fmul_ru(gam_ru, __fmaf_ru(nx, wmax[e], fabsf(bsm[e])));
          if ((selmask >> j) & 1ull) lo = fminf(lo, __fsub_rd(zg[j], bd));
          else hi = fmaxf(hi, __fadd_ru(zg[j], bd));
        }
        certain = lo > hi;
      }
    }
    for (int e = lane; e < a.N; e += 32) zd[e] = static_cast<double>(zf[e]);
    unsigned todo = __ballot_sync(0xffffffffu, !certain);
    __syncwarp();
    // fp64 re-evaluation of the groups whose decision was not certain.
    while (todo) {
      const int gg = __ffs(todo) - 1;
      todo &= todo - 1;
      for (int j = 0; j < a.M; ++j) {
        const int e = gg * a.M + j;
        double s64 = 0.0;
        for (int m = lane; m < a.d; m += 32)
          s64 = fma(static_cast<double>(bf16_to_f32(xr[m])), static_cast<double>(Wsm[m * S + e]), s64);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s64 += __shfl_xor_sync(0xffffffffu, s64, off);
        if (lane == 0) zd[e] = s64 + static_cast<double>(bsm[e]);
      }
    }
    __syncwarp();

    float psel_sum = 0.0f;
    if (g < a.G) {
      const double* zg = zd + g * a.M;
      if (!certain) {  // re-select on the fp64 logits
        selmask = 0;
        for (int s = 0; s < a.k; ++s) {
          double best = -INFINITY;
          int bj = -1;
          for (int j = 0; j < a.M; ++j) {
            if (!((selmask >> j) & 1ull) && (bj < 0 || zg[j] > best)) {
              best = zg[j];
              bj = j;
            }
          }
          selmask |= 1ull << bj;
        }
      }
      double zmax = zg[0];
      for (int j = 1; j < a.M; ++j) zmax = fmax(zmax, zg[j]);
      float den = 0.0f;
      for (int j = 0; j < a.M; ++j) den += expf(static_cast<float>(zg[j] - zmax));
      for (int j = 0; j < a.M; ++j)
        if ((selmask >> j) & 1ull) psel_sum += expf(static_cast<float>(zg[j] - zmax)) / den;
    }
    float tot = psel_sum;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, off);
    if (g < a.G) {
      const double* zg = zd + g * a.M;
      double zmax = zg[0];
      for (int j = 1; j < a.M; ++j) zmax = fmax(zmax, zg[j]);
      float den = 0.0f;
      for (int j = 0; j < a.M; ++j) den += expf(static_cast<float>(zg[j] - zmax));
      const size_t o = (static_cast<size_t>(row) * a.G + g) * a.k;
      int s = 0;
      for (int j = 0; j < a.M; ++j) {
        if ((selmask >> j) & 1ull) {
          const float p = expf(static_cast<float>(zg[j] - zmax)) / den;
          a.idx[o + s] = j;
          a.r[o + s] = p / psel_sum;
          a.omega[o + s] = p / tot;
          ++s;
        }
      }
    }
    __syncwarp();
  }
}


template <int NP>
int launch_np(const gqe_config& c, const RouterArgs& a, cudaStream_t st) {
  constexpr int S = router_row_floats(NP);
  const size_t smem = router_smem_bytes(c);
  if (smem > kRouterSmemLimit) return cudaErrorInvalidConfiguration;
  const int e = ensure_smem<router_kernel<NP>>(static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // One token per warp while that fills the GPU; larger batches loop.
  const int R = a.R;
  int grid = (R + kRouterWarps - 1) / kRouterWarps;
  if (grid > 4 * 148) grid = 4 * 148;
  if (grid < 1) grid = 1;
  return launch_pdl(router_kernel<NP>, dim3(grid), dim3(kRouterWarps * 32), smem, st, a);
}

}  // namespace router_impl
using namespace router_impl;

size_t router_smem_bytes(const gqe_config& c) {
  const int NP = router_np(c.G * c.M);
  const size_t zf = kRouterWarps * NP > kRouterWarps * 32 ? kRouterWarps * NP : kRouterWarps * 32;
  return static_cast<size_t>(c.d_model) * router_row_floats(NP) * 4 + 2 * NP * 4 +
         kRouterWarps * NP * 8 + zf * 4;
}

int launch_router(const gqe_config& c, const uint16_t* x, const float* W_r, const float* b_r,
                  int32_t* idx, float* r, float* omega, void* stream) {
  RouterArgs a{x, W_r, b_r, idx, r, omega, c.B * c.T, c.d_model, c.G, c.M, c.k, c.G * c.M};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (router_np(a.N)) {
    case 4: return launch_np<4>(c, a, st);
    case 8: return launch_np<8>(c, a, st);
    case 16: return launch_np<16>(c, a, st);
    case 32: return launch_np<32>(c, a, st);
    default: return launch_np<64>(c, a, st);
  }
}

}  // namespace gqe
