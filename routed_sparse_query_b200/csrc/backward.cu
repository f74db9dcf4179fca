// Backward of the GQE layer (the next row after the forward): the gradients
// of a loss L with respect to x and every weight, given dy = dL/dy, with the
// router's top-k selection held fixed. The selection is a discrete choice;
// the weighted slot is the layer's differentiable path from the loss to the
// router ("a differentiable path for the language-modelling loss to reach the
// router": gist.science Technical Summary, "Output Construction"; pptc.cn
// blog section 4.3).
//
// A first, plain path on the CUDA cores, in fp32 throughout, on the forward's
// own intermediates (recomputed by the forward kernels: routing, Q, K, V,
// slots):
//   - gemm_f32_kernel: C (+)= A B for any strides of A and B (bf16 or fp32),
//     64 x 64 tiles through shared memory. It carries dS = dy W_O^T,
//     dW_O = S^T dy and every weight and input gradient of the projections;
//   - slot_router_bwd_kernel, one CTA per token: the slots' backward (routed
//     outputs, shared head, weighted slot) and the router's (the renormalised
//     weights' quotient rule, then each group's softmax Jacobian) -> dz;
//   - attn_rows_bwd_kernel, one warp per query row of a stream: the row's
//     softmax statistics (max, sum), D = dO . O, and dq;
//   - attn_keys_bwd_kernel, one warp per key of a group: dK and dV summed
//     over every stream that attends to the group (no atomics: each output
//     row has one writer, so the result is deterministic).
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cmath>

#include "gqe_internal.h"
#include "ptx.cuh"

namespace gqe {

namespace bwd_impl {

__device__ __forceinline__ float to_f(uint16_t v) { return __uint_as_float(static_cast<uint32_t>(v) << 16); }
__device__ __forceinline__ float to_f(float v) { return v; }

template <typename TA, typename TB>
__global__ void __launch_bounds__(256) gemm_f32_kernel(const TA* A, long long sam, long long sak, const TB* B,
                                                       long long sbk, long long sbn, float* C, long long ldc,
                                                       int M, int N, int K, int beta) {
  __shared__ float As[16][65];  // [k][m]
  __shared__ float Bs[16][65];  // [k][n]
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const long long m0 = static_cast<long long>(blockIdx.y) * 64, n0 = static_cast<long long>(blockIdx.x) * 64;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int q = threadIdx.x; q < 1024; q += 256) {
      const int mm = q >> 4, ka = q & 15;
      const long long gm = m0 + mm;
      const int gk = k0 + ka;
      As[ka][mm] = (gm < M && gk < K) ? to_f(A[gm * sam + gk * sak]) : 0.0f;
      const int kb = q >> 6, nn = q & 63;
      const long long gn = n0 + nn;
      const int gk2 = k0 + kb;
      Bs[kb][nn] = (gk2 < K && gn < N) ? to_f(B[gk2 * sbk + gn * sbn]) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        b[i] = Bs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const long long gm = m0 + ty * 4 + i, gn = n0 + tx * 4 + j;
      if (gm < M && gn < N) {
        float v = acc[i][j];
        if (beta) v += C[gm * ldc + gn];
        C[gm * ldc + gn] = v;
      }
    }
}

struct SlotArgs {
  const uint16_t* x;      // [R, d]
  const float* W_r;       // [d, N]
  const float* b_r;       // [N] or null
  const int32_t* idx;     // [R, G, k]
  const float* omega;     // [R, G, k] (the forward's weights)
  const uint16_t* slots;  // [R, S*dh] (S = kG+2)
  const float* dS;        // [R, S*dh]
  float* dOr;             // [R, G, k, dh]
  float* dOs;             // [R, dh]
  float* dz;              // [R, N]
  int d, G, M, k, dh;
};

// One CTA (256 threads) per token row.
__global__ void __launch_bounds__(256) slot_router_bwd_kernel(SlotArgs a) {
  __shared__ float z[kMaxExperts], p[kMaxExperts], dp[kMaxExperts], dw[kMaxExperts];
  __shared__ float tot_sh, sdw_sh;
  const int r = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int N = a.G * a.M, gk = a.G * a.k, dh = a.dh, Sdh = (gk + 2) * dh;
  const uint16_t* xr = a.x + static_cast<size_t>(r) * a.d;
  const float* dSr = a.dS + static_cast<size_t>(r) * Sdh;
  const float* dSw = dSr + (gk + 1) * dh;
  const uint16_t* orow = a.slots + static_cast<size_t>(r) * Sdh;
  const float* om = a.omega + static_cast<size_t>(r) * gk;
  // Logits (fp32) and each group's softmax.
  for (int e = warp; e < N; e += 8) {
    float s = 0.0f;
    for (int i = lane; i < a.d; i += 32) s = fmaf(to_f(xr[i]), a.W_r[static_cast<size_t>(i) * N + e], s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) z[e] = s + (a.b_r != nullptr ? a.b_r[e] : 0.0f);
  }
  // dw[g, s] = <o[g, s], dS_w>.
  for (int q = warp; q < gk; q += 8) {
    float s = 0.0f;
    for (int c = lane; c < dh; c += 32) s = fmaf(to_f(orow[q * dh + c]), dSw[c], s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) dw[q] = s;
  }
  __syncthreads();
  if (tid < a.G) {
    const int g = tid;
    float mx = -INFINITY;
    for (int j = 0; j < a.M; ++j) mx = fmaxf(mx, z[g * a.M + j]);
    float sum = 0.0f;
    for (int j = 0; j < a.M; ++j) sum += expf(z[g * a.M + j] - mx);
    for (int j = 0; j < a.M; ++j) p[g * a.M + j] = expf(z[g * a.M + j] - mx) / sum;
  }
  __syncthreads();
  if (tid == 0) {
    float tot = 0.0f, sdw = 0.0f;
    for (int q = 0; q < gk; ++q) {
      const int g = q / a.k;
      tot += p[g * a.M + a.idx[static_cast<size_t>(r) * gk + q]];
      sdw += om[q] * dw[q];
    }
    tot_sh = tot;
    sdw_sh = sdw;
  }
  for (int e = tid; e < N; e += blockDim.x) dp[e] = 0.0f;
  __syncthreads();
  // w = psel / sum(psel): dpsel = (dw - sum(w dw)) / sum(psel).
  if (tid < gk) {
    const int g = tid / a.k;
    dp[g * a.M + a.idx[static_cast<size_t>(r) * gk + tid]] = (dw[tid] - sdw_sh) / tot_sh;
  }
  __syncthreads();
  // Each group's softmax Jacobian.
  if (tid < N) {
    const int g = tid / a.M;
    float s = 0.0f;
    for (int j = 0; j < a.M; ++j) s += p[g * a.M + j] * dp[g * a.M + j];
    a.dz[static_cast<size_t>(r) * N + tid] = p[tid] * (dp[tid] - s);
  }
  // Routed outputs: dS of their slot plus omega times dS of the weighted slot.
  for (int q = tid; q < gk * dh; q += blockDim.x) {
    const int gs = q / dh, c = q - gs * dh;
    a.dOr[static_cast<size_t>(r) * gk * dh + q] = dSr[q] + om[gs] * dSw[c];
  }
  for (int c = tid; c < dh; c += blockDim.x) a.dOs[static_cast<size_t>(r) * dh + c] = dSr[gk * dh + c];
}

struct AttnBwdArgs {
  const uint16_t* Qv;  // [B, G, k, T, dh]
  const uint16_t* Qs;  // [B, T, dh]
  const uint16_t* K;   // [B, G, T, dh]
  const uint16_t* V;
  const float* dOr;    // [R, G, k, dh]
  const float* dOs;    // [R, dh]
  float* stats;        // [B, H, T, 3]: max, sum, D
  float* dQr;          // [R, G, k, dh]
  float* dQs;          // [R, dh]
  float* dKf;          // [R, G*dh]
  float* dVf;          // [R, G*dh]
  int B, T, G, k, dh;
  float scale;         // 1 / sqrt(dh)
};

// Stream h of sequence b: routed slot (g, s) = (h / k, h % k) for h < kG, the
// shared head (group 0) for h == kG.
__device__ __forceinline__ const uint16_t* q_row(const AttnBwdArgs& a, int b, int h, int t) {
  const int gk = a.G * a.k;
  if (h < gk) return a.Qv + ((static_cast<size_t>(b) * gk + h) * a.T + t) * a.dh;
  return a.Qs + (static_cast<size_t>(b) * a.T + t) * a.dh;
}
__device__ __forceinline__ const float* do_row(const AttnBwdArgs& a, int b, int h, int t) {
  const int gk = a.G * a.k;
  const size_t row = static_cast<size_t>(b) * a.T + t;
  if (h < gk) return a.dOr + (row * gk + h) * a.dh;
  return a.dOs + row * a.dh;
}
__device__ __forceinline__ int group_of(const AttnBwdArgs& a, int h) { return h < a.G * a.k ? h / a.k : 0; }

constexpr int kMaxDh = 64;

// One warp per query row (b, h, t); 8 rows per CTA. Lane j takes keys
// u = j, j + 32, ... <= t. Pass 1: max and sum of exp(s - max); pass 2:
// D = sum_u P dP (= dO . O); pass 3: dq = scale * sum_u P (dP - D) K_u,
// through 32 keys at a time in shared memory (lane c takes columns c, c+32).
__global__ void __launch_bounds__(256) attn_rows_bwd_kernel(AttnBwdArgs a) {
  __shared__ float qs[8][kMaxDh], ds[8][kMaxDh], wbuf[8][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = a.G * a.k + 1;
  const long long gid = static_cast<long long>(blockIdx.x) * 8 + warp;
  if (gid >= static_cast<long long>(a.B) * H * a.T) return;
  const int t = static_cast<int>(gid % a.T);
  const int h = static_cast<int>((gid / a.T) % H);
  const int b = static_cast<int>(gid / (static_cast<long long>(a.T) * H));
  const int g = group_of(a, h), dh = a.dh;
  const uint16_t* qr = q_row(a, b, h, t);
  const float* dor = do_row(a, b, h, t);
  for (int c = lane; c < dh; c += 32) {
    qs[warp][c] = to_f(qr[c]);
    ds[warp][c] = dor[c];
  }
  __syncwarp();
  const uint16_t* Kb = a.K + (static_cast<size_t>(b) * a.G + g) * a.T * dh;
  const uint16_t* Vb = a.V + (static_cast<size_t>(b) * a.G + g) * a.T * dh;
  auto score = [&](int u) {
    float s = 0.0f;
    for (int c = 0; c < dh; ++c) s = fmaf(qs[warp][c], to_f(Kb[static_cast<size_t>(u) * dh + c]), s);
    return s * a.scale;
  };
  auto dprob = [&](int u) {
    float s = 0.0f;
    for (int c = 0; c < dh; ++c) s = fmaf(ds[warp][c], to_f(Vb[static_cast<size_t>(u) * dh + c]), s);
    return s;
  };
  float mx = -INFINITY;
  for (int u = lane; u <= t; u += 32) mx = fmaxf(mx, score(u));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float l = 0.0f;
  for (int u = lane; u <= t; u += 32) l += expf(score(u) - mx);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  float D = 0.0f;
  for (int u = lane; u <= t; u += 32) D += expf(score(u) - mx) / l * dprob(u);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) D += __shfl_xor_sync(0xffffffffu, D, o);
  float dq0 = 0.0f, dq1 = 0.0f;
  for (int u0 = 0; u0 <= t; u0 += 32) {
    const int u = u0 + lane;
    float w = 0.0f;
    if (u <= t) {
      const float P = expf(score(u) - mx) / l;
      w = P * (dprob(u) - D);
    }
    wbuf[warp][lane] = w;
    __syncwarp();
    const int n = min(32, t - u0 + 1);
    for (int jj = 0; jj < n; ++jj) {
      const float wj = wbuf[warp][jj];
      const uint16_t* kr = Kb + static_cast<size_t>(u0 + jj) * dh;
      dq0 = fmaf(wj, to_f(kr[lane]), dq0);
      if (lane + 32 < dh) dq1 = fmaf(wj, to_f(kr[lane + 32]), dq1);
    }
    __syncwarp();
  }
  const size_t row = static_cast<size_t>(b) * a.T + t;
  const int gk = a.G * a.k;
  float* dq = h < gk ? a.dQr + (row * gk + h) * dh : a.dQs + row * dh;
  if (lane < dh) dq[lane] = dq0 * a.scale;
  if (lane + 32 < dh) dq[lane + 32] = dq1 * a.scale;
  if (lane == 0) {
    float* st = a.stats + ((static_cast<size_t>(b) * H + h) * a.T + t) * 3;
    st[0] = mx;
    st[1] = l;
    st[2] = D;
  }
}

// One warp per key (b, g, u); 8 keys per CTA. For every stream h on group g
// and rows t >= u (32 at a time, lane j on row t0 + j): P = exp(s - max) / sum,
// dS = P (dP - D); then lane c accumulates dV[c] += P dO_t[c] and
// dK[c] += dS q_t[c] (columns c, c + 32) over those rows.
__global__ void __launch_bounds__(256) attn_keys_bwd_kernel(AttnBwdArgs a) {
  __shared__ float ks[8][kMaxDh], vs[8][kMaxDh], pbuf[8][32], sbuf[8][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = a.G * a.k + 1;
  const long long gid = static_cast<long long>(blockIdx.x) * 8 + warp;
  if (gid >= static_cast<long long>(a.B) * a.G * a.T) return;
  const int u = static_cast<int>(gid % a.T);
  const int g = static_cast<int>((gid / a.T) % a.G);
  const int b = static_cast<int>(gid / (static_cast<long long>(a.T) * a.G));
  const int dh = a.dh;
  const uint16_t* kr = a.K + ((static_cast<size_t>(b) * a.G + g) * a.T + u) * dh;
  const uint16_t* vr = a.V + ((static_cast<size_t>(b) * a.G + g) * a.T + u) * dh;
  for (int c = lane; c < dh; c += 32) {
    ks[warp][c] = to_f(kr[c]);
    vs[warp][c] = to_f(vr[c]);
  }
  __syncwarp();
  float dk0 = 0.0f, dk1 = 0.0f, dv0 = 0.0f, dv1 = 0.0f;
  for (int h = 0; h < H; ++h) {
    if (group_of(a, h) != g) continue;
    const float* st = a.stats + (static_cast<size_t>(b) * H + h) * a.T * 3;
    for (int t0 = u; t0 < a.T; t0 += 32) {
      const int t = t0 + lane;
      float P = 0.0f, dS = 0.0f;
      if (t < a.T) {
        const uint16_t* qr = q_row(a, b, h, t);
        const float* dor = do_row(a, b, h, t);
        float s = 0.0f, dp = 0.0f;
        for (int c = 0; c < dh; ++c) {
          s = fmaf(to_f(qr[c]), ks[warp][c], s);
          dp = fmaf(dor[c], vs[warp][c], dp);
        }
        P = expf(s * a.scale - st[t * 3]) / st[t * 3 + 1];
        dS = P * (dp - st[t * 3 + 2]);
      }
      pbuf[warp][lane] = P;
      sbuf[warp][lane] = dS;
      __syncwarp();
      const int n = min(32, a.T - t0);
      for (int jj = 0; jj < n; ++jj) {
        const uint16_t* qr = q_row(a, b, h, t0 + jj);
        const float* dor = do_row(a, b, h, t0 + jj);
        const float pj = pbuf[warp][jj], sj = sbuf[warp][jj];
        dv0 = fmaf(pj, dor[lane], dv0);
        dk0 = fmaf(sj, to_f(qr[lane]), dk0);
        if (lane + 32 < dh) {
          dv1 = fmaf(pj, dor[lane + 32], dv1);
          dk1 = fmaf(sj, to_f(qr[lane + 32]), dk1);
        }
      }
      __syncwarp();
    }
  }
  const size_t o = (static_cast<size_t>(b) * a.T + u) * a.G * dh + static_cast<size_t>(g) * dh;
  if (lane < dh) {
    a.dKf[o + lane] = dk0 * a.scale;
    a.dVf[o + lane] = dv0;
  }
  if (lane + 32 < dh) {
    a.dKf[o + lane + 32] = dk1 * a.scale;
    a.dVf[o + lane + 32] = dv1;
  }
}

// dQfull[r, e*dh + c] = dq of the slot of row r that selected expert e, 0 for
// the experts the row did not select.
__global__ void scatter_dq_kernel(const float* dQr, const int32_t* idx, float* dQfull, long long R, int G,
                                  int M, int k, int dh) {
  const long long n = R * G * M * dh;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(i % dh);
    const long long re = i / dh;
    const int e = static_cast<int>(re % (G * M));
    const long long r = re / (G * M);
    const int g = e / M, j = e - g * M;
    float v = 0.0f;
    for (int s = 0; s < k; ++s)
      if (idx[(r * G + g) * k + s] == j) v = dQr[((r * G + g) * k + s) * dh + c];
    dQfull[i] = v;
  }
}

// db[e] = sum over rows of dz[r, e].
__global__ void colsum_kernel(const float* dz, float* db, long long R, int N) {
  const int e = blockIdx.x;
  float s = 0.0f;
  for (long long r = threadIdx.x; r < R; r += blockDim.x) s += dz[r * N + e];
  __shared__ float red[256];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) db[e] = red[0];
}

}  // namespace bwd_impl
using namespace bwd_impl;

template <typename TA, typename TB>
int bwd_gemm(const TA* A, long long sam, long long sak, const TB* B, long long sbk, long long sbn, float* C,
             long long ldc, int M, int N, int K, bool accumulate, void* stream) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((N + 63) / 64), static_cast<unsigned>((M + 63) / 64));
  if (grid.y > 65535u) return cudaErrorInvalidConfiguration;
  gemm_f32_kernel<TA, TB><<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(A, sam, sak, B, sbk, sbn, C, ldc,
                                                                              M, N, K, accumulate ? 1 : 0);
  return cudaGetLastError();
}
template int bwd_gemm<uint16_t, float>(const uint16_t*, long long, long long, const float*, long long, long long,
                                       float*, long long, int, int, int, bool, void*);
template int bwd_gemm<float, uint16_t>(const float*, long long, long long, const uint16_t*, long long, long long,
                                       float*, long long, int, int, int, bool, void*);
template int bwd_gemm<float, float>(const float*, long long, long long, const float*, long long, long long,
                                    float*, long long, int, int, int, bool, void*);

int bwd_slots_router(const gqe_config& c, const uint16_t* x, const float* W_r, const float* b_r,
                     const int32_t* idx, const float* omega, const uint16_t* slots, const float* dS, float* dOr,
                     float* dOs, float* dz, void* stream) {
  SlotArgs a{x, W_r, b_r, idx, omega, slots, dS, dOr, dOs, dz, c.d_model, c.G, c.M, c.k, c.d_head};
  slot_router_bwd_kernel<<<c.B * c.T, 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return cudaGetLastError();
}

int bwd_attention(const gqe_config& c, const uint16_t* Qv, const uint16_t* Qs, const uint16_t* K,
                  const uint16_t* V, const float* dOr, const float* dOs, float* stats, float* dQr, float* dQs,
                  float* dKf, float* dVf, void* stream) {
  AttnBwdArgs a{Qv, Qs, K, V, dOr, dOs, stats, dQr, dQs, dKf, dVf, c.B, c.T, c.G, c.k, c.d_head,
                static_cast<float>(1.0 / std::sqrt(static_cast<double>(c.d_head)))};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long rows = static_cast<long long>(c.B) * (c.G * c.k + 1) * c.T;
  const long long keys = static_cast<long long>(c.B) * c.G * c.T;
  attn_rows_bwd_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_keys_bwd_kernel<<<static_cast<unsigned>((keys + 7) / 8), 256, 0, st>>>(a);
  return cudaGetLastError();
}

int bwd_scatter_dq(const gqe_config& c, const float* dQr, const int32_t* idx, float* dQfull, void* stream) {
  const long long R = static_cast<long long>(c.B) * c.T;
  scatter_dq_kernel<<<1024, 256, 0, static_cast<cudaStream_t>(stream)>>>(dQr, idx, dQfull, R, c.G, c.M, c.k,
                                                                         c.d_head);
  return cudaGetLastError();
}

int bwd_colsum(const float* dz, float* db, long long R, int N, void* stream) {
  colsum_kernel<<<N, 256, 0, static_cast<cudaStream_t>(stream)>>>(dz, db, R, N);
  return cudaGetLastError();
}

}  // namespace gqe
