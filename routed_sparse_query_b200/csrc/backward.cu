// Backward of the GQE layer (the next row after the forward): the gradients
// of a loss L with respect to x and every weight, given dy = dL/dy, with the
// router's top-k selection held fixed. The selection is a discrete choice;
// the weighted slot is the layer's differentiable path from the loss to the
// router ("a differentiable path for the language-modelling loss to reach the
// router": gist.science Technical Summary, "Output Construction"; pptc.cn
// blog section 4.3).
//
// On the forward's own intermediates (recomputed by the forward kernels:
// routing, Q, K, V, slots). The contractions of the projections (dS = dy W_O^T,
// dW_O = S^T dy, dx and every weight gradient) run on the tensor cores
// through the projection GEMM (fp32 output) on bf16 copies of their
// operands, made here:
//   - transpose_kernel / cast_kernel: bf16 copies (x^T, S^T, W_O^T, the
//     projection weights transposed, dy);
//   - pack_grads_kernel: the rows of [dQ of every expert | dQ of the shared
//     head | dK | dV | dz] in bf16, the A operand of dx and the B operand of
//     every weight gradient;
//   - slot_router_bwd_kernel, one CTA per token: the slots' backward (routed
//     outputs, shared head, weighted slot) and the router's (the renormalised
//     weights' quotient rule, then each group's softmax Jacobian) -> dz;
//   - attn_rows_bwd_kernel, one CTA per 64 query rows of a stream, the key
//     tiles staged in shared memory: the rows' softmax statistics (max, sum),
//     D = dO . O, and dq;
//   - attn_keys_bwd_kernel, one CTA per 64 keys of a group: dK and dV summed
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
constexpr int BT = 64;       // query rows / keys per tile
constexpr int LDS = BT + 1;  // padded row length of a shared tile (floats)

// Loads rows [r0, r0 + BT) x dh of a bf16 or fp32 matrix with row stride ld
// into a shared tile (rows past nrows and columns past dh read as 0).
template <typename T>
__device__ __forceinline__ void load_tile(float* dst, const T* src, long long ld, int r0, int nrows, int dh) {
  for (int q = threadIdx.x; q < BT * kMaxDh; q += blockDim.x) {
    const int r = q / kMaxDh, c = q - r * kMaxDh;
    dst[r * LDS + c] = (r0 + r < nrows && c < dh) ? to_f(src[static_cast<long long>(r0 + r) * ld + c]) : 0.0f;
  }
}

// out[i][j] = sum_c X[ri][c] * Y[cj][c] for the thread's 4 x 4 block
// (rows ty*4.., columns tx*4..) of a BT x BT product over dh.
__device__ __forceinline__ void tile_dot(const float* X, const float* Y, int dh, int ty, int tx, float (&o)[4][4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) o[i][j] = 0.0f;
  for (int c = 0; c < dh; ++c) {
    float x[4], y[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[i] = X[(ty * 4 + i) * LDS + c];
      y[i] = Y[(tx * 4 + i) * LDS + c];
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) o[i][j] = fmaf(x[i], y[j], o[i][j]);
  }
}

// One CTA (256 threads, 16 x 16) per 64 query rows of one stream (b, h).
// Pass 1 over the key tiles: each row's max and sum of exp(s - max) (4
// threads per row). Pass 2: P, dP = dO . V, and per row D = sum P dP,
// U = sum P dP K, W = sum P K (thread (ty, tx): rows ty*4.., dims tx*4..);
// then dq = scale (U - D W) -- the one-pass form of scale sum P (dP - D) K.
__global__ void __launch_bounds__(256) attn_rows_bwd_kernel(AttnBwdArgs a) {
  extern __shared__ float sm[];
  float* Qt = sm;
  float* dOt = Qt + BT * LDS;
  float* Kt = dOt + BT * LDS;
  float* Vt = Kt + BT * LDS;
  float* Pt = Vt + BT * LDS;
  float* Xt = Pt + BT * LDS;
  float* mrow = Xt + BT * LDS;  // [BT]
  float* lrow = mrow + BT;      // [BT]
  const int H = a.G * a.k + 1, gk = a.G * a.k, dh = a.dh;
  const int nqt = (a.T + BT - 1) / BT;
  const int qt = blockIdx.x % nqt;
  const int h = (blockIdx.x / nqt) % H;
  const int b = blockIdx.x / (nqt * H);
  const int g = group_of(a, h), t0 = qt * BT;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const uint16_t* Qb = h < gk ? a.Qv + (static_cast<size_t>(b) * gk + h) * a.T * dh
                              : a.Qs + static_cast<size_t>(b) * a.T * dh;
  const float* dOb = h < gk ? a.dOr + static_cast<size_t>(h) * dh : a.dOs;
  const long long ldo = h < gk ? static_cast<long long>(gk) * dh : dh;
  const size_t orow0 = static_cast<size_t>(b) * a.T;
  const uint16_t* Kb = a.K + (static_cast<size_t>(b) * a.G + g) * a.T * dh;
  const uint16_t* Vb = a.V + (static_cast<size_t>(b) * a.G + g) * a.T * dh;
  load_tile(Qt, Qb, dh, t0, a.T, dh);
  load_tile(dOt, dOb + orow0 * ldo, ldo, t0, a.T, dh);
  // Pass 1: max and sum, online over the key tiles (row ty*4+i, 4 threads per row: tx % 4).
  const int prow = tid >> 2, pq = tid & 3;  // row prow, columns pq*16 .. pq*16+15 of the tile
  float m = -INFINITY, l = 0.0f;
  const int nkt = qt + 1;  // causal: key tiles 0 .. qt
  for (int kt = 0; kt < nkt; ++kt) {
    __syncthreads();
    load_tile(Kt, Kb, dh, kt * BT, a.T, dh);
    __syncthreads();
    float o[4][4];
    tile_dot(Qt, Kt, dh, ty, tx, o);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int t = t0 + ty * 4 + i, u = kt * BT + tx * 4 + j;
        Pt[(ty * 4 + i) * LDS + tx * 4 + j] = (u <= t && u < a.T) ? o[i][j] * a.scale : -INFINITY;
      }
    __syncthreads();
    float bm = -INFINITY;
    for (int j = 0; j < 16; ++j) bm = fmaxf(bm, Pt[prow * LDS + pq * 16 + j]);
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
    const float mn = fmaxf(m, bm);
    float bs = 0.0f;
    if (mn != -INFINITY)
      for (int j = 0; j < 16; ++j) bs += expf(Pt[prow * LDS + pq * 16 + j] - mn);
    bs += __shfl_xor_sync(0xffffffffu, bs, 1);
    bs += __shfl_xor_sync(0xffffffffu, bs, 2);
    l = (m == -INFINITY ? 0.0f : l * expf(m - mn)) + bs;
    m = mn;
  }
  if (pq == 0) {
    mrow[prow] = m;
    lrow[prow] = l;
  }
  // Pass 2.
  float U[4][4], Wa[4][4], Dp[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    Dp[i] = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) U[i][j] = Wa[i][j] = 0.0f;
  }
  for (int kt = 0; kt < nkt; ++kt) {
    __syncthreads();
    load_tile(Kt, Kb, dh, kt * BT, a.T, dh);
    load_tile(Vt, Vb, dh, kt * BT, a.T, dh);
    __syncthreads();
    float s[4][4], dp[4][4];
    tile_dot(Qt, Kt, dh, ty, tx, s);
    tile_dot(dOt, Vt, dh, ty, tx, dp);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty * 4 + i, t = t0 + r;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int u = kt * BT + tx * 4 + j;
        const float P = (u <= t && u < a.T && t < a.T) ? expf(s[i][j] * a.scale - mrow[r]) / lrow[r] : 0.0f;
        Pt[r * LDS + tx * 4 + j] = P;
        Xt[r * LDS + tx * 4 + j] = P * dp[i][j];
        Dp[i] += P * dp[i][j];
      }
    }
    __syncthreads();
    // U[r][c] += sum_u (P dP)[r][u] K[u][c], W[r][c] += sum_u P[r][u] K[u][c] for dims c = tx*4..
    if (tx * 4 < dh) {
      for (int u = 0; u < BT; ++u) {
        float kv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) kv[j] = Kt[u * LDS + tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float x = Xt[(ty * 4 + i) * LDS + u], p = Pt[(ty * 4 + i) * LDS + u];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            U[i][j] = fmaf(x, kv[j], U[i][j]);
            Wa[i][j] = fmaf(p, kv[j], Wa[i][j]);
          }
        }
      }
    }
  }
  // D per row: sum of the 16 column threads' parts.
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float v = Dp[i];
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);  // the 16 tx of a ty share a half-warp
    Dp[i] = v;
  }
  const int gkk = gk;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= a.T || tx * 4 >= dh) continue;
    const size_t row = orow0 + t;
    float* dq = h < gkk ? a.dQr + (row * gkk + h) * dh : a.dQs + row * dh;
#pragma unroll
    for (int j = 0; j < 4; ++j) dq[tx * 4 + j] = (U[i][j] - Dp[i] * Wa[i][j]) * a.scale;
    if (tx == 0) {
      float* st = a.stats + ((static_cast<size_t>(b) * H + h) * a.T + t) * 3;
      st[0] = mrow[ty * 4 + i];
      st[1] = lrow[ty * 4 + i];
      st[2] = Dp[i];
    }
  }
}

// One CTA per 64 keys (b, g, key tile kt). For every stream on group g and
// query tiles qt >= kt: S = Q K^T, P = exp(S scale - m_t) / l_t (t >= u),
// dP = dO V^T, dS = P (dP - D_t); then dV += P^T dO and dK += scale dS^T Q
// (thread (ty, tx): keys ty*4.., dims tx*4..). One writer per output row.
__global__ void __launch_bounds__(256) attn_keys_bwd_kernel(AttnBwdArgs a) {
  extern __shared__ float sm[];
  float* Kt = sm;
  float* Vt = Kt + BT * LDS;
  float* Qt = Vt + BT * LDS;
  float* dOt = Qt + BT * LDS;
  float* Pt = dOt + BT * LDS;  // [t][u]
  float* St = Pt + BT * LDS;   // dS [t][u]
  float* srow = St + BT * LDS; // [BT][3] stats of the query tile
  const int H = a.G * a.k + 1, gk = a.G * a.k, dh = a.dh;
  const int nkt = (a.T + BT - 1) / BT;
  const int kt = blockIdx.x % nkt;
  const int g = (blockIdx.x / nkt) % a.G;
  const int b = blockIdx.x / (nkt * a.G);
  const int u0 = kt * BT;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const uint16_t* Kb = a.K + (static_cast<size_t>(b) * a.G + g) * a.T * dh;
  const uint16_t* Vb = a.V + (static_cast<size_t>(b) * a.G + g) * a.T * dh;
  load_tile(Kt, Kb, dh, u0, a.T, dh);
  load_tile(Vt, Vb, dh, u0, a.T, dh);
  float dK[4][4], dV[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) dK[i][j] = dV[i][j] = 0.0f;
  const size_t orow0 = static_cast<size_t>(b) * a.T;
  for (int h = 0; h < H; ++h) {
    if (group_of(a, h) != g) continue;
    const uint16_t* Qb = h < gk ? a.Qv + (static_cast<size_t>(b) * gk + h) * a.T * dh
                                : a.Qs + static_cast<size_t>(b) * a.T * dh;
    const float* dOb = h < gk ? a.dOr + static_cast<size_t>(h) * dh : a.dOs;
    const long long ldo = h < gk ? static_cast<long long>(gk) * dh : dh;
    const float* st = a.stats + (static_cast<size_t>(b) * H + h) * a.T * 3;
    for (int qt = kt; qt < nkt; ++qt) {
      const int t0 = qt * BT;
      __syncthreads();
      load_tile(Qt, Qb, dh, t0, a.T, dh);
      load_tile(dOt, dOb + orow0 * ldo, ldo, t0, a.T, dh);
      for (int q = tid; q < BT * 3; q += blockDim.x)
        srow[q] = t0 + q / 3 < a.T ? st[static_cast<size_t>(t0) * 3 + q] : 0.0f;
      __syncthreads();
      float s[4][4], dp[4][4];
      tile_dot(Qt, Kt, dh, ty, tx, s);   // rows t (ty), columns u (tx)
      tile_dot(dOt, Vt, dh, ty, tx, dp);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = ty * 4 + i, t = t0 + r;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int u = u0 + tx * 4 + j;
          float P = 0.0f;
          if (t < a.T && u < a.T && u <= t) P = expf(s[i][j] * a.scale - srow[r * 3]) / srow[r * 3 + 1];
          Pt[r * LDS + tx * 4 + j] = P;
          St[r * LDS + tx * 4 + j] = P * (dp[i][j] - srow[r * 3 + 2]);
        }
      }
      __syncthreads();
      // dV[u][c] += sum_t P[t][u] dO[t][c]; dK[u][c] += sum_t dS[t][u] Q[t][c] (keys ty*4.., dims tx*4..).
      if (tx * 4 < dh) {
        for (int t = 0; t < BT; ++t) {
          float qv[4], ov[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            qv[j] = Qt[t * LDS + tx * 4 + j];
            ov[j] = dOt[t * LDS + tx * 4 + j];
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float p = Pt[t * LDS + ty * 4 + i], ds = St[t * LDS + ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              dV[i][j] = fmaf(p, ov[j], dV[i][j]);
              dK[i][j] = fmaf(ds, qv[j], dK[i][j]);
            }
          }
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int u = u0 + ty * 4 + i;
    if (u >= a.T || tx * 4 >= dh) continue;
    const size_t o = (orow0 + u) * a.G * dh + static_cast<size_t>(g) * dh + tx * 4;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      a.dKf[o + j] = dK[i][j] * a.scale;
      a.dVf[o + j] = dV[i][j];
    }
  }
}

__device__ __forceinline__ uint16_t bf16_rn(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }

// out[c, r] = bf16(in[r, c]) for r < rows, c < cols: 32 x 32 tiles through
// shared memory (block 32 x 8), both sides coalesced.
template <typename TI>
__global__ void __launch_bounds__(256) transpose_kernel(const TI* in, long long ldi, int rows, int cols,
                                                        uint16_t* out, long long ldo) {
  __shared__ float tile[32][33];
  const long long r0 = static_cast<long long>(blockIdx.y) * 32, c0 = static_cast<long long>(blockIdx.x) * 32;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const long long r = r0 + i, c = c0 + threadIdx.x;
    tile[i][threadIdx.x] = (r < rows && c < cols) ? to_f(in[r * ldi + c]) : 0.0f;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += 8) {
    const long long c = c0 + i, r = r0 + threadIdx.x;
    if (c < cols && r < rows) out[c * ldo + r] = bf16_rn(tile[threadIdx.x][i]);
  }
}

// out[r, c] = bf16(in[r, c]) (row strides ldi, ldo).
__global__ void cast_kernel(const float* in, long long ldi, long long rows, int cols, uint16_t* out, long long ldo) {
  const long long n = rows * cols;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / cols;
    const int c = static_cast<int>(i - r * cols);
    out[r * ldo + c] = bf16_rn(in[r * ldi + c]);
  }
}

// Row r of Y (bf16, ld columns): [dQ of every expert (the slot of row r that
// selected expert e, 0 where none did) | dQ of the shared head | dK | dV |
// dz | 0 padding]. Each thread writes two adjacent columns.
__global__ void pack_grads_kernel(const float* dQr, const float* dQs, const float* dKf, const float* dVf,
                                  const float* dz, const int32_t* idx, uint16_t* Y, long long R, int G, int M,
                                  int k, int dh, int ld) {
  const int N = G * M, c1 = N * dh, c2 = c1 + dh, c3 = c2 + G * dh, c4 = c3 + G * dh, c5 = c4 + N;
  const int half = ld / 2;
  const long long n = R * half;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / half;
    const int c = 2 * static_cast<int>(i - r * half);
    float v[2] = {0.0f, 0.0f};
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int cc = c + q;
      if (cc < c1) {
        const int e = cc / dh, col = cc - e * dh, g = e / M, j = e - g * M;
        const int32_t* ip = idx + (r * G + g) * k;
        for (int s = 0; s < k; ++s)
          if (ip[s] == j) v[q] = dQr[((r * G + g) * k + s) * dh + col];
      } else if (cc < c2) {
        v[q] = dQs[r * dh + (cc - c1)];
      } else if (cc < c3) {
        v[q] = dKf[r * G * dh + (cc - c2)];
      } else if (cc < c4) {
        v[q] = dVf[r * G * dh + (cc - c3)];
      } else if (cc < c5) {
        v[q] = dz[r * N + (cc - c4)];
      }
    }
    *reinterpret_cast<uint32_t*>(Y + r * ld + c) = static_cast<uint32_t>(bf16_rn(v[0])) |
                                                  (static_cast<uint32_t>(bf16_rn(v[1])) << 16);
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

template <typename TI>
int bwd_transpose(const TI* in, long long ldi, int rows, int cols, uint16_t* out, long long ldo, void* stream) {
  if (rows <= 0 || cols <= 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((cols + 31) / 32), static_cast<unsigned>((rows + 31) / 32));
  if (grid.y > 65535u) return cudaErrorInvalidConfiguration;
  transpose_kernel<TI><<<grid, dim3(32, 8), 0, static_cast<cudaStream_t>(stream)>>>(in, ldi, rows, cols, out, ldo);
  return cudaGetLastError();
}
template int bwd_transpose<uint16_t>(const uint16_t*, long long, int, int, uint16_t*, long long, void*);
template int bwd_transpose<float>(const float*, long long, int, int, uint16_t*, long long, void*);

int bwd_cast(const float* in, long long ldi, long long rows, int cols, uint16_t* out, long long ldo, void* stream) {
  cast_kernel<<<1024, 256, 0, static_cast<cudaStream_t>(stream)>>>(in, ldi, rows, cols, out, ldo);
  return cudaGetLastError();
}

int bwd_pack(const gqe_config& c, const float* dQr, const float* dQs, const float* dKf, const float* dVf,
             const float* dz, const int32_t* idx, uint16_t* Y, int ld, void* stream) {
  const long long R = static_cast<long long>(c.B) * c.T;
  pack_grads_kernel<<<1184, 256, 0, static_cast<cudaStream_t>(stream)>>>(dQr, dQs, dKf, dVf, dz, idx, Y, R, c.G,
                                                                         c.M, c.k, c.d_head, ld);
  return cudaGetLastError();
}

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
  const long long ntiles = (c.T + BT - 1) / BT;
  const long long row_ctas = static_cast<long long>(c.B) * (c.G * c.k + 1) * ntiles;
  const long long key_ctas = static_cast<long long>(c.B) * c.G * ntiles;
  if (row_ctas > 0x7fffffffll || key_ctas > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  const int smem_rows = static_cast<int>((6 * BT * LDS + 2 * BT) * sizeof(float));
  const int smem_keys = static_cast<int>((6 * BT * LDS + 3 * BT) * sizeof(float));
  cudaError_t e = static_cast<cudaError_t>(ensure_smem<attn_rows_bwd_kernel>(smem_rows));
  if (e == cudaSuccess) e = static_cast<cudaError_t>(ensure_smem<attn_keys_bwd_kernel>(smem_keys));
  if (e != cudaSuccess) return e;
  attn_rows_bwd_kernel<<<static_cast<unsigned>(row_ctas), 256, smem_rows, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_keys_bwd_kernel<<<static_cast<unsigned>(key_ctas), 256, smem_keys, st>>>(a);
  return cudaGetLastError();
}

int bwd_colsum(const float* dz, float* db, long long R, int N, void* stream) {
  colsum_kernel<<<N, 256, 0, static_cast<cudaStream_t>(stream)>>>(dz, db, R, N);
  return cudaGetLastError();
}

}  // namespace gqe
