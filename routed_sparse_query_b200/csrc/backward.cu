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
// The attention's own backward (dq, dK, dV) runs on the tensor cores as well
// (attn_bwd.cu).
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
  uint16_t* dO16;         // [B, G*k + 1, T, dh]: dO per stream in bf16 (the attention backward's operand)
  int d, G, M, k, dh, T;
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
  const int bb = r / a.T, t = r - bb * a.T;
  uint16_t* o16 = a.dO16 + (static_cast<size_t>(bb) * (gk + 1) * a.T + t) * dh;
  const size_t hs = static_cast<size_t>(a.T) * dh;  // stream stride of dO16
  for (int q = tid; q < gk * dh; q += blockDim.x) {
    const int gs = q / dh, c = q - gs * dh;
    const float v = dSr[q] + om[gs] * dSw[c];
    a.dOr[static_cast<size_t>(r) * gk * dh + q] = v;
    o16[gs * hs + c] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  }
  for (int c = tid; c < dh; c += blockDim.x) {
    const float v = dSr[gk * dh + c];
    a.dOs[static_cast<size_t>(r) * dh + c] = v;
    o16[gk * hs + c] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
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
                     float* dOs, float* dz, uint16_t* dO16, void* stream) {
  SlotArgs a{x, W_r, b_r, idx, omega, slots, dS, dOr, dOs, dz, dO16, c.d_model, c.G, c.M, c.k, c.d_head, c.T};
  slot_router_bwd_kernel<<<c.B * c.T, 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return cudaGetLastError();
}

int bwd_colsum(const float* dz, float* db, long long R, int N, void* stream) {
  colsum_kernel<<<N, 256, 0, static_cast<cudaStream_t>(stream)>>>(dz, db, R, N);
  return cudaGetLastError();
}

}  // namespace gqe
