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

// Router logits z[r, e] = x[r] . W_r[:, e] + b[e] in fp32 (as the forward's
// router forms them), 16 rows per CTA; W_r and the 16 rows of x are staged
// in shared memory, then thread (row i, expert e) of a pass takes one dot
// product over d.
constexpr int kLogitRows = 16;
__global__ void __launch_bounds__(256) logits_kernel(const uint16_t* x, const float* W_r, const float* b_r,
                                                     float* z, long long R, int d, int N) {
  extern __shared__ float4 Ws4[];  // W_r [d][N] (d N is a multiple of 4: d is one of 64), then x rows [16][d] bf16
  const float* Ws = reinterpret_cast<const float*>(Ws4);
  const int nw = d * N / 4;
  uint4* xs4 = reinterpret_cast<uint4*>(Ws4 + nw);
  const float4* W4 = reinterpret_cast<const float4*>(W_r);
  const long long r0 = static_cast<long long>(blockIdx.x) * kLogitRows;
  const int rows = static_cast<int>(R - r0 < kLogitRows ? R - r0 : kLogitRows);
  const int xw = d / 8;  // 16-byte words per x row
#pragma unroll 8
  for (int i = threadIdx.x; i < nw; i += blockDim.x) Ws4[i] = __ldg(W4 + i);
#pragma unroll 4
  for (int i = threadIdx.x; i < rows * xw; i += blockDim.x)
    xs4[i] = __ldg(reinterpret_cast<const uint4*>(x + r0 * d) + i);
  __syncthreads();
  const int per = blockDim.x / N;  // rows per pass
  const int e = threadIdx.x % N, i0 = threadIdx.x / N;
  if (i0 >= per) return;
  for (int i = i0; i < rows; i += per) {
    const uint4* xr = xs4 + i * xw;
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // four partial sums, added in a fixed order
    for (int c8 = 0; c8 < xw; ++c8) {
      const uint4 v = xr[c8];
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[q] = fmaf(__uint_as_float(u[q] << 16), Ws[(c8 * 8 + 2 * q) * N + e], acc[q]);
        acc[q] = fmaf(__uint_as_float(u[q] & 0xffff0000u), Ws[(c8 * 8 + 2 * q + 1) * N + e], acc[q]);
      }
    }
    z[(r0 + i) * N + e] = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + (b_r != nullptr ? b_r[e] : 0.0f);
  }
}

struct SlotArgs {
  const uint16_t* x;      // [R, d]
  const float* W_r;       // [d, N]
  const float* b_r;       // [N] or null
  const float* zl;        // [R, N]: the router logits (logits_kernel)
  const int32_t* idx;     // [R, G, k]
  const float* omega;     // [R, G, k] (the forward's weights)
  const uint16_t* slots;  // [R, S*dh] (S = kG+2)
  const float* dS;        // [R, S*dh]
  float* dOr;             // [R, G, k, dh]
  float* dOs;             // [R, dh]
  float* dz;              // [R, N]
  uint16_t* dO16;         // [B, G*k + 1, T, dh]: dO per stream in bf16 (the attention backward's operand)
  float* Drow;            // [B, G*k + 1, Tp]: D = dO . O per stream and row (the attention backward's)
  int d, G, M, k, dh, T, Tp;
};

// One CTA (256 threads) per token row.
__global__ void __launch_bounds__(256) slot_router_bwd_kernel(SlotArgs a) {
  __shared__ float z[kMaxExperts], p[kMaxExperts], dp[kMaxExperts], dw[kMaxExperts];
  __shared__ float tot_sh, sdw_sh;
  const int r = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int N = a.G * a.M, gk = a.G * a.k, dh = a.dh, Sdh = (gk + 2) * dh;
  const float* dSr = a.dS + static_cast<size_t>(r) * Sdh;
  const float* dSw = dSr + (gk + 1) * dh;
  const uint16_t* orow = a.slots + static_cast<size_t>(r) * Sdh;
  const float* om = a.omega + static_cast<size_t>(r) * gk;
  // Logits (fp32) and each group's softmax.
  for (int e = tid; e < N; e += blockDim.x) z[e] = a.zl[static_cast<size_t>(r) * N + e];
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
  // D = dO . O of every stream (O = the forward's slot, bf16), one warp per stream.
  for (int h = warp; h <= gk; h += 8) {
    float sd = 0.0f;
    for (int c = lane; c < dh; c += 32) {
      const float v = h < gk ? dSr[h * dh + c] + om[h] * dSw[c] : dSr[gk * dh + c];
      sd = fmaf(v, to_f(orow[h * dh + c]), sd);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sd += __shfl_xor_sync(0xffffffffu, sd, o);
    if (lane == 0) a.Drow[(static_cast<size_t>(bb) * (gk + 1) + h) * a.Tp + t] = sd;
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

// The bf16 transpose on 64 x 64 tiles (block 32 x 8): each thread moves
// pairs of elements, so a warp reads and writes 128 contiguous bytes of a
// row. Needs even row strides and 4-byte aligned bases.
__global__ void __launch_bounds__(256) transpose_pairs_kernel(const uint16_t* in, long long ldi, int rows, int cols,
                                                              uint16_t* out, long long ldo) {
  __shared__ uint16_t tile[64][66];
  const long long r0 = static_cast<long long>(blockIdx.y) * 64, c0 = static_cast<long long>(blockIdx.x) * 64;
  const int tx = threadIdx.x;
  for (int i = threadIdx.y; i < 64; i += 8) {
    const long long r = r0 + i, c = c0 + 2 * tx;
    uint32_t v = 0u;
    if (r < rows && c + 1 < cols) v = __ldg(reinterpret_cast<const uint32_t*>(in + r * ldi + c));
    else if (r < rows && c < cols) v = in[r * ldi + c];
    tile[i][2 * tx] = static_cast<uint16_t>(v & 0xffffu);
    tile[i][2 * tx + 1] = static_cast<uint16_t>(v >> 16);
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 64; i += 8) {
    const long long c = c0 + i, r = r0 + 2 * tx;
    if (c >= cols) continue;
    const uint32_t lo = tile[2 * tx][i], hi = tile[2 * tx + 1][i];
    if (r + 1 < rows) *reinterpret_cast<uint32_t*>(out + c * ldo + r) = lo | (hi << 16);
    else if (r < rows) out[c * ldo + r] = static_cast<uint16_t>(lo);
  }
}

// out[r, c] = bf16(in[r, c]) (row strides ldi, ldo), four columns per thread
// where the row strides and cols allow 16-byte loads.
__global__ void cast4_kernel(const float* in, long long ldi, long long rows, int cols, uint16_t* out,
                             long long ldo) {
  const int q = cols / 4;
  const long long n = rows * q;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / q;
    const int c = 4 * static_cast<int>(i - r * q);
    const float4 v = __ldg(reinterpret_cast<const float4*>(in + r * ldi + c));
    uint2 o;
    o.x = pack_bf16x2(v.x, v.y);
    o.y = pack_bf16x2(v.z, v.w);
    *reinterpret_cast<uint2*>(out + r * ldo + c) = o;
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
// dz | 0 padding]. dK and dV of group g are the sums, in stream order, of the
// per-stream parts dKp, dVp [B, G k + 1, T, dh] of its k routed streams (and
// of the shared head for group 0); each of dQ, dK, dV arrives in two parts
// [2][...] that are added here. Each thread writes 8 adjacent columns;
// the segment bounds before dz are multiples of 32, so 8 columns never
// straddle two of them.
__global__ void pack_grads_kernel(const float* dQr, const float* dQs, const float* dKp, const float* dVp,
                                  const float* dz, const int32_t* idx, uint16_t* Y, long long R, int T, int G,
                                  int M, int k, int dh, int ld) {
  const int N = G * M, gk = G * k, c1 = N * dh, c2 = c1 + dh, c3 = c2 + G * dh, c4 = c3 + G * dh, c5 = c4 + N;
  const int per_row = ld / 8;
  const long long n = R * per_row;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / per_row;
    const int c = 8 * static_cast<int>(i - r * per_row);
    const long long bb = r / T, t = r - bb * T;
    float v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) v[q] = 0.0f;
    auto add8 = [&](const float* src) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(src)), b = __ldg(reinterpret_cast<const float4*>(src) + 1);
      v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
      v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
    };
    // Every attention gradient comes in two parts (the two halves of the
    // tiles an attention-backward CTA pair covers), added in a fixed order.
    if (c < c1) {
      const int e = c / dh, col = c - e * dh, g = e / M, j = e - g * M;
      const int32_t* ip = idx + (r * G + g) * k;
      for (int s = 0; s < k; ++s)
        if (ip[s] == j)
          for (int hf = 0; hf < 2; ++hf) add8(dQr + hf * R * gk * dh + ((r * G + g) * k + s) * dh + col);
    } else if (c < c2) {
      for (int hf = 0; hf < 2; ++hf) add8(dQs + hf * R * dh + r * dh + (c - c1));
    } else if (c < c4) {
      const bool is_k = c < c3;
      const int x = c - (is_k ? c2 : c3), g = x / dh, col = x - g * dh;
      const float* part = is_k ? dKp : dVp;
      const long long half_sz = R * (gk + 1) * dh;
      for (int hf = 0; hf < 2; ++hf) {
        for (int s = 0; s < k; ++s) add8(part + hf * half_sz + ((bb * (gk + 1) + g * k + s) * T + t) * dh + col);
        if (g == 0) add8(part + hf * half_sz + ((bb * (gk + 1) + gk) * T + t) * dh + col);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (c + q < c5) v[q] = dz[r * N + (c + q - c4)];
    }
    uint4 o;
    o.x = pack_bf16x2(v[0], v[1]);
    o.y = pack_bf16x2(v[2], v[3]);
    o.z = pack_bf16x2(v[4], v[5]);
    o.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4*>(Y + r * ld + c) = o;
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
  if (sizeof(TI) == 2 && ((ldi | ldo) & 1) == 0 &&
      ((reinterpret_cast<uintptr_t>(in) | reinterpret_cast<uintptr_t>(out)) & 3u) == 0) {
    const dim3 grid(static_cast<unsigned>((cols + 63) / 64), static_cast<unsigned>((rows + 63) / 64));
    if (grid.y > 65535u) return cudaErrorInvalidConfiguration;
    transpose_pairs_kernel<<<grid, dim3(32, 8), 0, static_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const uint16_t*>(in), ldi, rows, cols, out, ldo);
    return cudaGetLastError();
  }
  const dim3 grid(static_cast<unsigned>((cols + 31) / 32), static_cast<unsigned>((rows + 31) / 32));
  if (grid.y > 65535u) return cudaErrorInvalidConfiguration;
  transpose_kernel<TI><<<grid, dim3(32, 8), 0, static_cast<cudaStream_t>(stream)>>>(in, ldi, rows, cols, out, ldo);
  return cudaGetLastError();
}
template int bwd_transpose<uint16_t>(const uint16_t*, long long, int, int, uint16_t*, long long, void*);
template int bwd_transpose<float>(const float*, long long, int, int, uint16_t*, long long, void*);

int bwd_cast(const float* in, long long ldi, long long rows, int cols, uint16_t* out, long long ldo, void* stream) {
  if (((ldi | ldo | cols) & 3) == 0 &&
      ((reinterpret_cast<uintptr_t>(in) & 15u) | (reinterpret_cast<uintptr_t>(out) & 7u)) == 0)
    cast4_kernel<<<1184, 256, 0, static_cast<cudaStream_t>(stream)>>>(in, ldi, rows, cols, out, ldo);
  else
    cast_kernel<<<1024, 256, 0, static_cast<cudaStream_t>(stream)>>>(in, ldi, rows, cols, out, ldo);
  return cudaGetLastError();
}

int bwd_pack(const gqe_config& c, const float* dQr, const float* dQs, const float* dKp, const float* dVp,
             const float* dz, const int32_t* idx, uint16_t* Y, int ld, void* stream) {
  const long long R = static_cast<long long>(c.B) * c.T;
  pack_grads_kernel<<<1184, 256, 0, static_cast<cudaStream_t>(stream)>>>(dQr, dQs, dKp, dVp, dz, idx, Y, R, c.T,
                                                                         c.G, c.M, c.k, c.d_head, ld);
  return cudaGetLastError();
}

int bwd_slots_router(const gqe_config& c, const uint16_t* x, const float* W_r, const float* b_r, float* zl,
                     const int32_t* idx, const float* omega, const uint16_t* slots, const float* dS, float* dOr,
                     float* dOs, float* dz, uint16_t* dO16, float* Drow, void* stream) {
  const long long R = static_cast<long long>(c.B) * c.T;
  const int N = c.G * c.M;
  const int smem = c.d_model * N * static_cast<int>(sizeof(float)) + kLogitRows * c.d_model * 2;
  cudaError_t e = static_cast<cudaError_t>(ensure_smem<logits_kernel>(smem));
  if (e != cudaSuccess) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  logits_kernel<<<static_cast<unsigned>((R + kLogitRows - 1) / kLogitRows), 256, smem, st>>>(x, W_r, b_r, zl, R,
                                                                                           c.d_model, N);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  SlotArgs a{x,  W_r, b_r,       zl,  idx,    omega,  slots,    dS,      dOr, dOs, dz,
             dO16, Drow, c.d_model, c.G, c.M, c.k, c.d_head, c.T, (c.T + 63) / 64 * 64};
  slot_router_bwd_kernel<<<static_cast<unsigned>(R), 256, 0, st>>>(a);
  return cudaGetLastError();
}

int bwd_colsum(const float* dz, float* db, long long R, int N, void* stream) {
  colsum_kernel<<<N, 256, 0, static_cast<cudaStream_t>(stream)>>>(dz, db, R, N);
  return cudaGetLastError();
}

}  // namespace gqe
