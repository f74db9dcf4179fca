// Decode step (the next row after the prefill path): one new token per
// sequence against its dense, unchanged K/V cache ("the Key-Value projections
// and the KV cache stay dense and unchanged": gist.science Technical Summary,
// Dense KV path). The router, the routed + shared Q projection, the K/V of
// the new token (written straight into the cache at its position) and the
// weighted slot + W_O reuse the prefill kernels at T = 1; this file holds the
// attention of the new token's query heads against the cache.
//
// Attention of one token is a matrix-vector product over the cache, bound by
// HBM (the cache is read once per step): it runs on the CUDA cores, split
// over the keys. A CTA takes 256 keys of one (sequence, group) and every
// query head of that group (GQE: the k routed slots, plus the shared head in
// group 0; dense: the M heads), so each K/V row is read once for all of
// them; it writes the chunk's unnormalised output and (max, sum) per head.
// A second kernel merges the chunks: O = sum_c 2^(m_c - m) O_c / sum_c
// 2^(m_c - m) l_c.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cmath>

#include "gqe_internal.h"
#include "ptx.cuh"

namespace gqe {

namespace decode_impl {

constexpr int kCh = 256;      // keys per CTA (one per thread in the score phase)
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct DecodeArgs {
  const uint16_t* Kc;  // [B][G][cap][dh]
  const uint16_t* Vc;
  int B, G, cap, T;    // T keys: the cache after the step (new token at T - 1)
  int H;               // heads per group, maximum over the groups
  int dense;           // 0: GQE heads (Q = Qv [B][G][k][dh], Qs [B][dh]); 1: dense (Q [B][G*M][dh])
  int k, M;
  const uint16_t* Q;
  const uint16_t* Qs;
  float* part_o;       // [B][G][n_ch][H][dh]
  float2* part_ml;     // [B][G][n_ch][H]
  int n_ch;
  uint16_t* out;       // [B][ldo]
  int ldo;
  float scale_log2;    // log2(e) / sqrt(dh)
};

__device__ __forceinline__ int heads_of(const DecodeArgs& a, int g) {
  return a.dense ? a.M : a.k + (g == 0 ? 1 : 0);
}
// Query of head h of group g (GQE: h < k routed slot h, h == k the shared head).
template <int DH>
__device__ __forceinline__ const uint16_t* query_of(const DecodeArgs& a, int b, int g, int h) {
  if (a.dense) return a.Q + (static_cast<size_t>(b) * a.G * a.M + g * a.M + h) * DH;
  if (h < a.k) return a.Q + ((static_cast<size_t>(b) * a.G + g) * a.k + h) * DH;
  return a.Qs + static_cast<size_t>(b) * DH;
}
// Output column block (in head units) of head h of group g.
__device__ __forceinline__ int column_of(const DecodeArgs& a, int g, int h) {
  if (a.dense) return g * a.M + h;
  return h < a.k ? g * a.k + h : a.G * a.k;
}

__device__ __forceinline__ float bf16f(uint16_t v) { return __uint_as_float(static_cast<uint32_t>(v) << 16); }

// O phase: thread t takes 16-byte column chunk t % (DH/8) of the rows of row
// group t / (DH/8) (8 rows of a KV tile per pass for DH = 64).
template <int DH>
struct OShape {
  static constexpr int CPR = DH / 8;            // 16-byte chunks per row
  static constexpr int NG = kThreads / CPR;     // row groups (32 for DH = 64)
  static constexpr int PASSES = kCh / NG;       // rows per thread
};

// Dynamic shared memory: q [H][DH], scores / probabilities [H][kCh], warp
// partials [kWarps][H] (max, then sum), O partials [row groups][H][DH].
template <int DH>
size_t partial_smem(int H) {
  return static_cast<size_t>(H) * (DH + kCh + 2 * kWarps + OShape<DH>::NG * DH) * 4 + 2 * H * 4;
}

// HM: a bound on the heads per group (2, 4, 8 or 16) sizing the registers.
template <int DH, int HM>
__global__ void __launch_bounds__(kThreads) decode_partial_kernel(DecodeArgs a) {
  using OS = OShape<DH>;
  constexpr int NG = OS::NG;
  pdl_wait();
  pdl_launch_dependents();
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int H = heads_of(a, g);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  extern __shared__ __align__(16) float dsm[];
  float* qsm = dsm;                       // [H][DH], pre-scaled
  float* sc = qsm + a.H * DH;             // [H][kCh]
  float* wred = sc + a.H * kCh;           // [kWarps][H] then [kWarps][H]
  float* wsum = wred + kWarps * a.H;
  float* ored = wsum + kWarps * a.H;      // [NG][H][DH]
  float* mh = ored + NG * a.H * DH;       // [H] chunk max
  float* lh = mh + a.H;                   // [H] chunk sum

  for (int i = tid; i < H * DH; i += kThreads) {
    const int h = i / DH, d = i - h * DH;
    qsm[i] = bf16f(query_of<DH>(a, b, g, h)[d]) * a.scale_log2;
  }
  __syncthreads();

  // Scores: thread t takes key u = c * kCh + t.
  const size_t kv0 = (static_cast<size_t>(b) * a.G + g) * a.cap;
  const int u = c * kCh + tid;
  const bool valid = u < a.T;
  {
    float kr[DH];
    if (valid) {
      const uint4* kp = reinterpret_cast<const uint4*>(a.Kc + (kv0 + u) * DH);
#pragma unroll
      for (int q = 0; q < DH / 8; ++q) {
        const uint4 v = __ldg(kp + q);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          kr[8 * q + 2 * i] = __uint_as_float(w[i] << 16);
          kr[8 * q + 2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
      }
    }
    for (int h = 0; h < H; ++h) {
      float s = -INFINITY;
      if (valid) {
        float s4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int d = 0; d < DH; ++d) s4[d & 3] = fmaf(qsm[h * DH + d], kr[d], s4[d & 3]);
        s = (s4[0] + s4[1]) + (s4[2] + s4[3]);
      }
      sc[h * kCh + tid] = s;
      float m = s;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) wred[warp * a.H + h] = m;
    }
  }
  __syncthreads();
  for (int h = 0; h < H; ++h) {
    float m = wred[h];
    for (int w = 1; w < kWarps; ++w) m = fmaxf(m, wred[w * a.H + h]);
    const float p = valid ? exp2f(sc[h * kCh + tid] - m) : 0.0f;
    sc[h * kCh + tid] = p;
    float s = p;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) wsum[warp * a.H + h] = s;
    if (tid == 0) mh[h] = m;
  }
  __syncthreads();
  if (tid < H) {
    float s = 0.0f;
    for (int w = 0; w < kWarps; ++w) s += wsum[w * a.H + tid];
    lh[tid] = s;
  }

  // O: thread t takes columns 8*cc .. 8*cc+7 (cc = t % CPR) of rows rg,
  // rg + NG, ... (rg = t / CPR): 16-byte loads, all rows of a thread in flight.
  const int cc = tid % OS::CPR, rg = tid / OS::CPR;
  const int n_keys = min(kCh, a.T - c * kCh);
  uint4 vr[OS::PASSES];
#pragma unroll
  for (int q = 0; q < OS::PASSES; ++q) {
    const int ul = rg + q * NG;
    vr[q] = ul < n_keys ? __ldg(reinterpret_cast<const uint4*>(a.Vc + (kv0 + c * kCh + ul) * DH) + cc)
                        : make_uint4(0u, 0u, 0u, 0u);
  }
  float acc[HM][8];
#pragma unroll
  for (int h = 0; h < HM; ++h)
#pragma unroll
    for (int x = 0; x < 8; ++x) acc[h][x] = 0.0f;
#pragma unroll
  for (int q = 0; q < OS::PASSES; ++q) {
    const int ul = rg + q * NG;
    const uint32_t w[4] = {vr[q].x, vr[q].y, vr[q].z, vr[q].w};
    float v[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
#pragma unroll
    for (int h = 0; h < HM; ++h) {
      if (h < H) {
        const float p = ul < n_keys ? sc[h * kCh + ul] : 0.0f;
#pragma unroll
        for (int x = 0; x < 8; ++x) acc[h][x] = fmaf(p, v[x], acc[h][x]);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < HM; ++h) {
    if (h < H) {
      float4* dst = reinterpret_cast<float4*>(ored + (rg * a.H + h) * DH + 8 * cc);
      dst[0] = make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
      dst[1] = make_float4(acc[h][4], acc[h][5], acc[h][6], acc[h][7]);
    }
  }
  __syncthreads();
  const size_t blk = ((static_cast<size_t>(b) * a.G + g) * a.n_ch + c) * a.H;
  for (int i = tid; i < H * DH; i += kThreads) {
    const int h = i / DH, d = i - h * DH;
    float s = 0.0f;
    for (int q = 0; q < NG; ++q) s += ored[(q * a.H + h) * DH + d];
    a.part_o[(blk + h) * DH + d] = s;
  }
  if (tid < H) a.part_ml[blk + tid] = make_float2(mh[tid], lh[tid]);
}

// One CTA per (group, sequence), one thread per (head, dim).
template <int DH>
__global__ void __launch_bounds__(1024) decode_merge_kernel(DecodeArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int g = blockIdx.x, b = blockIdx.y;
  const int H = heads_of(a, g);
  const int h = threadIdx.x / DH, d = threadIdx.x % DH;
  if (h >= H) return;
  const size_t blk0 = (static_cast<size_t>(b) * a.G + g) * a.n_ch;
  float m = -INFINITY;
#pragma unroll 8
  for (int c = 0; c < a.n_ch; ++c) m = fmaxf(m, a.part_ml[(blk0 + c) * a.H + h].x);
  float o = 0.0f, l = 0.0f;
#pragma unroll 8
  for (int c = 0; c < a.n_ch; ++c) {
    const float2 ml = a.part_ml[(blk0 + c) * a.H + h];
    const float w = exp2f(ml.x - m);
    l = fmaf(w, ml.y, l);
    o = fmaf(w, a.part_o[((blk0 + c) * a.H + h) * DH + d], o);
  }
  const __nv_bfloat16 r = __float2bfloat16_rn(o / l);
  a.out[static_cast<size_t>(b) * a.ldo + column_of(a, g, h) * DH + d] =
      *reinterpret_cast<const uint16_t*>(&r);
}

template <int DH, int HM>
int launch_partial(const DecodeArgs& a, void* stream) {
  const size_t smem = partial_smem<DH>(a.H);
  const int e = ensure_smem<decode_partial_kernel<DH, HM>>(static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_partial_kernel<DH, HM>, dim3(a.n_ch, a.G, a.B), dim3(kThreads), smem,
                    stream, a);
}

template <int DH>
int launch(const DecodeArgs& a, void* stream) {
  const int e = a.H <= 2   ? launch_partial<DH, 2>(a, stream)
                : a.H <= 4 ? launch_partial<DH, 4>(a, stream)
                : a.H <= 8 ? launch_partial<DH, 8>(a, stream)
                           : launch_partial<DH, 16>(a, stream);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_merge_kernel<DH>, dim3(a.G, a.B), dim3(a.H * DH), 0, stream, a);
}

}  // namespace decode_impl
using namespace decode_impl;

int decode_heads(const gqe_config& c, bool dense) { return dense ? c.M : c.k + 1; }

size_t decode_attention_ws_bytes(const gqe_config& c, bool dense) {
  const size_t n_ch = (static_cast<size_t>(c.T) + kCh - 1) / kCh;
  const size_t units = static_cast<size_t>(c.B) * c.G * n_ch * decode_heads(c, dense);
  return ((units * c.d_head * 4 + 255) / 256) * 256 + units * 8;
}

int decode_attention(const gqe_config& c, bool dense, const uint16_t* Q, const uint16_t* Qs,
                     const uint16_t* Kc, const uint16_t* Vc, int cap, uint16_t* out, int ldo,
                     void* ws, void* stream) {
  DecodeArgs a{};
  a.Kc = Kc;
  a.Vc = Vc;
  a.B = c.B;
  a.G = c.G;
  a.cap = cap;
  a.T = c.T;
  a.dense = dense ? 1 : 0;
  a.k = c.k;
  a.M = c.M;
  a.H = decode_heads(c, dense);
  if (a.H > 16) return cudaErrorInvalidConfiguration;
  a.Q = Q;
  a.Qs = Qs;
  a.n_ch = (c.T + kCh - 1) / kCh;
  const size_t units = static_cast<size_t>(c.B) * c.G * a.n_ch * a.H;
  char* w = static_cast<char*>(ws);
  a.part_o = reinterpret_cast<float*>(w);
  a.part_ml = reinterpret_cast<float2*>(w + ((units * c.d_head * 4 + 255) / 256) * 256);
  a.out = out;
  a.ldo = ldo;
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(c.d_head)));
  if (c.d_head == 64) return launch<64>(a, stream);
  return launch<32>(a, stream);
}

}  // namespace gqe
