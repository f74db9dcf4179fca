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
// over the keys. Every CTA handles one (sequence, group) and every query head
// of that group (GQE: the k routed slots, plus the shared head in group 0;
// dense: the M heads), so each K/V row is read once for all of them, and
// writes unnormalised outputs with (max, sum) per head. A second kernel
// merges them: O = sum_c 2^(m_c - m) O_c / sum_c 2^(m_c - m) l_c.
//  - decode_span_kernel (d_head = 64, up to 4 heads, cache of 256+ rows): a
//    span of 256-key chunks per CTA, streamed by TMA through a 3-deep ring,
//    online softmax per warp;
//  - decode_partial_kernel (the rest): 256 keys per CTA, loaded by its
//    threads.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cmath>

#include "gqe_internal.h"
#include "ptx.cuh"
#include "tmap.h"

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

// ---------------------------------------------------------------------------
// Streaming form for d_head = 64 and at most 4 heads per group: one CTA takes
// a span of consecutive 256-key chunks of one (sequence, group). A producer
// warp streams each chunk's K and V rows (one TMA box of 256 x 64 each,
// 128B-swizzled) through a 3-deep ring, so the cache keeps flowing while the
// consumers compute. Consumer warp w owns keys 32w..32w+31 of every chunk for
// both phases: lane j scores key j against every head, and the warp keeps its
// own running max, sum and output (online softmax), lane l holding output
// dims 2l, 2l+1. The 8 warps' states are combined once at the end of the
// span into one partial per head, which decode_merge_kernel then combines
// over the spans. No block-wide barrier sits inside the key loop.
constexpr int kSpanCh = 256;       // keys per chunk (one TMA box)
constexpr int kSpanStages = 3;
constexpr int kSpanWarps = 8;      // consumer warps
constexpr int kSpanThreads = 32 * (kSpanWarps + 1);
constexpr int kSpanMaxHeads = 4;
constexpr int kSpanTile = kSpanCh * 64 * 2;  // bytes of one K (or V) box

constexpr size_t span_smem() {
  return 1024 + 2ull * kSpanStages * kSpanTile + kSpanMaxHeads * 64 * 4 +
         kSpanWarps * kSpanMaxHeads * (64 + 2) * 4 + 2 * kSpanStages * 8 + 16;
}

template <int HM>
__global__ void __launch_bounds__(kSpanThreads, 1)
    decode_span_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       DecodeArgs a, int span_ch) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sp = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sK = sp;                                         // [stages][256 rows x 128 B]
  uint8_t* sV = sK + kSpanStages * kSpanTile;
  float* qsm = reinterpret_cast<float*>(sV + kSpanStages * kSpanTile);  // [HM][64], pre-scaled
  float* wst = qsm + kSpanMaxHeads * 64;                    // [warps][HM][64 acc + m + l]
  uint64_t* full = reinterpret_cast<uint64_t*>(wst + kSpanWarps * kSpanMaxHeads * 66);
  uint64_t* empty = full + kSpanStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kSpanStages);

  const int span = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int H = heads_of(a, g);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n_ch = (a.T + kSpanCh - 1) / kSpanCh;
  const int ch0 = span * span_ch, ch1 = min(n_ch, ch0 + span_ch);
  const int nchunks = ch1 - ch0;
  if (tid == 0) {
    for (int s = 0; s < kSpanStages; ++s) {
      mbar_init(&full[s], 1u);
      mbar_init(&empty[s], kSpanWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kSpanWarps && lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  pdl_wait();  // Q and the new token's K/V row come from earlier kernels
  pdl_launch_dependents();
  for (int i = tid; i < H * 64; i += kSpanThreads) {
    const int h = i / 64, d = i - h * 64;
    qsm[i] = bf16f(query_of<64>(a, b, g, h)[d]) * a.scale_log2;
  }
  __syncthreads();

  const int zkv = b * a.G + g;
  if (warp == kSpanWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      for (int i = 0; i < nchunks; ++i) {
        const int s = i % kSpanStages;
        const uint32_t ph = (i / kSpanStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) break;
        mbar_arrive_expect_tx(&full[s], 2 * kSpanTile);
        tma_load_3d(sK + s * kSpanTile, &tmK, &full[s], 0, (ch0 + i) * kSpanCh, zkv);
        tma_load_3d(sV + s * kSpanTile, &tmV, &full[s], 0, (ch0 + i) * kSpanCh, zkv);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    float m[HM], l[HM], acc[HM][2];
#pragma unroll
    for (int h = 0; h < HM; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.0f;
      acc[h][0] = acc[h][1] = 0.0f;
    }
    const int r = warp * 32 + lane;  // this lane's key row in every chunk
    for (int i = 0; i < nchunks; ++i) {
      const int s = i % kSpanStages;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (i / kSpanStages) & 1, abort_flag))) break;
      const uint8_t* kt = sK + s * kSpanTile;
      const uint8_t* vt = sV + s * kSpanTile;
      const bool valid = (ch0 + i) * kSpanCh + r < a.T;
      // Scores of key r: its K row (16-byte chunks at their swizzled places).
      float sc[HM];
#pragma unroll
      for (int h = 0; h < HM; ++h) sc[h] = 0.0f;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        const uint4 kv = *reinterpret_cast<const uint4*>(kt + r * 128 + ((cc ^ (r & 7)) << 4));
        const uint32_t w[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int h = 0; h < HM; ++h) {
          if (h < H) {
            const float4 q0 = *reinterpret_cast<const float4*>(qsm + h * 64 + cc * 8);
            const float4 q1 = *reinterpret_cast<const float4*>(qsm + h * 64 + cc * 8 + 4);
            sc[h] = fmaf(q0.x, __uint_as_float(w[0] << 16), sc[h]);
            sc[h] = fmaf(q0.y, __uint_as_float(w[0] & 0xffff0000u), sc[h]);
            sc[h] = fmaf(q0.z, __uint_as_float(w[1] << 16), sc[h]);
            sc[h] = fmaf(q0.w, __uint_as_float(w[1] & 0xffff0000u), sc[h]);
            sc[h] = fmaf(q1.x, __uint_as_float(w[2] << 16), sc[h]);
            sc[h] = fmaf(q1.y, __uint_as_float(w[2] & 0xffff0000u), sc[h]);
            sc[h] = fmaf(q1.z, __uint_as_float(w[3] << 16), sc[h]);
            sc[h] = fmaf(q1.w, __uint_as_float(w[3] & 0xffff0000u), sc[h]);
          }
        }
      }
      // Online softmax per head over this warp's 32 keys.
      float p[HM];
#pragma unroll
      for (int h = 0; h < HM; ++h) {
        const float sv = valid ? sc[h] : -INFINITY;
        float cm = sv;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
        const float mn = fmaxf(m[h], cm);
        // A warp whose keys so far are all past the end keeps m = -inf.
        const float alpha = mn == -INFINITY ? 1.0f : exp2f(m[h] - mn);
        p[h] = mn == -INFINITY ? 0.0f : exp2f(sv - mn);
        l[h] = fmaf(l[h], alpha, p[h]);
        acc[h][0] *= alpha;
        acc[h][1] *= alpha;
        m[h] = mn;
      }
      // O += P V over the warp's keys: lane l holds dims 2l, 2l+1.
      const int cw = lane >> 2, off = (lane & 3) * 4;
#pragma unroll 8
      for (int jj = 0; jj < 32; ++jj) {
        const int rr = warp * 32 + jj;
        const uint32_t v2 = *reinterpret_cast<const uint32_t*>(vt + rr * 128 + ((cw ^ (rr & 7)) << 4) + off);
        const float v0 = __uint_as_float(v2 << 16), v1 = __uint_as_float(v2 & 0xffff0000u);
#pragma unroll
        for (int h = 0; h < HM; ++h) {
          const float pj = __shfl_sync(0xffffffffu, p[h], jj);
          acc[h][0] = fmaf(pj, v0, acc[h][0]);
          acc[h][1] = fmaf(pj, v1, acc[h][1]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    // This warp's state: m (uniform), l summed over the lanes, O per lane.
#pragma unroll
    for (int h = 0; h < HM; ++h) {
      float ls = l[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
      float* st = wst + (warp * kSpanMaxHeads + h) * 66;
      st[2 * lane] = acc[h][0];
      st[2 * lane + 1] = acc[h][1];
      if (lane == 0) {
        st[64] = m[h];
        st[65] = ls;
      }
    }
  }
  __syncthreads();
  // Combine the warps: thread (h, d).
  if (tid < H * 64) {
    const int h = tid / 64, d = tid - h * 64;
    float mx = -INFINITY;
    for (int w = 0; w < kSpanWarps; ++w) mx = fmaxf(mx, wst[(w * kSpanMaxHeads + h) * 66 + 64]);
    float o = 0.0f, ls = 0.0f;
    for (int w = 0; w < kSpanWarps; ++w) {
      const float* st = wst + (w * kSpanMaxHeads + h) * 66;
      const float wt = st[64] == -INFINITY ? 0.0f : exp2f(st[64] - mx);
      o = fmaf(wt, st[d], o);
      ls = fmaf(wt, st[65], ls);
    }
    const size_t blk = ((static_cast<size_t>(b) * a.G + g) * a.n_ch + span) * a.H;
    a.part_o[(blk + h) * 64 + d] = o;
    if (d == 0) a.part_ml[blk + h] = make_float2(mx, ls);
  }
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

template <int HM>
int launch_span(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a, int span_ch,
                void* stream) {
  const int e = ensure_smem<decode_span_kernel<HM>>(static_cast<int>(span_smem()));
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_span_kernel<HM>, dim3(a.n_ch, a.G, a.B), dim3(kSpanThreads), span_smem(), stream,
                    tk, tv, a, span_ch);
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
  if (c.d_head == 64 && a.H <= kSpanMaxHeads && cap >= kSpanCh) {
    // Streaming form: spans of chunks, about 8 CTAs per SM over the whole grid.
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int n_ch0 = (c.T + kSpanCh - 1) / kSpanCh;
    const long long bg = static_cast<long long>(c.B) * c.G;
    int n_span = static_cast<int>((8ll * sms + bg - 1) / bg);
    n_span = n_span < 1 ? 1 : n_span > n_ch0 ? n_ch0 : n_span;
    const int span_ch = (n_ch0 + n_span - 1) / n_span;
    a.n_ch = (n_ch0 + span_ch - 1) / span_ch;  // partials per (sequence, group): one per span
    CUtensorMap tk, tv;
    const uint64_t rows = static_cast<uint64_t>(c.B) * c.G;
    if (!make_tmap_bf16_3d(&tk, Kc, 64, static_cast<uint64_t>(cap), rows, 64, kSpanCh) ||
        !make_tmap_bf16_3d(&tv, Vc, 64, static_cast<uint64_t>(cap), rows, 64, kSpanCh))
      return cudaErrorInvalidValue;
    const int e = a.H <= 2 ? launch_span<2>(tk, tv, a, span_ch, stream) : launch_span<4>(tk, tv, a, span_ch, stream);
    if (e != cudaSuccess) return e;
    return launch_pdl(decode_merge_kernel<64>, dim3(a.G, a.B), dim3(a.H * 64), 0, stream, a);
  }
  if (c.d_head == 64) return launch<64>(a, stream);
  return launch<32>(a, stream);
}

}  // namespace gqe
