// Router (steps a1-a4 of the GQE layer): per-token logits x . W_r + b in
// fp32, softmax inside each of the G groups, top-k per group with ties to the
// lower expert index, and the two renormalisations of the selected
// probabilities. ("Grouped Query Experts: Mixture-of-Experts on GQA
// Self-Attention": router choosing k query-head experts in every GQA group,
// gist.science Technical Summary, Methodology; softmax before top-k inside
// the group, pptc.cn blog section 7.)
//
// The logits are a small fp32 GEMM on the CUDA cores. A CTA takes a block of
// TB tokens (TB * NP = 128 * TPT logits); W_r (zero padded to NP columns) and
// the block's x rows sit in shared memory. Warp w of W (16, or 8 when d is
// not a multiple of 128) sums rows [w d/W, (w+1) d/W) of the dot products;
// each thread keeps TPT tokens x 4 experts, so one 16-byte W_r read (one
// shared-memory pass per quarter warp) feeds 4 TPT FMAs. Large batches take
// TPT = 6 (4 where that block does not fit in shared memory, e.g. 32 experts
// at d = 1024), small ones TPT = 2 so that the blocks spread over the SMs. The W warp partials are then added in warp
// order, so every logit is one fixed sequence of roundings (the result is
// deterministic and the same for every TPT). The threads then take the
// (token, group) pairs and decide.
//
// Exact selection: each fp32 logit carries the bound
//   |z_fp32 - z| <= gamma_h * (||x||_1 * max_i |W_r[i,e]| + |b_e|),
// h = d/W + W roundings on its longest path (d/W FMAs in one warp, W - 1
// adds of the warp partials, the bias add), gamma_h = h u / (1 - h u), u = 2^-24 (Higham,
// "Accuracy and Stability of Numerical Algorithms", 2nd ed., sec. 3.1). A
// group whose top-k decision is not certain under these intervals (computed
// with directed rounding) recomputes its logits in fp64 (products of a bf16
// and an fp32 value are exact in fp64), and the fp64 decision is certified
// the same way with its own path length and u = 2^-53. A group that even
// the fp64 intervals do not settle (exact ties, or logits closer than about
// 1e-15 of their size) is decided on the exact logits: every product is an
// integer multiple of 2^-282, so the sum is accumulated exactly as a
// 576-bit integer in 32-bit limbs (kept in 64-bit words so that no carry is
// lost) and compared exactly. The selection therefore equals the
// exact-arithmetic one in every case.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <atomic>

#include "gqe_internal.h"
#include "ptx.cuh"

namespace gqe {

namespace router_impl {

constexpr int kMaxRouterWarps = 16;

// Tokens per CTA block: lanes are (token lane tt, expert quad et) with NP/4
// quads, so a warp covers 128/NP token lanes of TPT tokens each.
__host__ __device__ constexpr int router_tb(int NP, int TPT) { return TPT * 128 / NP; }
// Warps per CTA: warp w sums rows [w d/W, (w+1) d/W), a multiple of 8 rows.
__host__ __device__ constexpr int router_warps(int d) { return d % 128 == 0 ? 16 : 8; }

__device__ __forceinline__ float bf16_to_f32(uint16_t v) {
  return __uint_as_float(static_cast<uint32_t>(v) << 16);
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

struct RouterArgs {
  const uint16_t* x;
  const float* W_r;
  const float* b_r;
  int32_t* idx;
  float* r;
  float* omega;
  int R, d, G, M, k, N;
  int wmode;  // omega: 0 = p / selected p of all groups, 1 = r / G, 2 = p
};

// Uncertain groups per round of the fp64 fallback.
__host__ __device__ constexpr int router_fb(int NP) { return NP >= 64 ? 1 : NP >= 32 ? 2 : 4; }

// Dynamic shared memory of one CTA (byte offsets). The warp partials
// [warp][TB][NP] share their space with the block's x rows: they are written
// once every warp has finished reading x, and the next block's rows are
// fetched once the partials have been summed.
struct RouterLayout {
  size_t w, xs, zd, sel, fb, zf, ez, wmax, bsm, nx, ps, dn, list, total;
};
__host__ __device__ inline RouterLayout router_layout(int d, int NP, int TPT) {
  const int TB = router_tb(NP, TPT), W = router_warps(d);
  const size_t xbytes = static_cast<size_t>(TB) * (d + 8) * 2;  // x [TB][d + 8]
  const size_t pbytes = static_cast<size_t>(W) * TB * NP * 4;   // partials [warp][TB][NP]
  RouterLayout L;
  size_t o = 0;
  L.w = o;     o += static_cast<size_t>(d) * NP * 4;                  // W_r [d][NP]
  L.xs = o;    o += ((xbytes > pbytes ? xbytes : pbytes) + 15) & ~static_cast<size_t>(15);
  L.zd = o;    o += static_cast<size_t>(TB) * NP * 8;                 // fp64 logits
  L.sel = o;   o += static_cast<size_t>(TB) * NP * 8;                 // selection mask per pair
  L.fb = o;    o += static_cast<size_t>(router_fb(NP)) * W * NP * 8;   // fp64 warp partials (fallback)
  L.zf = o;    o += static_cast<size_t>(TB) * NP * 4;                 // fp32 logits
  L.ez = o;    o += static_cast<size_t>(TB) * NP * 4;                 // exp(z - group max)
  L.wmax = o;  o += NP * 4;                                            // max_i |W_r[i, e]|
  L.bsm = o;   o += NP * 4;                                            // bias
  L.nx = o;    o += TB * 4;                                            // ||x||_1
  L.ps = o;    o += static_cast<size_t>(TB) * NP * 4;                 // selected mass per pair
  L.dn = o;    o += static_cast<size_t>(TB) * NP * 4;                 // softmax denominator per pair
  L.list = o;  o += static_cast<size_t>(TB) * NP * 4;                 // uncertain pairs
  L.total = (o + 15) & ~static_cast<size_t>(15);
  return L;
}

// Top-k of one group's M logits (descending, ties to the lower index) as a
// bitmask over j.
template <typename V>
__device__ __forceinline__ uint64_t group_topk(const V* zg, int M, int k) {
  uint64_t sel = 0;
  for (int s = 0; s < k; ++s) {
    V best = -INFINITY;
    int bj = -1;
    for (int j = 0; j < M; ++j) {
      if (!((sel >> j) & 1ull) && (bj < 0 || zg[j] > best)) {
        best = zg[j];
        bj = j;
      }
    }
    sel |= 1ull << bj;
  }
  return sel;
}

// Group softmax of pair (t, g) from its logits zg (fp32, or fp64 for a
// group decided in fp64): exp(z - max) into ez, the denominator into *den,
// and the selected mass (sum of the selected probabilities) returned.
template <typename V>
__device__ __forceinline__ float group_softmax(const V* zg, int M, uint64_t sel, float* ez, float* den) {
  V zmax = zg[0];
  for (int j = 1; j < M; ++j) zmax = zg[j] > zmax ? zg[j] : zmax;
  float dsum = 0.0f;
  for (int j = 0; j < M; ++j) {
    const float e = expf(static_cast<float>(zg[j] - zmax));
    ez[j] = e;
    dsum += e;
  }
  float psel = 0.0f;
  for (int j = 0; j < M; ++j)
    if ((sel >> j) & 1ull) psel += ez[j] / dsum;
  *den = dsum;
  return psel;
}

// Exact logits. A bf16 value is m * 2^(E' - 134) with an 8-bit integer m
// and E' = max(E, 1) (E its biased exponent); an fp32 value is m * 2^(E' -
// 150) with a 24-bit m. A product is therefore a 32-bit integer times 2^p,
// p + 282 in [0, 508], and the bias a 24-bit integer times 2^p, p + 282 in
// [133, 386]. W_r sits in shared memory, so d < 2^15, and the sum of d + 1
// terms stays below 2^556 (in units of 2^-282): 18 limbs of 32 bits hold it,
// the top one signed. The limbs are 64-bit words and each receives fewer
// than 2^16 additions below 2^32, so nothing overflows before the carries
// are propagated.
constexpr int kExactLimbs = 18;

// Adds sign * m * 2^bitpos (m < 2^32) to the shared limbs.
__device__ __forceinline__ void exact_add(long long* limbs, uint32_t m, int bitpos, bool neg) {
  const unsigned long long v = static_cast<unsigned long long>(m) << (bitpos & 31);
  const int l = bitpos >> 5;
  const unsigned long long lo = v & 0xffffffffull, hi = v >> 32;
  auto* u = reinterpret_cast<unsigned long long*>(limbs);
  if (lo) atomicAdd(u + l, neg ? 0ull - lo : lo);
  if (hi) atomicAdd(u + l + 1, neg ? 0ull - hi : hi);
}

__device__ __forceinline__ void exact_add_product(long long* limbs, uint16_t xb, float w) {
  const uint32_t wb = __float_as_uint(w);
  const int ex = (xb >> 7) & 0xff, ew = (wb >> 23) & 0xff;
  const uint32_t mx = ex ? (0x80u | (xb & 0x7fu)) : (xb & 0x7fu);
  const uint32_t mw = ew ? (0x800000u | (wb & 0x7fffffu)) : (wb & 0x7fffffu);
  const uint32_t m = mx * mw;
  if (m == 0u) return;
  // exponent (max(ex,1) - 134) + (max(ew,1) - 150), offset by +282
  exact_add(limbs, m, (ex ? ex : 1) + (ew ? ew : 1) - 2, ((xb >> 15) ^ (wb >> 31)) & 1u);
}

__device__ __forceinline__ void exact_add_bias(long long* limbs, float b) {
  const uint32_t bb = __float_as_uint(b);
  const int eb = (bb >> 23) & 0xff;
  const uint32_t m = eb ? (0x800000u | (bb & 0x7fffffu)) : (bb & 0x7fffffu);
  if (m == 0u) return;
  exact_add(limbs, m, (eb ? eb : 1) - 150 + 282, (bb >> 31) & 1u);
}

// Carries the limbs so that limbs 0..16 lie in [0, 2^32) and limb 17 holds
// the signed rest: one canonical form per value.
__device__ __forceinline__ void exact_normalize(long long* limbs) {
  for (int l = 0; l + 1 < kExactLimbs; ++l) {
    const long long c = limbs[l] >> 32;  // floor division by 2^32
    limbs[l] -= c * 4294967296ll;
    limbs[l + 1] += c;
  }
}

// a > b for canonical limbs.
__device__ __forceinline__ bool exact_greater(const long long* a, const long long* b) {
  if (a[kExactLimbs - 1] != b[kExactLimbs - 1]) return a[kExactLimbs - 1] > b[kExactLimbs - 1];
  for (int l = kExactLimbs - 2; l >= 0; --l)
    if (a[l] != b[l]) return a[l] > b[l];
  return false;
}

// Exact decisions of the ne pairs in list (exact ties and logits closer
// than the fp64 bound only), one pair at a time; every thread of the CTA
// calls it. The k selections are taken one by one: each pass computes the
// exact logit of every unselected expert (the whole CTA adds the products
// into shared limbs, cur) and keeps the largest (best), the lower index on
// equality. Out of line: the rare path stays out of the main loop's
// register allocation.
__device__ __noinline__ void exact_decide(const uint16_t* x, int d, int G, int M, int k, const float* Ws,
                                          int NP, const float* bsm, long long* cur, const int* list,
                                          int ne, int row0, const double* zd, float* ez, float* dn,
                                          float* ps, uint64_t* selp, unsigned long long* sel_sh,
                                          int* best_sh) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  long long* best = cur + kExactLimbs;
  for (int v = 0; v < ne; ++v) {
    const int pv = list[v];
    const int tv = pv / G, gv = pv - tv * G;
    const uint16_t* xr = x + static_cast<size_t>(row0 + tv) * d;
    if (tid == 0) *sel_sh = 0ull;
    __syncthreads();
    for (int s = 0; s < k; ++s) {
      if (tid == 0) *best_sh = -1;
      for (int j = 0; j < M; ++j) {
        if ((*sel_sh >> j) & 1ull) continue;  // uniform (shared, set before a barrier)
        const int e = gv * M + j;
        if (tid < kExactLimbs) cur[tid] = 0;
        __syncthreads();
        for (int i = tid; i < d; i += nthr) exact_add_product(cur, __ldg(xr + i), Ws[i * NP + e]);
        if (tid == 0) exact_add_bias(cur, bsm[e]);
        __syncthreads();
        if (tid == 0) {
          exact_normalize(cur);
          if (*best_sh < 0 || exact_greater(cur, best)) {
            for (int l = 0; l < kExactLimbs; ++l) best[l] = cur[l];
            *best_sh = j;
          }
        }
        __syncthreads();
      }
      if (tid == 0) *sel_sh |= 1ull << *best_sh;
      __syncthreads();
    }
    if (tid == 0) {
      const int zo = tv * NP + gv * M;
      ps[pv] = group_softmax(zd + zo, M, *sel_sh, ez + zo, dn + pv);
      selp[pv] = *sel_sh;
    }
    __syncthreads();
  }
}

template <int NP, int WARPS, int TPT>
__global__ void __launch_bounds__(WARPS * 32) router_kernel(RouterArgs a) {
  constexpr int THREADS = WARPS * 32;
  constexpr int TB = router_tb(NP, TPT);
  constexpr int EG = NP / 4;   // expert quads
  constexpr int TG = 32 / EG;  // token lanes per warp; TB == TPT * TG
  static_assert(TB == TPT * TG, "block shape");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ int n_uncertain, n_exact, exact_best;
  __shared__ unsigned long long exact_sel;
  const RouterLayout L = router_layout(a.d, NP, TPT);
  float* Ws = reinterpret_cast<float*>(smem_raw + L.w);
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem_raw + L.xs);
  float* part = reinterpret_cast<float*>(smem_raw + L.xs);  // shares the x rows' space
  double* zd = reinterpret_cast<double*>(smem_raw + L.zd);
  uint64_t* selp = reinterpret_cast<uint64_t*>(smem_raw + L.sel);
  float* zf = reinterpret_cast<float*>(smem_raw + L.zf);
  float* ez = reinterpret_cast<float*>(smem_raw + L.ez);
  float* wmax = reinterpret_cast<float*>(smem_raw + L.wmax);
  float* bsm = reinterpret_cast<float*>(smem_raw + L.bsm);
  float* nxs = reinterpret_cast<float*>(smem_raw + L.nx);
  float* ps = reinterpret_cast<float*>(smem_raw + L.ps);
  float* dn = reinterpret_cast<float*>(smem_raw + L.dn);
  int* list = reinterpret_cast<int*>(smem_raw + L.list);

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int et = lane % EG, tt = lane / EG;
  const int XS = a.d + 8;  // x row stride in shared memory (16-byte pad: no bank conflicts)
  const int cpr = a.d / 8;  // 16-byte chunks per x row
  const int n_blk = (a.R + TB - 1) / TB;

  // Stages the TB rows of a block (rows past R repeat the last row); always
  // commits one cp.async group (empty past the end).
  auto stage_x = [&](int blk) {
    if (blk < n_blk) {
      for (int t = warp; t < TB; t += WARPS) {
        const uint16_t* src = a.x + static_cast<size_t>(min(blk * TB + t, a.R - 1)) * a.d;
        for (int c = lane; c < cpr; c += 32) cp_async_16(smem_u32(xs + t * XS + c * 8), src + c * 8, 16u);
      }
    }
    cp_async_commit();
  };

  pdl_wait();
  pdl_launch_dependents();

  // W_r into shared memory. Each CTA starts at a different chunk so that the
  // CTAs do not all read the same L2 lines at once.
  if (a.N == NP) {
    const int total = a.d * NP / 4;  // 16-byte chunks
    const int rot = static_cast<int>((static_cast<long long>(blockIdx.x) * 256) % total);
    for (int i = tid; i < total; i += THREADS) {
      int j = i + rot;
      if (j >= total) j -= total;
      cp_async_16(smem_u32(Ws + 4 * j), a.W_r + 4 * static_cast<size_t>(j), 16u);
    }
  } else {
    for (int i = tid; i < a.d * NP; i += THREADS) {
      const int row = i / NP, col = i % NP;
      Ws[i] = col < a.N ? a.W_r[static_cast<size_t>(row) * a.N + col] : 0.0f;
    }
  }
  cp_async_commit();
  int blk = blockIdx.x;
  stage_x(blk);
  cp_async_wait<1>();  // this thread's part of W_r is in
  for (int e = tid; e < NP; e += THREADS) bsm[e] = (e < a.N && a.b_r != nullptr) ? a.b_r[e] : 0.0f;
  __syncthreads();
  // max_i |W_r[i, e]|: thread t scans column t % NP over every (THREADS/NP)-th
  // row, then one thread per column combines the parts.
  {
    constexpr int parts = THREADS / NP;
    const int col = tid % NP, p0 = tid / NP;
    float m0 = 0.0f, m1 = 0.0f, m2 = 0.0f, m3 = 0.0f;
    int row = p0;
    for (; row + 3 * parts < a.d; row += 4 * parts) {
      m0 = fmaxf(m0, fabsf(Ws[row * NP + col]));
      m1 = fmaxf(m1, fabsf(Ws[(row + parts) * NP + col]));
      m2 = fmaxf(m2, fabsf(Ws[(row + 2 * parts) * NP + col]));
      m3 = fmaxf(m3, fabsf(Ws[(row + 3 * parts) * NP + col]));
    }
    for (; row < a.d; row += parts) m0 = fmaxf(m0, fabsf(Ws[row * NP + col]));
    // Scratch: the fp64 logit space (THREADS floats fit in it; the x space
    // is receiving the first block's rows).
    float* scratch = reinterpret_cast<float*>(zd);
    scratch[tid] = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
    __syncthreads();
    if (tid < NP) {
      float mx = 0.0f;
      for (int q = 0; q < parts; ++q) mx = fmaxf(mx, scratch[q * NP + tid]);
      wmax[tid] = mx;
    }
  }

  const int h = a.d / WARPS + WARPS;  // d/W FMAs, W - 1 partial additions, the bias
  const float u = 5.9604644775390625e-08f;  // 2^-24
  const float gam = (h * u) / (1.0f - h * u);
  const float gam_ru = __fmul_ru(gam, 1.01f);
  const int slice = a.d / WARPS;
  const int P = TB * a.G;  // (token, group) pairs of a block
  // fp64 fix-up path: slice/8 FMAs into each of two accumulators, their sum,
  // two shuffle adds, W adds of the warp sums, the bias.
  const int h64 = slice / 8 + WARPS + 4;
  const double u64 = 1.1102230246251565e-16;  // 2^-53
  const double gam64_ru = __dmul_ru((h64 * u64) / (1.0 - h64 * u64), 1.01);

  for (; blk < n_blk; blk += gridDim.x) {
    cp_async_wait<0>();
    __syncthreads();  // x rows in; the previous block's outputs are written

    // Partial logits over this warp's rows, in ascending row order: per 8
    // rows, one 16-byte x read per token and one W_r row quad per row.
    float acc[TPT][4];
#pragma unroll
    for (int i = 0; i < TPT; ++i)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[i][q] = 0.0f;
    {
      const int m_lo = warp * slice, m_hi = m_lo + slice;
#pragma unroll 2
      for (int m = m_lo; m < m_hi; m += 8) {
        uint4 xv[TPT];
#pragma unroll
        for (int i = 0; i < TPT; ++i) xv[i] = *reinterpret_cast<const uint4*>(xs + (tt + TG * i) * XS + m);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 wv = *reinterpret_cast<const float4*>(Ws + (m + q) * NP + 4 * et);
#pragma unroll
          for (int i = 0; i < TPT; ++i) {
            const uint32_t word = q < 2 ? xv[i].x : q < 4 ? xv[i].y : q < 6 ? xv[i].z : xv[i].w;
            const float xf = (q & 1) ? bf16_hi(word) : bf16_lo(word);
            acc[i][0] = fmaf(xf, wv.x, acc[i][0]);
            acc[i][1] = fmaf(xf, wv.y, acc[i][1]);
            acc[i][2] = fmaf(xf, wv.z, acc[i][2]);
            acc[i][3] = fmaf(xf, wv.w, acc[i][3]);
          }
        }
      }
    }
    // ||x||_1 per token (warp-strided tokens, lane-strided chunks).
    for (int t = warp; t < TB; t += WARPS) {
      float sx = 0.0f;
      for (int c = lane; c < cpr; c += 32) {
        const uint4 v = *reinterpret_cast<const uint4*>(xs + t * XS + c * 8);
        sx += fabsf(bf16_lo(v.x)) + fabsf(bf16_hi(v.x)) + fabsf(bf16_lo(v.y)) + fabsf(bf16_hi(v.y)) +
              fabsf(bf16_lo(v.z)) + fabsf(bf16_hi(v.z)) + fabsf(bf16_lo(v.w)) + fabsf(bf16_hi(v.w));
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sx += __shfl_xor_sync(0xffffffffu, sx, off);
      if (lane == 0) nxs[t] = sx;
    }
    if (tid == 0) n_uncertain = 0;
    __syncthreads();  // x is consumed: its space takes the partials
#pragma unroll
    for (int i = 0; i < TPT; ++i)
      *reinterpret_cast<float4*>(part + (warp * TB + tt + TG * i) * NP + 4 * et) =
          make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    __syncthreads();
    // Every pair (t, g): the group's logits (warp partials added in warp
    // order, then the bias), top-k, certified by the bound; certain groups go
    // straight on to their softmax.
    for (int p = tid; p < P; p += THREADS) {
      const int t = p / a.G, g = p - t * a.G;
      const int zo = t * NP + g * a.M;
      float* zg = zf + zo;
      for (int j = 0; j < a.M; ++j) {
        float z = part[zo + j];
#pragma unroll
        for (int w = 1; w < WARPS; ++w) z += part[w * TB * NP + zo + j];
        zg[j] = z + bsm[g * a.M + j];
      }
      if (blk * TB + t >= a.R) continue;
      const uint64_t sel = group_topk(zg, a.M, a.k);
      bool certain = true;
      if (a.k < a.M) {
        const float nx = nxs[t];
        float lo = INFINITY, hi = -INFINITY;
        for (int j = 0; j < a.M; ++j) {
          const int e = g * a.M + j;
          const float bd = __fmul_ru(gam_ru, __fmaf_ru(nx, wmax[e], fabsf(bsm[e])));
          if ((sel >> j) & 1ull) lo = fminf(lo, __fsub_rd(zg[j], bd));
          else hi = fmaxf(hi, __fadd_ru(zg[j], bd));
        }
        certain = lo > hi;
      }
      if (certain) {
        ps[p] = group_softmax(zg, a.M, sel, ez + zo, dn + p);
        selp[p] = sel;
      } else {
        list[atomicAdd(&n_uncertain, 1)] = p;
      }
    }
    __syncthreads();
    // The partials are consumed: fetch the next block's rows while this one
    // is finished.
    stage_x(blk + gridDim.x);
    const int nu = n_uncertain;  // the same value in every thread: the barriers below are uniform
    if (nu > 0) {
      // fp64 logits of the uncertain groups (products of a bf16 and an fp32
      // value are exact in fp64), up to FB groups per round. A round's logits
      // (group vb, column j) are items; warp w sums rows [w d/W, (w+1) d/W)
      // of every item, lanes 4i..4i+3 taking item i (8 per pass) and a
      // quarter of the slice each, so that the fp64 work is one product and
      // one add per row and item, and the lane sums are reduced in two
      // shuffle steps. x comes from global memory in 16-byte loads (the
      // block's x rows are being replaced), W_r from shared memory. Warp sums
      // are then added in warp order, so every logit is one fixed sequence of
      // roundings.
      constexpr int FB = router_fb(NP);
      double* fb = reinterpret_cast<double*>(smem_raw + L.fb);  // [FB][WARPS][NP]
      const int quarter = slice / 4;                             // a multiple of 2
      for (int v0 = 0; v0 < nu; v0 += FB) {
        const int nv = min(FB, nu - v0);
        const int items = nv * a.M;
        for (int i0 = 0; i0 < items; i0 += 8) {
          const int item = i0 + (lane >> 2);
          const int it = item < items ? item : items - 1;
          const int vb = it / a.M, j = it - vb * a.M;
          const int pv = list[v0 + vb];
          const int tv = pv / a.G;
          const int e = (pv - tv * a.G) * a.M + j;
          const int m0 = warp * slice + (lane & 3) * quarter;
          const uint16_t* xp = a.x + static_cast<size_t>(blk * TB + tv) * a.d + m0;
          const float* wp = Ws + m0 * NP + e;
          double acc0 = 0.0, acc1 = 0.0;  // even and odd rows
          if (quarter % 8 == 0) {
            // 16-byte x loads (8 rows each; m0 is a multiple of 8).
#pragma unroll 2
            for (int r0 = 0; r0 < quarter; r0 += 8) {
              const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xp + r0));
              const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                acc0 = fma(static_cast<double>(bf16_lo(xw[q])), static_cast<double>(wp[(r0 + 2 * q) * NP]), acc0);
                acc1 = fma(static_cast<double>(bf16_hi(xw[q])), static_cast<double>(wp[(r0 + 2 * q + 1) * NP]),
                           acc1);
              }
            }
          } else {
            for (int r = 0; r < quarter; r += 2) {
              acc0 = fma(static_cast<double>(bf16_to_f32(__ldg(xp + r))), static_cast<double>(wp[r * NP]), acc0);
              acc1 = fma(static_cast<double>(bf16_to_f32(__ldg(xp + r + 1))), static_cast<double>(wp[(r + 1) * NP]),
                         acc1);
            }
          }
          double acc = acc0 + acc1;
          acc += __shfl_xor_sync(0xffffffffu, acc, 1);
          acc += __shfl_xor_sync(0xffffffffu, acc, 2);
          if ((lane & 3) == 0 && item < items) fb[(vb * WARPS + warp) * NP + e] = acc;
        }
        __syncthreads();
        for (int u = tid; u < items; u += THREADS) {
          const int vb = u / a.M, j = u - vb * a.M;
          const int pv = list[v0 + vb];
          const int tv = pv / a.G, gv = pv - tv * a.G;
          const int e = gv * a.M + j;
          double z = 0.0;
          for (int w = 0; w < WARPS; ++w) z += fb[(vb * WARPS + w) * NP + e];
          zd[tv * NP + e] = z + static_cast<double>(bsm[e]);
        }
        __syncthreads();
      }
      // fp64 decisions, certified by the fp64 bound (directed rounding; the
      // 1 % in gam64_ru covers the fp32 rounding of ||x||_1). A pair that
      // stays uncertain is marked with an empty selection.
      for (int v = tid; v < nu; v += THREADS) {
        const int pv = list[v];
        const int tv = pv / a.G, gv = pv - tv * a.G;
        const int zo = tv * NP + gv * a.M;
        const uint64_t sel = group_topk(zd + zo, a.M, a.k);
        bool certain = true;
        if (a.k < a.M) {
          const double nx = static_cast<double>(nxs[tv]);
          double lo = INFINITY, hi = -INFINITY;
          for (int j = 0; j < a.M; ++j) {
            const int e = gv * a.M + j;
            const double bd =
                __dmul_ru(gam64_ru, __fma_ru(nx, static_cast<double>(wmax[e]), fabs(static_cast<double>(bsm[e]))));
            if ((sel >> j) & 1ull) lo = fmin(lo, __dsub_rd(zd[zo + j], bd));
            else hi = fmax(hi, __dadd_ru(zd[zo + j], bd));
          }
          certain = lo > hi;
        }
        if (certain) ps[pv] = group_softmax(zd + zo, a.M, sel, ez + zo, dn + pv);
        selp[pv] = certain ? sel : 0ull;
      }
      __syncthreads();
      // Pairs left undecided, compacted in place (one thread).
      if (tid == 0) {
        int ne = 0;
        for (int v = 0; v < nu; ++v)
          if (selp[list[v]] == 0ull) list[ne++] = list[v];
        n_exact = ne;
      }
      __syncthreads();
      const int ne = n_exact;  // uniform: the call below holds barriers
      if (ne > 0)
        exact_decide(a.x, a.d, a.G, a.M, a.k, Ws, NP, bsm, reinterpret_cast<long long*>(smem_raw + L.fb),
                     list, ne, blk * TB, zd, ez, dn, ps, selp, &exact_sel, &exact_best);
    }
    // idx, r (renormalised in the group) and omega (over the token's groups).
    for (int p = tid; p < P; p += THREADS) {
      const int t = p / a.G, g = p - t * a.G;
      if (blk * TB + t >= a.R) continue;
      const int zo = t * NP + g * a.M;
      float tot = 0.0f;  // selected mass of the token over its groups
      for (int g2 = 0; g2 < a.G; ++g2) tot += ps[t * a.G + g2];
      const float psel = ps[p], den = dn[p];
      const uint64_t sel = selp[p];
      const size_t o = (static_cast<size_t>(blk * TB + t) * a.G + g) * a.k;
      int s = 0;
      for (int j = 0; j < a.M; ++j) {
        if ((sel >> j) & 1ull) {
          const float pj = ez[zo + j] / den;
          a.idx[o + s] = j;
          a.r[o + s] = pj / psel;
          a.omega[o + s] = a.wmode == 0 ? pj / tot : a.wmode == 1 ? (pj / psel) / a.G : pj;
          ++s;
        }
      }
    }
  }
  cp_async_wait<0>();
}

// SMs of the current device and resident CTAs per SM of one router kernel.
inline int device_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <int NP, int WARPS, int TPT>
int launch_tpt(const gqe_config& c, const RouterArgs& a, cudaStream_t st) {
  const size_t smem = router_layout(c.d_model, NP, TPT).total;
  if (smem > kRouterSmemLimit) return cudaErrorInvalidConfiguration;
  const int e = ensure_smem<router_kernel<NP, WARPS, TPT>>(static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // Resident CTAs per SM, looked up once per device (devices may differ).
  static std::atomic<int> per_sm[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = -1;
  int ps = dev >= 0 ? per_sm[dev].load(std::memory_order_relaxed) : 0;
  if (ps <= 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ps, router_kernel<NP, WARPS, TPT>, WARPS * 32,
                                                      smem) != cudaSuccess || ps < 1)
      ps = 1;
    if (dev >= 0) per_sm[dev].store(ps, std::memory_order_relaxed);
  }
  // One token block per CTA while that fills the GPU; larger batches loop.
  const int n_blk = (a.R + router_tb(NP, TPT) - 1) / router_tb(NP, TPT);
  const int slots = ps * device_sms();
  const int grid = n_blk < slots ? n_blk : slots;
  return launch_pdl(router_kernel<NP, WARPS, TPT>, dim3(grid > 0 ? grid : 1), dim3(WARPS * 32), smem, st, a);
}

// Rows from which a launch takes more tokens per thread: each W_r quad read
// from shared memory then feeds 6 (or 4, where shared memory is short)
// tokens instead of 2, at the price of fewer, larger token blocks (which
// small batches cannot spread over the SMs).
constexpr int kRouterWideRows = 4096;

template <int NP, int WARPS>
int launch_np(const gqe_config& c, const RouterArgs& a, cudaStream_t st) {
  if (a.R >= kRouterWideRows) {
    if (router_layout(c.d_model, NP, 6).total <= kRouterSmemLimit) return launch_tpt<NP, WARPS, 6>(c, a, st);
    if (router_layout(c.d_model, NP, 4).total <= kRouterSmemLimit) return launch_tpt<NP, WARPS, 4>(c, a, st);
  }
  return launch_tpt<NP, WARPS, 2>(c, a, st);
}

template <int NP>
int launch_w(const gqe_config& c, const RouterArgs& a, cudaStream_t st) {
  return router_warps(c.d_model) == 16 ? launch_np<NP, 16>(c, a, st) : launch_np<NP, 8>(c, a, st);
}

}  // namespace router_impl
using namespace router_impl;

// The narrowest block shape (2 tokens per thread) is the one every batch can
// take.
size_t router_smem_bytes(const gqe_config& c) {
  return router_layout(c.d_model, router_np(c.G * c.M), 2).total;
}

int launch_router(const gqe_config& c, const uint16_t* x, const float* W_r, const float* b_r,
                  int32_t* idx, float* r, float* omega, void* stream) {
  RouterArgs a{x, W_r, b_r, idx, r, omega, c.B * c.T, c.d_model, c.G, c.M, c.k, c.G * c.M, omega_mode(c)};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (router_np(a.N)) {
    case 4: return launch_w<4>(c, a, st);
    case 8: return launch_w<8>(c, a, st);
    case 16: return launch_w<16>(c, a, st);
    case 32: return launch_w<32>(c, a, st);
    default: return launch_w<64>(c, a, st);
  }
}

}  // namespace gqe
