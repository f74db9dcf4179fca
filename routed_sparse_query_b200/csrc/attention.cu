// Causal flash attention on tcgen05 for the routed and shared heads of the
// GQE layer (steps a8, a9) and for the dense GQA comparison layer.
//
// Every routed slot stream (b, g, s) is a dense, position-ordered stream of T
// query rows (each token selects exactly k experts of every group), so it is
// plain causal attention of T queries against the group's K/V; the shared
// head is one more stream against group 0. Only the selected experts' queries
// exist, so the work is (kG+1)/N of the dense layer ("GQE keeps the KV cache
// benefits of GQA and reduces only the active query-head computation":
// chatpaper / hotpaper abstract; 9 of 16 heads active: gist.science Technical
// Summary, Experimental Results).
//
// One CTA = two consecutive 128-row query tiles (a, b) of one stream, or a
// KV chunk of them (split-KV for short sequences); KV tiles of 128 keys up to
// the diagonal (fully masked tiles are never loaded). Warp roles (320
// threads):
//   warps 0-7  softmax, warpgroup t for tile t: thread i owns query row i
//              (TMEM lane i); online softmax in fp32 (exp2 with the
//              1/sqrt(dh)*log2(e) scale folded in); P is written back over S
//              in tensor memory as bf16 pairs; O is rescaled in TMEM only when
//              the row max grows by more than 2^8; final O / l stored;
//   warp 8     TMA loads of Q and of K/V tiles (4-stage ring);
//   warp 9     issues S = Q K^T into three rotating TMEM S buffers and
//              O += P V with P read from tensor memory.
// TMEM columns: S buffers [0,128), [128,256), [256,384); O_a, O_b at 384.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cmath>

#include "gqe_internal.h"
#include "ptx.cuh"
#include "tmap.h"

namespace gqe {

namespace attn_impl {

constexpr int BQ = 128;
constexpr int BKV = 128;
constexpr int KV_STAGES = 4;
constexpr int kThreads = 320;  // 2 softmax warpgroups + TMA warp + UMMA warp
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
// O is rescaled only when a row's running max grows by more than this many
// powers of two; until then the stale max is kept and P may reach 2^8.
constexpr float kRescaleLog2 = 8.0f;

template <int DH>
struct AttnCfg {
  static constexpr int SWB = DH * 2;  // bytes per Q/K/V row = swizzle width
  static constexpr uint32_t LAYOUT = SWB == 128 ? kLayoutSW128 : kLayoutSW64;
  static constexpr int TILE_BYTES = BQ * DH * 2;
  static constexpr size_t SMEM = 1024 + static_cast<size_t>(TILE_BYTES) * (2 + 2 * KV_STAGES) + 512;
  static constexpr uint32_t TMEM_COLS = 512;  // 3 rotating S buffers (128 each), O_a, O_b (DH each)
};

struct AttnParams {
  int T, B, H;       // tokens per sequence, sequences, query streams per sequence
  int G, k, M;       // groups, selected per group, experts per group
  int dense;         // 0: GQE streams (kG routed + shared), 1: dense GQA heads
  int n_qt;          // 128-row query tiles per stream
  int n_pairs;       // pairs of consecutive query tiles per stream
  int chunk;         // KV tiles per CTA (split-KV); >= n_qt: no split
  int items;         // CTAs per stream
  uint16_t* out;     // [B*T, ldo]
  int ldo;
  float scale_log2;  // log2(e) / sqrt(dh)
  float* part;       // split-KV partial O: [B*H][items][2][128][dh] fp32
  float2* part_ml;   // split-KV partial (m, l): [B*H][items][2][128]
  int* counters;     // split-KV arrivals per (stream, pair), zero between calls
  // Expert-major routed tiles (em = 1): a query tile is 128 consecutive
  // entries of one (expert, sequence) token list, the Q rows in list order
  // (row r of the layer's routed queries = list entry r); each row is masked
  // by its own original position tok[r]. The first em_units CTAs take pairs
  // of such tiles (an upper bound: CTAs past the last pair exit); the rest
  // take the shared head's stream, as in the slot-major layout.
  int em;
  int em_units;
  int N;
  const int32_t* offsets;  // [N*B + 1]: list starts in (expert, sequence) order
  const int32_t* tok;      // list entries: positions t
  const int32_t* idx;      // [B*T, G, k]: selections (the output slot of a row)
  // Optional (slot-major streams only): each row's log-sum-exp in base 2 of
  // s log2(e)/sqrt(dh), lse[stream][lse_ld] (the backward's softmax statistics).
  float* lse;
  int lse_ld;
};

// Expert-major decode: routed unit u -> (list l = e*B + b, pair q of its
// tiles). Units are counted list by list; inside a list the pair with the
// largest positions (the longest KV range) comes first. Warp-cooperative;
// every lane returns the same values. False past the last unit.
__device__ __forceinline__ bool em_find_unit(const AttnParams& p, int u, int lane, int& l_out,
                                             int& list0, int& cnt, int& q) {
  const int NB = p.N * p.B;
  int base = 0;
  for (int l0 = 0; l0 < NB; l0 += 32) {
    const int l = l0 + lane;
    int c = 0;
    if (l < NB) c = p.offsets[l + 1] - p.offsets[l];
    const int pairs = (c + 2 * BQ - 1) / (2 * BQ);
    int incl = pairs;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (u < base + total) {
      const unsigned m = __ballot_sync(0xffffffffu, u < base + incl);
      const int src = __ffs(m) - 1;
      const int src_pairs = __shfl_sync(0xffffffffu, pairs, src);
      const int src_excl = __shfl_sync(0xffffffffu, incl, src) - src_pairs;
      cnt = __shfl_sync(0xffffffffu, c, src);
      l_out = l0 + src;
      q = src_pairs - 1 - (u - base - src_excl);
      list0 = __ldg(p.offsets + l_out) + 2 * BQ * q;
      return true;
    }
    base += total;
  }
  return false;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Packed fp32 pairs (sm_100 f32x2 instructions: one issue slot for two lanes
// of arithmetic).
__device__ __forceinline__ uint64_t as_u64(float2 v) { return *reinterpret_cast<uint64_t*>(&v); }
__device__ __forceinline__ float2 as_f2(uint64_t v) { return *reinterpret_cast<float2*>(&v); }
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(as_u64(a)), "l"(as_u64(b)), "l"(as_u64(c)));
  return as_f2(r);
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(as_u64(a)), "l"(as_u64(b)));
  return as_f2(r);
}
__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(as_u64(a)), "l"(as_u64(b)));
  return as_f2(r);
}

// 2^x on the FMA pipe for a pair of values: x = n + f with n = round(x)
// (the 1.5*2^23 shift rounds to nearest), 2^f by a degree-3 minimax
// polynomial on [-1/2, 1/2] (relative error 7.5e-5; coefficients from
// exp2_poly_fit.py), 2^n added into the exponent field. Inputs below -125 are
// clamped (result ~1e-38). Additions and the polynomial use f32x2.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 shift = make_float2(12582912.0f, 12582912.0f);
  const float2 t = fadd2(x, shift);
  const float2 f = fsub2(x, fsub2(t, shift));
  float2 q = ffma2(make_float2(5.517166853e-02f, 5.517166853e-02f), f,
                   make_float2(2.426111251e-01f, 2.426111251e-01f));
  q = ffma2(q, f, make_float2(6.932609677e-01f, 6.932609677e-01f));
  q = ffma2(q, f, make_float2(9.999280572e-01f, 9.999280572e-01f));
  return make_float2(__int_as_float(__float_as_int(q.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(q.y) + (__float_as_int(t.y) << 23)));
}

// Online softmax of one query row against one 128-key tile held in TMEM
// (tS): pass 1 takes the row max, pass 2 computes P = 2^(s*scale - m), adds
// it to l and writes it as bf16 pairs over the first 64 columns of the same
// S buffer (the A operand of the PV product; each 32-column chunk of S is
// read before the P columns over it are written). Only the diagonal tile
// (MASK) tests keys against the row's position: key x is visible iff
// x <= lim. O (tO) is rescaled only when the max grows by more than
// kRescaleLog2; the rescale first waits for the previous PV (pv_prev).
template <int DH, bool MASK>
__device__ __forceinline__ bool softmax_tile(uint32_t tS, uint32_t tO, int lim, float sc,
                                             bool first, float& m, float& l, uint64_t* pv_prev,
                                             uint32_t pv_parity, volatile int* abort_flag) {
  // TMEM loads are software-pipelined: chunk c+1 (32 columns) is in flight
  // while chunk c is processed.
  float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  auto row_max = [&](const uint32_t (&v)[32], int c) {
#pragma unroll
    for (int x = 0; x < 32; x += 8) {
      float a[8];
#pragma unroll
      for (int y = 0; y < 8; ++y) {
        a[y] = __uint_as_float(v[x + y]);
        if (MASK && c * 32 + x + y > lim) a[y] = -INFINITY;
      }
      mx[0] = max3(mx[0], a[0], a[4]);
      mx[1] = max3(mx[1], a[1], a[5]);
      mx[2] = max3(mx[2], a[2], a[6]);
      mx[3] = max3(mx[3], a[3], a[7]);
    }
  };
  uint32_t va[32], vb[32];
  tmem_ld32_nowait(tS + 0, va);
  tmem_ld_wait(va);
  tmem_ld32_nowait(tS + 32, vb);
  row_max(va, 0);
  tmem_ld_wait(vb);
  tmem_ld32_nowait(tS + 64, va);
  row_max(vb, 1);
  tmem_ld_wait(va);
  tmem_ld32_nowait(tS + 96, vb);
  row_max(va, 2);
  tmem_ld_wait(vb);
  tmem_ld32_nowait(tS + 0, va);  // first chunk of pass 2
  row_max(vb, 3);

  const float mc = fmaxf(max3(mx[0], mx[1], mx[2]), mx[3]) * sc;
  const bool need = mc > m + kRescaleLog2;
  if (__any_sync(0xffffffffu, need)) {
    if (pv_prev != nullptr) {  // O holds earlier tiles: their PV must be complete
      if (!__all_sync(0xffffffffu, mbar_wait(pv_prev, pv_parity, abort_flag))) {
        tmem_ld_wait(va);
        return false;
      }
      tc_fence_after();
    }
    const float m_new = need ? mc : m;
    const float alpha = ex2(m - m_new);
    if (!first) {
#pragma unroll
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tO + c * 32, v);
#pragma unroll
        for (int x = 0; x < 32; ++x) v[x] = __float_as_uint(__uint_as_float(v[x]) * alpha);
        tmem_st32(tO + c * 32, v);
      }
      tmem_st_wait();
    }
    l *= alpha;
    m = m_new;
  }
  const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(-m, -m);
  float2 lsum[4] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f),
                    make_float2(0.0f, 0.0f)};  // independent partial sums (no serial chain)
  auto exp_chunk = [&](const uint32_t (&v)[32], int c) {
    uint32_t pw[16];
#pragma unroll
    for (int c8 = 0; c8 < 4; ++c8) {
      const int c16 = c * 4 + c8;  // 8-key chunk index in the row
      float e8[8];
#pragma unroll
      for (int x = 0; x < 8; x += 2) {
        float2 z = ffma2(make_float2(__uint_as_float(v[c8 * 8 + x]), __uint_as_float(v[c8 * 8 + x + 1])),
                         sc2, nm2);
        if (MASK) {
          if (c16 * 8 + x > lim) z.x = -INFINITY;
          if (c16 * 8 + x + 1 > lim) z.y = -INFINITY;
        }
        float2 e;
        if ((c8 & 1) && x >= 4) {  // 4 of every 16 on the FMA pipe, the rest on MUFU
          e = exp2_poly2(z);
          if (MASK) {
            if (c16 * 8 + x > lim) e.x = 0.0f;
            if (c16 * 8 + x + 1 > lim) e.y = 0.0f;
          }
        } else {
          e = make_float2(ex2(z.x), ex2(z.y));
        }
        e8[x] = e.x;
        e8[x + 1] = e.y;
        lsum[x >> 1] = fadd2(lsum[x >> 1], e);
      }
      pw[4 * c8 + 0] = pack_bf16x2(e8[0], e8[1]);
      pw[4 * c8 + 1] = pack_bf16x2(e8[2], e8[3]);
      pw[4 * c8 + 2] = pack_bf16x2(e8[4], e8[5]);
      pw[4 * c8 + 3] = pack_bf16x2(e8[6], e8[7]);
    }
    tmem_st16(tS + c * 16, pw);  // keys 32c..32c+31 -> columns 16c..16c+15
  };
  tmem_ld_wait(va);
  tmem_ld32_nowait(tS + 32, vb);
  exp_chunk(va, 0);
  tmem_ld_wait(vb);
  tmem_ld32_nowait(tS + 64, va);
  exp_chunk(vb, 1);
  tmem_ld_wait(va);
  tmem_ld32_nowait(tS + 96, vb);
  exp_chunk(va, 2);
  tmem_ld_wait(vb);
  exp_chunk(vb, 3);
  tmem_st_wait();
  const float2 l01 = fadd2(lsum[0], lsum[1]), l23 = fadd2(lsum[2], lsum[3]);
  const float2 l4 = fadd2(l01, l23);
  l += l4.x + l4.y;
  return true;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Stores 32 fp32 values times `scale` as bf16 (64 contiguous bytes).
__device__ __forceinline__ void store_row32(uint16_t* dst, const uint32_t (&v)[32], float scale) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    uint4 o;
    o.x = pack_bf16x2(__uint_as_float(v[8 * q4 + 0]) * scale, __uint_as_float(v[8 * q4 + 1]) * scale);
    o.y = pack_bf16x2(__uint_as_float(v[8 * q4 + 2]) * scale, __uint_as_float(v[8 * q4 + 3]) * scale);
    o.z = pack_bf16x2(__uint_as_float(v[8 * q4 + 4]) * scale, __uint_as_float(v[8 * q4 + 5]) * scale);
    o.w = pack_bf16x2(__uint_as_float(v[8 * q4 + 6]) * scale, __uint_as_float(v[8 * q4 + 7]) * scale);
    d4[q4] = o;
  }
}

// Item n of a CTA's S sequence over its KV tiles j0..: (a,j0), (b,j0),
// (a,j0+1), (b,j0+1), ..., then tile b's further tiles (one diagonal tile in
// the slot-major layout, possibly more with expert-major tiles); tile a
// alone when the CTA has no tile b. na = tile a's KV tiles in the CTA.
__device__ __forceinline__ void seq_item(int n, bool has_b, int j0, int na, int& t, int& j) {
  if (!has_b) {
    t = 0;
    j = j0 + n;
  } else if (n < 2 * na) {
    t = n & 1;
    j = j0 + (n >> 1);
  } else {
    t = 1;
    j = j0 + na + (n - 2 * na);
  }
}

template <int DH>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQs,
                const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                const AttnParams p) {
  using C = AttnCfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sp = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = sp;                                // [2][TILE]
  uint8_t* sK = sQ + 2 * C::TILE_BYTES;            // [KV_STAGES][TILE]
  uint8_t* sV = sK + KV_STAGES * C::TILE_BYTES;    // [KV_STAGES][TILE]
  uint64_t* bar = reinterpret_cast<uint64_t*>(sV + KV_STAGES * C::TILE_BYTES);
  uint64_t* q_full = bar;
  uint64_t* k_full = bar + 1;
  uint64_t* v_full = k_full + KV_STAGES;
  uint64_t* kv_empty = v_full + KV_STAGES;
  uint64_t* s_full = kv_empty + KV_STAGES;  // [3] one per S buffer
  uint64_t* p_full = s_full + 3;            // [2] one per query tile
  uint64_t* o_done = p_full + 2;            // [2] one per query tile
  uint64_t* drain = o_done + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  volatile int* s_last = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = p.B * p.H;
  // Work of this CTA. Slot-major (and the shared head of an expert-major
  // launch): (stream, query-tile pair, KV chunk), longest pairs first, decoded
  // from the launch parameters. Expert-major routed tiles: decoded after
  // pdl_wait from the token lists (below).
  const bool em_routed = p.em != 0 && static_cast<int>(blockIdx.x) < p.em_units;
  int bh = 0, b = 0, zq = 0, grp = 0, slot = 0, pair = 0, chunk_id = 0, n_chunks = 1, item_base = 0;
  int qa = 0, qb = 0;    // Q rows (TMA coordinate) of tiles a and b
  int mfa = 0, mfb = 0;  // first KV tile that needs the causal mask, per tile
  int j0 = 0, ja1 = 0, jb1 = 0;
  bool has_b = false;
  int em_e = 0, em_list0 = 0, em_rows_a = 0, em_rows_b = 0;
  const CUtensorMap* tq = &tmQ;
  if (!em_routed) {
    int ord, h;
    if (p.em) {  // the shared head of an expert-major launch: B streams
      const int u2 = static_cast<int>(blockIdx.x) - p.em_units;
      b = u2 % p.B;
      ord = u2 / p.B;
      h = p.G * p.k;
      bh = b * p.H + h;
    } else {
      if (p.chunk >= p.n_qt && p.n_pairs >= 1024) {
        // Long sequences: stream-major, so that the CTAs in flight share one
        // group's K/V in L2 (longest pairs first inside each stream).
        bh = static_cast<int>(blockIdx.x) / p.items;
        ord = static_cast<int>(blockIdx.x) % p.items;
      } else {
        // Longest pairs of every stream first (balanced tail).
        bh = static_cast<int>(blockIdx.x) % BH;
        ord = static_cast<int>(blockIdx.x) / BH;
      }
      b = bh / p.H;
      h = bh % p.H;
    }
    item_base = ord;
    if (p.chunk >= p.n_qt) {
      pair = p.n_pairs - 1 - ord;
    } else {
      item_base = 0;
      for (pair = p.n_pairs - 1; pair > 0; --pair) {
        const int nc = (2 * pair + 1 + p.chunk - 1) / p.chunk;
        if (ord < nc) break;
        ord -= nc;
        item_base += nc;
      }
      n_chunks = (2 * pair + 1 + p.chunk - 1) / p.chunk;
      chunk_id = ord;
    }
    if (p.dense) {
      zq = b * p.H + h;
      grp = h / p.M;
      slot = h;
    } else if (h < p.G * p.k) {
      zq = b * p.G * p.k + h;
      grp = h / p.k;
      slot = h;
    } else {
      zq = b;
      grp = 0;
      slot = p.G * p.k;
      tq = &tmQs;
    }
    const int qt0 = 2 * pair;
    has_b = qt0 + 1 < p.n_qt;
    // Causal: query tile qt needs KV tiles 0..qt (tile a = qt0, tile b =
    // qt0+1). This CTA takes KV tiles [j0, ja1) for tile a and [j0, jb1) for
    // tile b; the last chunk also holds tile b's extra diagonal tile.
    j0 = chunk_id * (p.chunk < p.n_qt ? p.chunk : 0);
    const bool last_chunk = chunk_id == n_chunks - 1;
    ja1 = last_chunk ? qt0 + 1 : j0 + p.chunk;
    jb1 = has_b ? (last_chunk ? qt0 + 2 : ja1) : j0;
    qa = qt0 * BQ;
    qb = qa + BQ;
    mfa = qt0;  // only the diagonal tile is masked
    mfb = qt0 + 1;
  }
  int na = ja1 - j0;
  int jend = has_b ? jb1 : ja1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < KV_STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b3 = 0; b3 < 3; ++b3) mbar_init(&s_full[b3], 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&p_full[t], 128);
      mbar_init(&o_done[t], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kTmaWarp && lane == 0) {
    prefetch_tmap(tq);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == kMmaWarp) tmem_alloc(tslot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  pdl_wait();  // every input (Q, K, V) is read after this point
  pdl_launch_dependents();
  if (em_routed) {
    // Expert-major routed pair: tiles of 128 consecutive list entries; the KV
    // range of a tile ends at the tile containing its last (largest)
    // position, and the mask starts at the first tile not entirely below its
    // first (smallest) position. A CTA past the last pair loads one Q tile
    // and exits.
    int l = 0, cnt = 0, q = 0, list0 = 0;
    if (em_find_unit(p, static_cast<int>(blockIdx.x), lane, l, list0, cnt, q)) {
      em_e = l / p.B;
      b = l % p.B;
      grp = em_e / p.M;
      em_list0 = list0;
      const int rem = cnt - 2 * BQ * q;
      em_rows_a = rem < BQ ? rem : BQ;
      em_rows_b = rem - BQ < BQ ? rem - BQ : BQ;
      has_b = em_rows_b > 0;
      const int pa0 = __ldg(p.tok + list0), pa1 = __ldg(p.tok + list0 + em_rows_a - 1);
      qa = list0;
      qb = list0 + BQ;
      mfa = (pa0 + 1) / BKV;
      ja1 = pa1 / BKV + 1;
      if (has_b) {
        const int pb0 = __ldg(p.tok + list0 + BQ), pb1 = __ldg(p.tok + list0 + BQ + em_rows_b - 1);
        mfb = (pb0 + 1) / BKV;
        jb1 = pb1 / BKV + 1;
      } else {
        jb1 = 0;
      }
    }
    na = ja1 - j0;
    jend = has_b ? jb1 : ja1;
  }
  const int zkv = b * p.G + grp;

  if (warp == kTmaWarp) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, C::TILE_BYTES * (has_b ? 2 : 1));
      tma_load_3d(sQ, tq, q_full, 0, qa, zq);
      if (has_b) tma_load_3d(sQ + C::TILE_BYTES, tq, q_full, 0, qb, zq);
      for (int j = j0; j < jend; ++j) {
        const int st = (j - j0) % KV_STAGES;
        const uint32_t ph = ((j - j0) / KV_STAGES) & 1;
        if (!mbar_wait(&kv_empty[st], ph ^ 1u, abort_flag)) break;
        mbar_arrive_expect_tx(&k_full[st], C::TILE_BYTES);
        tma_load_3d(sK + st * C::TILE_BYTES, &tmK, &k_full[st], 0, j * BKV, zkv);
        mbar_arrive_expect_tx(&v_full[st], C::TILE_BYTES);
        tma_load_3d(sV + st * C::TILE_BYTES, &tmV, &v_full[st], 0, j * BKV, zkv);
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- UMMA issuer
    // S tiles are computed in sequence n = 0, 1, 2, ... ((a,0), (b,0),
    // (a,1), (b,1), ...) into TMEM buffer n % 3. Once the softmax of item m
    // has published P (so it has finished reading S(m)), the issuer computes
    // PV of item m and then S(m+3) into that buffer, so every tile's next S
    // is ready while its current softmax runs. The whole warp runs this
    // loop; elect.sync picks the lane that issues.
    {
      constexpr uint32_t idS = idesc_bf16_f32(BQ, BKV, 0, 0);
      constexpr uint32_t idO = idesc_bf16_f32(BQ, DH, 0, 1);
      // Descriptors are built once; an operand at a byte offset from its base
      // is the base descriptor plus (offset >> 4) in the start-address field
      // (shared-memory addresses stay below 2^18, so the field never carries).
      const uint64_t dQ = smem_desc(smem_u32(sQ), 16, 8 * C::SWB, C::LAYOUT);
      const uint64_t dK = smem_desc(smem_u32(sK), 16, 8 * C::SWB, C::LAYOUT);
      const uint64_t dV = smem_desc(smem_u32(sV), C::TILE_BYTES, 8 * C::SWB, C::LAYOUT);
      auto wait_all = [&](uint64_t* b, uint32_t par) {
        return __all_sync(0xffffffffu, mbar_wait(b, par, abort_flag));
      };
      auto issue_S = [&](int n) -> bool {
        int t, j;
        seq_item(n, has_b, j0, na, t, j);
        const int st = (j - j0) % KV_STAGES;
        if (!wait_all(&k_full[st], ((j - j0) / KV_STAGES) & 1)) return false;
        tc_fence_after();
        const uint64_t q0 = dQ + static_cast<uint64_t>((t * C::TILE_BYTES) >> 4);
        const uint64_t k0 = dK + static_cast<uint64_t>((st * C::TILE_BYTES) >> 4);
        const uint32_t d = tmem + (n % 3) * 128;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk)
          umma_bf16_ss_elect(d, q0 + 2 * kk, k0 + 2 * kk, idS, kk > 0 ? 1u : 0u);
        umma_commit_elect(&s_full[n % 3]);
        return true;
      };
      const int n_total = has_b ? 2 * na + (jb1 - ja1) : na;
      bool ok = wait_all(q_full, 0);
      for (int n = 0; ok && n < 3 && n < n_total; ++n) ok = issue_S(n);
      for (int m = 0; ok && m < n_total; ++m) {
        int t, j;
        seq_item(m, has_b, j0, na, t, j);
        const int jr = j - j0;
        const int st = jr % KV_STAGES;
        if (!wait_all(&p_full[t], jr & 1) || !wait_all(&v_full[st], (jr / KV_STAGES) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // P(m) sits over the first 64 columns of S buffer m % 3.
        const uint32_t aP = tmem + (m % 3) * 128;
        const uint64_t v0 = dV + static_cast<uint64_t>((st * C::TILE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk)
          umma_bf16_ts_elect(tmem + 384 + t * DH, aP + kk * 8, v0 + (kk * 16 * C::SWB) / 16, idO,
                             (jr > 0 || kk > 0) ? 1u : 0u);
        umma_commit_elect(&o_done[t]);
        if (t == 1 || !has_b) umma_commit_elect(&kv_empty[st]);  // last reader of K_j, V_j
        // S(m+3) follows PV(m): with one tile it needs K_{j+3}, which shares a
        // stage with V_j (measured: issuing S first is not faster with two).
        if (m + 3 < n_total) ok = issue_S(m + 3);
      }
      umma_commit_elect(drain);
    }
  } else {
    // ---------------------------------------------------------- softmax
    const int t = warp >> 2;            // 0: tile a, 1: tile b
    const int i = threadIdx.x & 127;    // row in tile = TMEM lane
    const int jt1 = t == 0 ? ja1 : jb1;  // this tile's KV tiles: [j0, jt1)
    const int n_t = (t == 0 || has_b) ? jt1 - j0 : 0;
    const int mask_from = t == 0 ? mfa : mfb;
    // The row's original position (qi) and whether it holds a query.
    int qi;
    bool row_ok;
    if (em_routed) {
      const int rows = t == 0 ? em_rows_a : em_rows_b;
      row_ok = i < rows;
      qi = rows > 0 ? __ldg(p.tok + em_list0 + t * BQ + (row_ok ? i : rows - 1)) : 0;
    } else {
      qi = (qa / BQ + t) * BQ + i;
      row_ok = qi < p.T;
    }
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tO = tmem + 384 + t * DH + lane_off;
    const float sc = p.scale_log2;
    float m = -INFINITY, l = 0.0f;
    bool ok = n_t > 0;
    for (int jr = 0; ok && jr < n_t; ++jr) {
      const int j = j0 + jr;
      // This tile's S for KV tile j is sequence item n, in TMEM buffer n % 3.
      const int n = has_b ? (j < ja1 ? 2 * jr + t : 2 * na + (j - ja1)) : jr;
      const uint32_t tS = tmem + (n % 3) * 128 + lane_off;
      // Waits are made warp-uniform: tcgen05.ld/st below are .sync.aligned.
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[n % 3], (n / 3) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // PV(jr - 1) must be complete before O is rescaled (softmax_tile waits
      // for it only then) and before P(jr) is published: the issuer waits for
      // the phases of p_full[t] one at a time, so this tile may run at most
      // one phase ahead of it. The exp pass overlaps PV(jr - 1).
      uint64_t* pv_prev = jr > 0 ? &o_done[t] : nullptr;
      const uint32_t pv_par = static_cast<uint32_t>(jr - 1) & 1u;
      bool w_ok = true;
      if (j >= mask_from)  // a tile with keys after some row's position
        w_ok = softmax_tile<DH, true>(tS, tO, qi - j * BKV, sc, jr == 0, m, l, pv_prev, pv_par,
                                      abort_flag);
      else
        w_ok = softmax_tile<DH, false>(tS, tO, BKV, sc, jr == 0, m, l, pv_prev, pv_par, abort_flag);
      if (w_ok && jr >= 1) w_ok = __all_sync(0xffffffffu, mbar_wait(pv_prev, pv_par, abort_flag));
      if (!w_ok) {
        ok = false;
        break;
      }
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }
    const bool fin =
        ok && n_t > 0 && __all_sync(0xffffffffu, mbar_wait(&o_done[t], (n_t - 1) & 1, abort_flag));
    if (n_chunks == 1) {
      if (fin) {
        tc_fence_after();
        const float inv = 1.0f / l;
        int col = slot;
        if (em_routed && row_ok) {
          // The row's slot: rank of its expert among its selections in the group.
          const int g = em_e / p.M, jj = em_e % p.M;
          const int32_t* ip = p.idx + (static_cast<size_t>(b) * p.T + qi) * p.G * p.k + g * p.k;
          int s2 = 0;
          for (int s3 = 0; s3 < p.k; ++s3)
            if (__ldg(ip + s3) == jj) s2 = s3;
          col = g * p.k + s2;
        }
        uint16_t* dst = p.out + (static_cast<size_t>(b) * p.T + qi) * p.ldo + col * DH;
#pragma unroll
        for (int c = 0; c < DH / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tO + c * 32, v);
          if (row_ok) store_row32(dst + c * 32, v, inv);
        }
        if (p.lse != nullptr && row_ok) p.lse[static_cast<size_t>(bh) * p.lse_ld + qi] = m + log2f(l);
      }
    } else {
      // Split-KV: publish this chunk's unnormalised rows (O relative to the
      // row's m, and l); the last CTA of the pair to arrive merges all chunks:
      // O = sum_c 2^(m_c - m*) O_c, l = sum_c 2^(m_c - m*) l_c, out = O / l.
      // Partial rows are stored column-major by 16-byte word ([chunk][tile]
      // [dh/4][128 rows] float4): the 32 lanes of a warp (32 consecutive rows)
      // touch 32 consecutive words.
      const size_t blk = (static_cast<size_t>(bh) * p.items + item_base + chunk_id) * 2 + t;
      if (fin) {
        tc_fence_after();
        float4* dst = reinterpret_cast<float4*>(p.part) + blk * (BQ * DH / 4) + i;
#pragma unroll
        for (int c = 0; c < DH / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tO + c * 32, v);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[(c * 8 + q) * BQ] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                                __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
        }
        p.part_ml[blk * BQ + i] = make_float2(m, l);
      }
      named_bar_sync(1, 256);
      if (threadIdx.x == 0) {
        __threadfence();
        const int old = atomicAdd(&p.counters[bh * p.n_pairs + pair], 1);
        *s_last = old == n_chunks - 1;
      }
      named_bar_sync(1, 256);
      if (*s_last) {
        __threadfence();
        if (n_t > 0 && row_ok) {
          const size_t blk0 = (static_cast<size_t>(bh) * p.items + item_base) * 2 + t;
          float ms = -INFINITY;
          for (int c = 0; c < n_chunks; ++c) ms = fmaxf(ms, __ldcg(&p.part_ml[(blk0 + 2 * c) * BQ + i]).x);
          float acc[DH];
#pragma unroll
          for (int x = 0; x < DH; ++x) acc[x] = 0.0f;
          float lt = 0.0f;
#pragma unroll 2
          for (int c = 0; c < n_chunks; ++c) {
            const float2 ml = __ldcg(&p.part_ml[(blk0 + 2 * c) * BQ + i]);
            const float w = ex2(ml.x - ms);
            lt += w * ml.y;
            const float4* src = reinterpret_cast<const float4*>(p.part) + (blk0 + 2 * c) * (BQ * DH / 4) + i;
#pragma unroll
            for (int q = 0; q < DH / 4; ++q) {
              const float4 o = __ldcg(src + q * BQ);
              acc[4 * q] += w * o.x;
              acc[4 * q + 1] += w * o.y;
              acc[4 * q + 2] += w * o.z;
              acc[4 * q + 3] += w * o.w;
            }
          }
          uint16_t* dst = p.out + (static_cast<size_t>(b) * p.T + qi) * p.ldo + slot * DH;
          const float inv = 1.0f / lt;
          if (p.lse != nullptr) p.lse[static_cast<size_t>(bh) * p.lse_ld + qi] = ms + log2f(lt);
#pragma unroll
          for (int c = 0; c < DH / 32; ++c) {
            uint32_t v[32];
#pragma unroll
            for (int x = 0; x < 32; ++x) v[x] = __float_as_uint(acc[c * 32 + x]);
            store_row32(dst + c * 32, v, inv);
          }
        }
        if (threadIdx.x == 0) p.counters[bh * p.n_pairs + pair] = 0;  // ready for the next call
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    volatile int none = 0;
    mbar_wait(drain, 0, &none, 500000000ull);
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int DH>
int launch_attn(const CUtensorMap& q, const CUtensorMap& qs, const CUtensorMap& k,
                const CUtensorMap& v, const AttnParams& p, long long grid, void* stream) {
  using C = AttnCfg<DH>;
  const int e = ensure_smem<attn_kernel<DH>>(static_cast<int>(C::SMEM));
  if (e != cudaSuccess) return e;
  if (grid <= 0) return cudaSuccess;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  return launch_pdl(attn_kernel<DH>, dim3(static_cast<unsigned>(grid)), dim3(kThreads), C::SMEM,
                    stream, q, qs, k, v, p);
}

int run(const gqe_config& c, const uint16_t* Q, uint64_t nq_streams, const uint16_t* Qs,
        const uint16_t* K, const uint16_t* V, uint16_t* out, int ldo, int H, int dense, void* ws,
        size_t ws_bytes, bool counters_zeroed, void* stream, float* lse = nullptr) {
  const int dh = c.d_head;
  const AttnPlan plan = attention_plan(c, H);
  if (plan.total > 0 && (ws == nullptr || ws_bytes < plan.total)) return cudaErrorInvalidValue;
  CUtensorMap tq, tqs, tk, tv;
  if (!make_tmap_bf16_3d(&tq, Q, dh, c.T, nq_streams, dh, BQ)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_3d(&tqs, Qs ? Qs : Q, dh, c.T, Qs ? c.B : nq_streams, dh, BQ))
    return cudaErrorInvalidValue;
  if (!make_tmap_bf16_3d(&tk, K, dh, c.T, static_cast<uint64_t>(c.B) * c.G, dh, BKV))
    return cudaErrorInvalidValue;
  if (!make_tmap_bf16_3d(&tv, V, dh, c.T, static_cast<uint64_t>(c.B) * c.G, dh, BKV))
    return cudaErrorInvalidValue;
  AttnParams p{};
  p.T = c.T;
  p.B = c.B;
  p.H = H;
  p.G = c.G;
  p.k = c.k;
  p.M = c.M;
  p.dense = dense;
  p.n_qt = plan.n_qt;
  p.n_pairs = plan.n_pairs;
  p.chunk = plan.chunk;
  p.items = plan.items;
  p.out = out;
  p.ldo = ldo;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(dh)));
  p.lse = lse;
  p.lse_ld = (c.T + 63) / 64 * 64;
  char* w = static_cast<char*>(ws);
  p.part = plan.total ? reinterpret_cast<float*>(w + plan.part) : nullptr;
  p.part_ml = plan.total ? reinterpret_cast<float2*>(w + plan.ml) : nullptr;
  p.counters = plan.total ? reinterpret_cast<int*>(w + plan.counters) : nullptr;
  if (plan.total && !counters_zeroed) {
    const cudaError_t e = cudaMemsetAsync(p.counters, 0, plan.counter_bytes,
                                          static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return e;
  }
  const long long grid = static_cast<long long>(p.items) * p.B * p.H;
  if (dh == 64) return launch_attn<64>(tq, tqs, tk, tv, p, grid, stream);
  return launch_attn<32>(tq, tqs, tk, tv, p, grid, stream);
}

// Expert-major routed attention plus the shared head (one launch, no split).
int run_em(const gqe_config& c, const uint16_t* Qe, const uint16_t* Qs, const uint16_t* K,
           const uint16_t* V, const int32_t* idx, const int32_t* offsets, const int32_t* tok,
           uint16_t* slots, void* stream) {
  const int dh = c.d_head;
  const long long R = static_cast<long long>(c.B) * c.T;
  const long long rows = R * c.G * c.k;  // routed query rows, in list order
  CUtensorMap tq, tqs, tk, tv;
  if (!make_tmap_bf16_3d(&tq, Qe, dh, static_cast<uint64_t>(rows), 1, dh, BQ)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_3d(&tqs, Qs ? Qs : Qe, dh, c.T, c.B, dh, BQ)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_3d(&tk, K, dh, c.T, static_cast<uint64_t>(c.B) * c.G, dh, BKV))
    return cudaErrorInvalidValue;
  if (!make_tmap_bf16_3d(&tv, V, dh, c.T, static_cast<uint64_t>(c.B) * c.G, dh, BKV))
    return cudaErrorInvalidValue;
  AttnParams p{};
  p.T = c.T;
  p.B = c.B;
  p.H = n_streams(c);
  p.G = c.G;
  p.k = c.k;
  p.M = c.M;
  p.dense = 0;
  p.n_qt = (c.T + BQ - 1) / BQ;
  p.n_pairs = (p.n_qt + 1) / 2;
  p.chunk = p.n_qt;  // no split
  p.items = p.n_pairs;
  p.out = slots;
  p.ldo = n_slots(c) * dh;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(dh)));
  p.em = 1;
  p.N = c.G * c.M;
  // Pairs of 128-row tiles over all lists: at most rows / 256 + one partial
  // pair per list.
  p.em_units = static_cast<int>(rows / (2 * BQ) + static_cast<long long>(p.N) * c.B + 1);
  p.offsets = offsets;
  p.tok = tok;
  p.idx = idx;
  const long long grid =
      static_cast<long long>(p.em_units) + (has_shared_head(c) ? static_cast<long long>(p.n_pairs) * c.B : 0);
  if (dh == 64) return launch_attn<64>(tq, tqs, tk, tv, p, grid, stream);
  return launch_attn<32>(tq, tqs, tk, tv, p, grid, stream);
}

}  // namespace attn_impl
using namespace attn_impl;

AttnPlan attention_plan(const gqe_config& c, int H) {
  AttnPlan pl{};
  pl.n_qt = (c.T + BQ - 1) / BQ;
  pl.n_pairs = (pl.n_qt + 1) / 2;
  const long long streams = static_cast<long long>(c.B) * H;
  // One CTA per SM: with fewer pair-CTAs than SMs, the longest pair (2 query
  // tiles x n_qt KV tiles) sets the time. Split the pairs' KV ranges into the
  // smallest chunks that still fit one wave.
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  pl.chunk = pl.n_qt;
  pl.items = pl.n_pairs;
  if (static_cast<long long>(pl.n_pairs) * streams < sms) {
    for (int ch = 2; ch < pl.n_qt; ++ch) {
      int items = 0;
      for (int q = 0; q < pl.n_pairs; ++q) items += (2 * q + 1 + ch - 1) / ch;
      if (static_cast<long long>(items) * streams <= sms) {
        pl.chunk = ch;
        pl.items = items;
        break;
      }
    }
  }
  if (pl.chunk < pl.n_qt) {
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    const size_t rows = static_cast<size_t>(streams) * pl.items * 2 * BQ;
    pl.part = 0;
    pl.ml = up(rows * c.d_head * 4);
    pl.counters = up(pl.ml + rows * 8);
    pl.counter_bytes = static_cast<size_t>(streams) * pl.n_pairs * 4;
    pl.total = up(pl.counters + pl.counter_bytes);
  }
  return pl;
}

int attention_gqe(const gqe_config& c, const uint16_t* Qv, const uint16_t* Qs, const uint16_t* K,
                  const uint16_t* V, uint16_t* slots, void* ws, size_t ws_bytes,
                  bool counters_zeroed, void* stream, float* lse) {
  return run(c, Qv, static_cast<uint64_t>(c.B) * c.G * c.k, Qs, K, V, slots, n_slots(c) * c.d_head,
             n_streams(c), 0, ws, ws_bytes, counters_zeroed, stream, lse);
}

int attention_gqe_em(const gqe_config& c, const uint16_t* Qe, const uint16_t* Qs, const uint16_t* K,
                     const uint16_t* V, const int32_t* idx, const int32_t* offsets, const int32_t* tok,
                     uint16_t* slots, void* stream) {
  return run_em(c, Qe, Qs, K, V, idx, offsets, tok, slots, stream);
}

int attention_dense(const gqe_config& c, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                    uint16_t* O, void* ws, size_t ws_bytes, bool counters_zeroed, void* stream) {
  const int N = c.G * c.M;
  return run(c, Q, static_cast<uint64_t>(c.B) * N, nullptr, K, V, O, N * c.d_head, N, 1, ws,
             ws_bytes, counters_zeroed, stream);
}

int zero_attention_counters(const gqe_config& c, int H, void* ws, void* stream) {
  const AttnPlan plan = attention_plan(c, H);
  if (plan.total == 0) return cudaSuccess;
  return cudaMemsetAsync(static_cast<char*>(ws) + plan.counters, 0, plan.counter_bytes,
                         static_cast<cudaStream_t>(stream));
}

}  // namespace gqe
