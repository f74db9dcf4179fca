// Dispatch (step a5): token lists per (expert, sequence), built from the
// router's selections in three deterministic passes with no inter-CTA waits:
//   1. count   one CTA per tile of kDispatchTile tokens of one sequence; a
//              shared-memory histogram gives the tile's count per expert;
//   2. scan    one CTA: exclusive prefix sum of the tile counts in
//              (expert, sequence, tile) order -> each tile's base in the lists,
//              counts, offsets, and the grouped-GEMM tile table;
//   3. scatter one CTA per tile; warp ballots give every token its rank among
//              the tile's tokens of the same expert (ascending t), so the
//              lists are stable and bit-exact.
// Only the selected experts receive rows ("a router selects a sparse subset
// of k query-head experts from each GQA group": gist.science Technical
// Summary, Methodology), and every group gets exactly k entries per token.
//
// Also the weighted slot (step a10): slots[row, kG+1] = sum omega * routed
// slot ("a weighted sum of the selected expert outputs using router
// probabilities": gist.science Technical Summary, Output Construction).
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "gqe_internal.h"
#include "ptx.cuh"

namespace gqe {

namespace dispatch_impl {

constexpr int kThreads = 256;
static_assert(kDispatchTile == kThreads, "one token per thread in count/scatter");

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct ListArgs {
  const int32_t* idx;
  int32_t* counts;
  int32_t* offsets;
  int32_t* tok;
  int32_t* slot_pos;
  int32_t* tile_counts;  // [N][num_tiles]
  int32_t* tile_base;    // [N][num_tiles]
  int4* qtiles;
  int32_t* n_qtiles;
  int B, T, G, M, k, N, num_tiles, tiles_per_seq, max_qtiles;
};

// Selection bitmask of one token over the N experts (bit e = g*M + j);
// returns false if the row is not a valid top-k selection.
__device__ __forceinline__ bool token_mask(const ListArgs& a, size_t row, uint64_t& mask) {
  const int32_t* p = a.idx + row * a.G * a.k;
  mask = 0;
  bool ok = true;
  for (int g = 0; g < a.G; ++g) {
    int prev = -1;
    for (int s = 0; s < a.k; ++s) {
      const int j = p[g * a.k + s];
      if (j <= prev || j >= a.M) {
        ok = false;
        continue;
      }
      prev = j;
      mask |= 1ull << (g * a.M + j);
    }
  }
  return ok;
}

// One CTA per tile of kDispatchTile (= kThreads) tokens, one token per
// thread; per-expert counts by warp ballots, summed over the CTA's warps.
__global__ void __launch_bounds__(kThreads) count_kernel(ListArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ int wc[kThreads / 32][kMaxExperts];
  const int tile = blockIdx.x;
  const int b = tile / a.tiles_per_seq;
  const int t = (tile % a.tiles_per_seq) * kDispatchTile + threadIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint64_t m = 0;
  bool ok = true;
  if (t < a.T) ok = token_mask(a, static_cast<size_t>(b) * a.T + t, m);
  if (!ok) set_status(GQE_ERR_DEVICE_CHECK);
  for (int e = 0; e < a.N; ++e) {
    const unsigned bal = __ballot_sync(0xffffffffu, (m >> e) & 1ull);
    if (lane == 0) wc[warp][e] = __popc(bal);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < a.N; e += blockDim.x) {
    int c = 0;
    for (int w = 0; w < kThreads / 32; ++w) c += wc[w][e];
    a.tile_counts[static_cast<size_t>(e) * a.num_tiles + tile] = c;
  }
}

// Block-wide exclusive scan of one int per thread (1024 threads).
__device__ int block_exclusive_scan(int v, int* total) {
  __shared__ int warp_sums[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int w = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  const int before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
  *total = warp_sums[(blockDim.x >> 5) - 1];
  __syncthreads();
  return before;
}

__global__ void __launch_bounds__(1024) scan_kernel(ListArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int L = a.N * a.num_tiles;
  const int per = (L + blockDim.x - 1) / blockDim.x;
  const int lo = min(L, threadIdx.x * per), hi = min(L, lo + per);
  int sum = 0;
  for (int i = lo; i < hi; ++i) sum += a.tile_counts[i];
  int total;
  int run = block_exclusive_scan(sum, &total);
  for (int i = lo; i < hi; ++i) {
    a.tile_base[i] = run;
    run += a.tile_counts[i];
  }
  __syncthreads();
  // counts / offsets per (e, b); grouped-GEMM tiles per (e, b).
  const int EB = a.N * a.B;
  const int per2 = (EB + blockDim.x - 1) / blockDim.x;
  const int lo2 = min(EB, threadIdx.x * per2), hi2 = min(EB, lo2 + per2);
  int nq = 0;
  for (int i = lo2; i < hi2; ++i) {
    const int e = i / a.B, b = i % a.B;
    const size_t f0 = static_cast<size_t>(e) * a.num_tiles + static_cast<size_t>(b) * a.tiles_per_seq;
    int c = 0;
    for (int tb = 0; tb < a.tiles_per_seq; ++tb) c += a.tile_counts[f0 + tb];
    a.counts[i] = c;
    a.offsets[i] = a.tile_base[f0];
    nq += (c + kQTileRows - 1) / kQTileRows;
  }
  int nq_total;
  int qbase = block_exclusive_scan(nq, &nq_total);
  for (int i = lo2; i < hi2; ++i) {
    const int e = i / a.B, b = i % a.B;
    const int c = a.counts[i];
    for (int s = 0; s < c; s += kQTileRows) {
      if (qbase < a.max_qtiles) a.qtiles[qbase] = make_int4(e, b, s, min(kQTileRows, c - s));
      ++qbase;
    }
  }
  if (threadIdx.x == 0) {
    a.offsets[EB] = total;
    *a.n_qtiles = min(nq_total, a.max_qtiles);
    if (nq_total > a.max_qtiles || total != a.k * a.G * a.B * a.T) set_status(GQE_ERR_DEVICE_CHECK);
  }
}

__global__ void __launch_bounds__(kThreads) scatter_kernel(ListArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ int wcnt[kThreads / 32][kMaxExperts];
  __shared__ int run[kMaxExperts];
  __shared__ int base[kMaxExperts];
  const int tile = blockIdx.x;
  const int b = tile / a.tiles_per_seq;
  const int t0 = (tile % a.tiles_per_seq) * kDispatchTile;
  const int t1 = min(a.T, t0 + kDispatchTile);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned lt = (1u << lane) - 1u;
  for (int e = threadIdx.x; e < a.N; e += blockDim.x) {
    run[e] = 0;
    base[e] = a.tile_base[static_cast<size_t>(e) * a.num_tiles + tile];
  }
  __syncthreads();
  for (int c0 = t0; c0 < t1; c0 += blockDim.x) {
    const int t = c0 + threadIdx.x;
    const size_t row = static_cast<size_t>(b) * a.T + t;
    uint64_t m = 0;
    if (t < t1) token_mask(a, row, m);
    for (int e = 0; e < a.N; ++e) {
      const unsigned bal = __ballot_sync(0xffffffffu, (m >> e) & 1ull);
      if (lane == 0) wcnt[warp][e] = __popc(bal);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < a.N; e += blockDim.x) {
      int pre = run[e];
      for (int w = 0; w < kThreads / 32; ++w) {
        const int c = wcnt[w][e];
        wcnt[w][e] = pre;
        pre += c;
      }
      run[e] = pre;
    }
    __syncthreads();
    for (int e = 0; e < a.N; ++e) {
      const bool f = (m >> e) & 1ull;
      const unsigned bal = __ballot_sync(0xffffffffu, f);
      if (f) {
        const int pos = base[e] + wcnt[warp][e] + __popc(bal & lt);
        a.tok[pos] = t;
        const int g = e / a.M, j = e % a.M;
        const uint64_t gm = (m >> (g * a.M)) & ((1ull << j) - 1ull);
        const int s = __popcll(static_cast<long long>(gm));
        a.slot_pos[(row * a.G + g) * a.k + s] = pos;
      }
    }
    __syncthreads();
  }
}

// Single-CTA dispatch for small batches (kSmallRows rows or fewer): counts,
// (expert, sequence) prefix sums, stable scatter and the grouped-GEMM tile
// table in one kernel, with the same results as the three-pass path. Rows are
// visited sequence by sequence, kSmallThreads at a time (one per thread), so
// ranks within an (expert, sequence) list follow the positions t.
constexpr int kSmallThreads = 1024;

__global__ void __launch_bounds__(kSmallThreads) small_dispatch_kernel(ListArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ int wcnt[kSmallThreads / 32][kMaxExperts];
  __shared__ int run[kMaxExperts];
  extern __shared__ int eb_counts[];  // [N*B] counts, then exclusive offsets
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const int EB = a.N * a.B;
  for (int i = threadIdx.x; i < EB; i += blockDim.x) eb_counts[i] = 0;
  __syncthreads();
  // Pass 1: counts per (e, b).
  bool bad = false;
  for (int row = threadIdx.x; row < a.B * a.T; row += blockDim.x) {
    uint64_t m;
    bad |= !token_mask(a, row, m);
    const int b = row / a.T;
    while (m) {
      const int e = __ffsll(static_cast<long long>(m)) - 1;
      m &= m - 1;
      atomicAdd(&eb_counts[e * a.B + b], 1);
    }
  }
  if (bad) set_status(GQE_ERR_DEVICE_CHECK);
  __syncthreads();
  // Exclusive scan in (e, b) order; counts and offsets out; tile counts.
  int total;
  const int per = (EB + blockDim.x - 1) / blockDim.x;
  const int lo = min(EB, threadIdx.x * per), hi = min(EB, lo + per);
  int sum = 0, nq = 0;
  for (int i = lo; i < hi; ++i) {
    sum += eb_counts[i];
    nq += (eb_counts[i] + kQTileRows - 1) / kQTileRows;
  }
  int base = block_exclusive_scan(sum, &total);
  int nq_total;
  int qbase = block_exclusive_scan(nq, &nq_total);
  for (int i = lo; i < hi; ++i) {
    const int c = eb_counts[i];
    a.counts[i] = c;
    a.offsets[i] = base;
    const int e = i / a.B, b = i % a.B;
    for (int s = 0; s < c; s += kQTileRows) {
      if (qbase < a.max_qtiles) a.qtiles[qbase] = make_int4(e, b, s, min(kQTileRows, c - s));
      ++qbase;
    }
    eb_counts[i] = base;  // becomes the list start
    base += c;
  }
  if (threadIdx.x == 0) {
    a.offsets[EB] = total;
    *a.n_qtiles = min(nq_total, a.max_qtiles);
    if (nq_total > a.max_qtiles || total != a.k * a.G * a.B * a.T) set_status(GQE_ERR_DEVICE_CHECK);
  }
  __syncthreads();
  // Pass 2: stable ranks, sequence by sequence.
  for (int b = 0; b < a.B; ++b) {
    for (int e = threadIdx.x; e < a.N; e += blockDim.x) run[e] = 0;
    __syncthreads();
    for (int c0 = 0; c0 < a.T; c0 += blockDim.x) {
      const int t = c0 + threadIdx.x;
      const size_t row = static_cast<size_t>(b) * a.T + t;
      uint64_t m = 0;
      if (t < a.T) token_mask(a, row, m);
      for (int e = 0; e < a.N; ++e) {
        const unsigned bal = __ballot_sync(0xffffffffu, (m >> e) & 1ull);
        if (lane == 0) wcnt[warp][e] = __popc(bal);
      }
      __syncthreads();
      for (int e = threadIdx.x; e < a.N; e += blockDim.x) {
        int pre = run[e];
        for (int w = 0; w < kSmallThreads / 32; ++w) {
          const int c = wcnt[w][e];
          wcnt[w][e] = pre;
          pre += c;
        }
        run[e] = pre;
      }
      __syncthreads();
      for (int e = 0; e < a.N; ++e) {
        const bool f = (m >> e) & 1ull;
        const unsigned bal = __ballot_sync(0xffffffffu, f);
        if (f) {
          const int pos = eb_counts[e * a.B + b] + wcnt[warp][e] + __popc(bal & lt);
          a.tok[pos] = t;
          const int g = e / a.M, j = e % a.M;
          const uint64_t gm = (m >> (g * a.M)) & ((1ull << j) - 1ull);
          a.slot_pos[(row * a.G + g) * a.k + __popcll(static_cast<long long>(gm))] = pos;
        }
      }
      __syncthreads();
    }
  }
}

// Weighted slot: one thread per 8 columns of one row.
__global__ void __launch_bounds__(256) weighted_slot_kernel(uint16_t* slots, const float* omega,
                                                            int R, int G, int k, int dh) {
  pdl_wait();
  pdl_launch_dependents();
  const int per_row = dh / 8;
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= static_cast<long long>(R) * per_row) return;
  const int row = static_cast<int>(gid / per_row);
  const int c8 = static_cast<int>(gid % per_row);
  const int ld = (k * G + 2) * dh;
  uint16_t* base = slots + static_cast<size_t>(row) * ld + c8 * 8;
  const float* w = omega + static_cast<size_t>(row) * G * k;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
  for (int gs = 0; gs < G * k; ++gs) {
    const float wi = w[gs];
    const uint4 v = *reinterpret_cast<const uint4*>(base + gs * dh);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] = fmaf(wi, __uint_as_float(u[i] << 16), acc[2 * i]);
      acc[2 * i + 1] = fmaf(wi, __uint_as_float(u[i] & 0xffff0000u), acc[2 * i + 1]);
    }
  }
  uint4 o;
  o.x = pack_bf16x2(acc[0], acc[1]);
  o.y = pack_bf16x2(acc[2], acc[3]);
  o.z = pack_bf16x2(acc[4], acc[5]);
  o.w = pack_bf16x2(acc[6], acc[7]);
  *reinterpret_cast<uint4*>(base + (k * G + 1) * dh) = o;
}

}  // namespace dispatch_impl
using namespace dispatch_impl;

DispatchWs dispatch_ws_layout(const gqe_config& c) {
  DispatchWs L{};
  const int N = c.G * c.M;
  L.tiles_per_seq = (c.T + kDispatchTile - 1) / kDispatchTile;
  L.num_tiles = c.B * L.tiles_per_seq;
  const long long R = static_cast<long long>(c.B) * c.T;
  L.max_qtiles = static_cast<int>((static_cast<long long>(c.k) * c.G * R) / kQTileRows + N * c.B + 1);
  size_t o = 0;
  L.tile_counts = o;
  o = align_up(o + static_cast<size_t>(N) * L.num_tiles * 4, 256);
  L.tile_base = o;
  o = align_up(o + static_cast<size_t>(N) * L.num_tiles * 4, 256);
  L.qtiles = o;
  o = align_up(o + static_cast<size_t>(L.max_qtiles) * 16, 256);
  L.n_qtiles = o;
  o = align_up(o + 4, 256);
  L.total = o;
  return L;
}

int launch_dispatch_lists(const gqe_config& c, const int32_t* idx, int32_t* counts,
                          int32_t* offsets, int32_t* tok, int32_t* slot_pos, void* ws,
                          const DispatchWs& L, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  ListArgs a;
  a.idx = idx;
  a.counts = counts;
  a.offsets = offsets;
  a.tok = tok;
  a.slot_pos = slot_pos;
  a.tile_counts = reinterpret_cast<int32_t*>(w + L.tile_counts);
  a.tile_base = reinterpret_cast<int32_t*>(w + L.tile_base);
  a.qtiles = reinterpret_cast<int4*>(w + L.qtiles);
  a.n_qtiles = reinterpret_cast<int32_t*>(w + L.n_qtiles);
  a.B = c.B;
  a.T = c.T;
  a.G = c.G;
  a.M = c.M;
  a.k = c.k;
  a.N = c.G * c.M;
  a.num_tiles = L.num_tiles;
  a.tiles_per_seq = L.tiles_per_seq;
  a.max_qtiles = L.max_qtiles;
  const long long R = static_cast<long long>(c.B) * c.T;
  if (R <= kSmallRows && static_cast<long long>(a.N) * c.B <= 8192) {
    const size_t smem = static_cast<size_t>(a.N) * c.B * 4;
    return launch_pdl(small_dispatch_kernel, dim3(1), dim3(kSmallThreads), smem, st, a);
  }
  cudaError_t e = launch_pdl(count_kernel, dim3(L.num_tiles), dim3(kThreads), 0, st, a);
  if (e == cudaSuccess) e = launch_pdl(scan_kernel, dim3(1), dim3(1024), 0, st, a);
  if (e == cudaSuccess) e = launch_pdl(scatter_kernel, dim3(L.num_tiles), dim3(kThreads), 0, st, a);
  return e;
}

int launch_weighted_slot(const gqe_config& c, uint16_t* slots, const float* omega, void* stream) {
  const long long R = static_cast<long long>(c.B) * c.T;
  const long long n = R * (c.d_head / 8);
  const int grid = static_cast<int>((n + 255) / 256);
  return launch_pdl(weighted_slot_kernel, dim3(grid), dim3(256), 0, stream, slots, omega,
                    static_cast<int>(R), c.G, c.k, c.d_head);
}

}  // namespace gqe
