// Dispatch (step a5): token lists per (expert, sequence), built from the
// router's selections in deterministic passes with no inter-CTA waits:
//   1. masks   one CTA per tile of kDispatchTile tokens of one sequence: each
//              token's selections become a bitmask over the N experts (kept
//              in the workspace), and warp ballots give the tile's count per
//              expert;
//   2. scan    exclusive prefix sum of the tile counts in (expert, sequence,
//              tile) order -> each tile's base in the lists, counts, offsets
//              and the grouped-GEMM tile table;
//   3. scatter one CTA per tile; warp ballots give every token its rank among
//              the tile's tokens of the same expert (ascending t), so the
//              lists are stable and bit-exact.
// When the tile counts are few (kFusedScanMax), every scatter CTA computes
// the prefix sum it needs itself and one more CTA writes the shared outputs,
// so steps 2 and 3 are one launch.
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
  uint64_t* masks;       // [R] selection bitmask per token
  int32_t* tile_counts;  // [N][num_tiles]
  int32_t* tile_base;    // [N][num_tiles]
  int4* qtiles;
  int32_t* n_qtiles;
  int B, T, G, M, k, N, num_tiles, tiles_per_seq, max_qtiles;
};

// Selection bitmask of one token row over the N experts (bit e = g*M + j);
// returns false if the row is not a valid top-k selection (k strictly
// increasing expert indices below M in every group). The row's G*k entries
// are loaded 16 bytes at a time when G*k is a multiple of 4.
__device__ __forceinline__ bool row_mask(const ListArgs& a, size_t row, uint64_t& mask) {
  const int GK = a.G * a.k;
  const int32_t* p = a.idx + row * GK;
  mask = 0;
  bool ok = true;
  int g = 0, s = 0, prev = -1;
  auto take = [&](int j) {
    if (s == 0) prev = -1;
    if (j > prev && j < a.M) mask |= 1ull << (g * a.M + j);
    else ok = false;
    prev = j;
    if (++s == a.k) {
      s = 0;
      ++g;
    }
  };
  if ((GK & 3) == 0) {
    const int4* p4 = reinterpret_cast<const int4*>(p);
#pragma unroll 4
    for (int q = 0; q < GK / 4; ++q) {
      const int4 v = __ldg(p4 + q);
      take(v.x);
      take(v.y);
      take(v.z);
      take(v.w);
    }
  } else {
#pragma unroll 4
    for (int q = 0; q < GK; ++q) take(__ldg(p + q));
  }
  return ok;
}

// Step 1: one CTA per tile of kDispatchTile (= kThreads) tokens, one token
// per thread; the masks go to the workspace, per-expert counts by warp
// ballots summed over the CTA's warps.
__global__ void __launch_bounds__(kThreads) mask_count_kernel(ListArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ int wc[kThreads / 32][kMaxExperts];
  const int tile = blockIdx.x;
  const int b = tile / a.tiles_per_seq;
  const int t = (tile % a.tiles_per_seq) * kDispatchTile + threadIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint64_t m = 0;
  if (t < a.T) {
    const size_t row = static_cast<size_t>(b) * a.T + t;
    if (!row_mask(a, row, m)) set_status(GQE_ERR_DEVICE_CHECK);
    a.masks[row] = m;
  }
  int c0 = 0, c1 = 0;  // lane e (e + 32): this warp's count of expert e (e + 32)
  for (int e = 0; e < a.N; ++e) {
    const int n = __popc(__ballot_sync(0xffffffffu, (m >> e) & 1ull));
    if (e == lane) c0 = n;
    if (e == lane + 32) c1 = n;
  }
  if (lane < a.N) wc[warp][lane] = c0;
  if (lane + 32 < a.N) wc[warp][lane + 32] = c1;
  __syncthreads();
  for (int e = threadIdx.x; e < a.N; e += blockDim.x) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) c += wc[w][e];
    a.tile_counts[static_cast<size_t>(e) * a.num_tiles + tile] = c;
  }
}

// Block-wide exclusive scan of one int per thread.
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

// Exclusive prefix of the flat tile counts [N][num_tiles] (= (expert,
// sequence, tile) order). Every thread sums a contiguous run; the prefix at
// each index is passed to visit(i, prefix). Returns the total.
template <typename Visit>
__device__ int tile_prefix(const ListArgs& a, Visit visit) {
  const int F = a.N * a.num_tiles;
  const int per = (F + blockDim.x - 1) / blockDim.x;
  const int lo = min(F, static_cast<int>(threadIdx.x) * per), hi = min(F, lo + per);
  int sum = 0;
#pragma unroll 4
  for (int i = lo; i < hi; ++i) sum += a.tile_counts[i];
  int total;
  int run = block_exclusive_scan(sum, &total);
  for (int i = lo; i < hi; ++i) {
    visit(i, run);
    run += a.tile_counts[i];
  }
  return total;
}

// Counts, offsets and the grouped-GEMM tile table from the tile bases (all
// of tile_base written and visible to the calling CTA).
__device__ void write_list_meta(const ListArgs& a, int total) {
  const int EB = a.N * a.B;
  const int F = a.N * a.num_tiles;
  const int per = (EB + blockDim.x - 1) / blockDim.x;
  const int lo = min(EB, static_cast<int>(threadIdx.x) * per), hi = min(EB, lo + per);
  int nq = 0;
  for (int i = lo; i < hi; ++i) {
    const int e = i / a.B, b = i % a.B;
    const int f0 = e * a.num_tiles + b * a.tiles_per_seq, f1 = f0 + a.tiles_per_seq;
    const int start = a.tile_base[f0];
    const int c = (f1 < F ? a.tile_base[f1] : total) - start;
    a.counts[i] = c;
    a.offsets[i] = start;
    nq += (c + kQTileRows - 1) / kQTileRows;
  }
  int nq_total;
  int qbase = block_exclusive_scan(nq, &nq_total);
  for (int i = lo; i < hi; ++i) {
    const int e = i / a.B, b = i % a.B;
    const int c = a.counts[i], start = a.offsets[i];
    for (int s = 0; s < c; s += kQTileRows) {
      // (expert, sequence, first list entry, rows): the GEMM reads its rows'
      // positions straight from tok.
      if (qbase < a.max_qtiles) a.qtiles[qbase] = make_int4(e, b, start + s, min(kQTileRows, c - s));
      ++qbase;
    }
  }
  if (threadIdx.x == 0) {
    a.offsets[EB] = total;
    *a.n_qtiles = min(nq_total, a.max_qtiles);
    if (nq_total > a.max_qtiles || total != a.k * a.G * a.B * a.T) set_status(GQE_ERR_DEVICE_CHECK);
  }
}

// Step 2 on its own (many tiles): one CTA of 1024 threads.
__global__ void __launch_bounds__(1024) scan_kernel(ListArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int total = tile_prefix(a, [&](int i, int pre) { a.tile_base[i] = pre; });
  __syncthreads();
  write_list_meta(a, total);
}

// The selection mask of this thread's token in tile `tile` (0 past T).
__device__ __forceinline__ uint64_t tile_token_mask(const ListArgs& a, int tile) {
  const int b = tile / a.tiles_per_seq;
  const int t = (tile % a.tiles_per_seq) * kDispatchTile + threadIdx.x;
  return t < a.T ? a.masks[static_cast<size_t>(b) * a.T + t] : 0ull;
}

// Step 3 for one tile, given the tile's list bases per expert in shared
// memory (base[e]) and this thread's token mask m.
__device__ void scatter_tile(const ListArgs& a, int tile, const int* base, uint64_t m) {
  __shared__ int wcnt[kThreads / 32][kMaxExperts];
  const int b = tile / a.tiles_per_seq;
  const int t = (tile % a.tiles_per_seq) * kDispatchTile + threadIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const size_t row = static_cast<size_t>(b) * a.T + t;
  int c0 = 0, c1 = 0;
  for (int e = 0; e < a.N; ++e) {
    const int n = __popc(__ballot_sync(0xffffffffu, (m >> e) & 1ull));
    if (e == lane) c0 = n;
    if (e == lane + 32) c1 = n;
  }
  if (lane < a.N) wcnt[warp][lane] = c0;
  if (lane + 32 < a.N) wcnt[warp][lane + 32] = c1;
  __syncthreads();
  // Exclusive prefix over the warps, per expert (one thread per expert).
  for (int e = threadIdx.x; e < a.N; e += blockDim.x) {
    int pre = base[e];
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) {
      const int c = wcnt[w][e];
      wcnt[w][e] = pre;
      pre += c;
    }
  }
  __syncthreads();
  int g = 0, j = 0;  // e = g * M + j, stepped with e
  for (int e = 0; e < a.N; ++e) {
    const bool f = (m >> e) & 1ull;
    const unsigned bal = __ballot_sync(0xffffffffu, f);
    if (f) {
      const int pos = wcnt[warp][e] + __popc(bal & lt);
      a.tok[pos] = t;
      const uint64_t gm = (m >> (g * a.M)) & ((1ull << j) - 1ull);
      a.slot_pos[(row * a.G + g) * a.k + __popcll(static_cast<long long>(gm))] = pos;
    }
    if (++j == a.M) {
      j = 0;
      ++g;
    }
  }
}

__global__ void __launch_bounds__(kThreads) scatter_kernel(ListArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ int base[kMaxExperts];
  for (int e = threadIdx.x; e < a.N; e += blockDim.x)
    base[e] = a.tile_base[static_cast<size_t>(e) * a.num_tiles + blockIdx.x];
  __syncthreads();
  scatter_tile(a, blockIdx.x, base, tile_token_mask(a, blockIdx.x));
}

// Steps 2 and 3 in one launch (few tiles): every scatter CTA scans the tile
// counts for its own bases (its tokens' masks are loaded first, so that load
// overlaps the scan); one more CTA (the last) writes tile_base, counts,
// offsets and the tile table.
constexpr int kFusedScanMax = 16384;  // N * num_tiles

__global__ void __launch_bounds__(kThreads) scan_scatter_kernel(ListArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ int base[kMaxExperts];
  const int tile = blockIdx.x;
  const bool lead = blockIdx.x == static_cast<unsigned>(a.num_tiles);
  const uint64_t m = lead ? 0ull : tile_token_mask(a, tile);
  const int F = a.N * a.num_tiles;
  const int per = (F + kThreads - 1) / kThreads;
  const int lo = min(F, static_cast<int>(threadIdx.x) * per), hi = min(F, lo + per);
  int sum = 0;
#pragma unroll 4
  for (int i = lo; i < hi; ++i) sum += a.tile_counts[i];
  int total;
  int run = block_exclusive_scan(sum, &total);
  int e = lo / a.num_tiles, tl = lo - e * a.num_tiles;  // index i = e * num_tiles + tl
  for (int i = lo; i < hi; ++i) {
    if (tl == tile) base[e] = run;
    if (lead) a.tile_base[i] = run;
    run += a.tile_counts[i];
    if (++tl == a.num_tiles) {
      tl = 0;
      ++e;
    }
  }
  __syncthreads();
  if (lead) {
    write_list_meta(a, total);
    return;
  }
  scatter_tile(a, tile, base, m);
}

// Weighted slot: one thread per 8 columns of one row.
__global__ void __launch_bounds__(256) weighted_slot_kernel(uint16_t* slots, const float* omega,
                                                            int R, int G, int k, int dh, int S) {
  pdl_wait();
  pdl_launch_dependents();
  const int per_row = dh / 8;
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= static_cast<long long>(R) * per_row) return;
  const int row = static_cast<int>(gid / per_row);
  const int c8 = static_cast<int>(gid % per_row);
  const int ld = S * dh;  // the weighted slot is the last of the S slots
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
  *reinterpret_cast<uint4*>(base + (S - 1) * dh) = o;
}

// Weighted concatenation: slots[row, gs*dh + c] *= omega[row, gs] (routed
// slots only; one thread per 8 columns, one bf16 rounding of the product).
__global__ void __launch_bounds__(256) scale_slots_kernel(uint16_t* slots, const float* omega, int R,
                                                          int gk, int dh, int ld) {
  pdl_wait();
  pdl_launch_dependents();
  const int per_row = gk * dh / 8;
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= static_cast<long long>(R) * per_row) return;
  const int row = static_cast<int>(gid / per_row);
  const int c8 = static_cast<int>(gid % per_row);
  uint16_t* p = slots + static_cast<size_t>(row) * ld + c8 * 8;
  const float w = omega[static_cast<size_t>(row) * gk + (c8 * 8) / dh];
  uint4 v = *reinterpret_cast<const uint4*>(p);
  uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    u[i] = pack_bf16x2(w * __uint_as_float(u[i] << 16), w * __uint_as_float(u[i] & 0xffff0000u));
  *reinterpret_cast<uint4*>(p) = make_uint4(u[0], u[1], u[2], u[3]);
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
  L.masks = o;
  o = align_up(o + static_cast<size_t>(R) * 8, 256);
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
  a.masks = reinterpret_cast<uint64_t*>(w + L.masks);
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
  cudaError_t e = launch_pdl(mask_count_kernel, dim3(L.num_tiles), dim3(kThreads), 0, st, a);
  if (e != cudaSuccess) return e;
  if (static_cast<long long>(a.N) * L.num_tiles <= kFusedScanMax)
    return launch_pdl(scan_scatter_kernel, dim3(L.num_tiles + 1), dim3(kThreads), 0, st, a);
  e = launch_pdl(scan_kernel, dim3(1), dim3(1024), 0, st, a);
  if (e == cudaSuccess) e = launch_pdl(scatter_kernel, dim3(L.num_tiles), dim3(kThreads), 0, st, a);
  return e;
}

int launch_weighted_slot(const gqe_config& c, uint16_t* slots, const float* omega, void* stream) {
  const long long R = static_cast<long long>(c.B) * c.T;
  const long long n = R * (c.d_head / 8);
  const int grid = static_cast<int>((n + 255) / 256);
  return launch_pdl(weighted_slot_kernel, dim3(grid), dim3(256), 0, stream, slots, omega,
                    static_cast<int>(R), c.G, c.k, c.d_head, n_slots(c));
}

}  // namespace gqe

namespace gqe {

int launch_scale_slots(const gqe_config& c, uint16_t* slots, const float* omega, void* stream) {
  const long long R = static_cast<long long>(c.B) * c.T;
  const int gk = c.G * c.k;
  const long long n = R * gk * c.d_head / 8;
  const int grid = static_cast<int>((n + 255) / 256);
  return launch_pdl(scale_slots_kernel, dim3(grid), dim3(256), 0, stream, slots, omega,
                    static_cast<int>(R), gk, c.d_head, n_slots(c) * c.d_head);
}

}  // namespace gqe
