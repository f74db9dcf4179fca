// tcgen05 GEMM for the projections of the layer: C[128 x BN] tiles of
// A[rows, K] (bf16, K contiguous) times B[K, N] (bf16, N contiguous), fp32
// accumulation in tensor memory, bf16 output through a scatter epilogue.
//
//  - K/V projection (step a6) and the shared-head / dense query projections:
//    A tiles come from TMA (128B swizzle), the epilogue writes head-split
//    layouts [b][h][t][dh].
//  - Routed query projection (step a7, "only the selected query experts"):
//    one tile = up to 128 consecutive entries of one (expert, sequence) token
//    list; the A rows are gathered with cp.async into the same swizzled
//    layout TMA would produce, and the epilogue writes each row to its
//    slot-major stream Qv[b][g][s][t][:]. With at least two tiles per SM,
//    qgemm_kernel (below) walks the tiles with one CTA per SM and keeps the
//    expert's weights resident; otherwise gemm_kernel<BN, true> takes one
//    tile per CTA.
//  - W_O projection (step a11): plain row-major output. With d_head = 64 the
//    weighted slot (step a10) is exactly one K block of A: the epilogue warps,
//    idle during the main loop, sum it from the routed slots' stages as they
//    land (weighted by omega), write it into that K block's stage in the
//    swizzled layout (and, in the CTAs of the first column tile, back to the
//    slot buffer), and the TMA warp
//    loads only B for that block.
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 issues the UMMAs
// (one thread) and owns the TMEM allocation, warps 2-5 gather A rows (routed
// mode) and run the epilogue (warp w reads TMEM lanes 32*(w%4)..+31).
// B is read MN-major: 64-column (or 32-column) boxes, LBO = distance between
// column boxes, SBO = 8 rows.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "gqe_internal.h"
#include "ptx.cuh"
#include "tmap.h"

namespace gqe {

namespace gemm_impl {

constexpr int BM = 128;
constexpr int BK = 64;

template <int BN>
struct GemmCfg {
  static constexpr int B_ATOM = BN >= 64 ? 64 : BN;  // B columns per swizzle row
  static constexpr int B_SWB = B_ATOM * 2;           // bytes per B swizzle row
  static constexpr uint32_t B_LAYOUT = B_SWB == 128 ? kLayoutSW128 : kLayoutSW64;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BK * BN * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // Tiles up to 128 wide keep two CTAs per SM (<= ~113 KB of shared memory
  // each): small projections are latency-bound and the second CTA hides it.
  static constexpr int STAGES = BN <= 128 ? (110 * 1024) / STAGE_BYTES : 4;
  static constexpr uint32_t TMEM_COLS = BN < 32 ? 32 : BN;
  static constexpr size_t SMEM = 1024 + static_cast<size_t>(STAGES) * STAGE_BYTES + 256;
};

struct Epi {
  uint16_t* out;
  long long sb, sh, st;  // element strides of sequence, head, token
  int T;                 // rows per sequence
  int hd;                // columns per head
  int rows, cols;        // valid extent of C
  // Weighted-slot fusion (W_O projection): K block kb_w of A is
  // sum_gs omega[row, gs] * A[row, gs*BK ...] over gs < gk, computed in the
  // kernel (kb_w < 0: off).
  int kb_w = -1;
  int gk = 0;
  const float* omega = nullptr;
  uint16_t* wslots = nullptr;  // A itself, written back by the blockIdx.y == 0 CTAs
  int lda = 0;                 // A row length (elements)
  // fp32 output instead (row-major, row stride ldf): C[row, col] for
  // row < rows, col < cols. fvec: ldf and outf allow 16-byte stores.
  float* outf = nullptr;
  long long ldf = 0;
  int fvec = 0;
  // Routed head-split output (every expert's queries computed, only the
  // routed ones stored): column block h is expert h of the row's token; it
  // goes to slot s of its group, out + ((b G + g) k + s) sh + t st + c, where
  // sel[row][g][s] == h % M; rows that did not select h store nothing.
  const int32_t* sel = nullptr;
  int G = 0, M = 0, k = 0;
  int h0 = 0;  // expert of column block 0 (a launch over a slice of the experts)
  // The main loop reads only the layer's inputs (x, W), complete before the
  // previous kernel started, since every kernel of the chain lets its
  // dependents start only after its own wait. So it runs while the previous
  // kernel (the router) finishes, and the epilogue threads wait for that kernel
  // before they read its selections or store anything.
  int late_wait = 0;
};

struct Gather {
  const uint16_t* x;
  const int32_t* tok;
  const int4* qtiles;
  const int32_t* n_qtiles;
  const int32_t* idx;
  uint16_t* Qv;
  uint16_t* Qs;     // shared-head output [B*T, dh] (tiles after the routed ones)
  int max_qtiles;   // CTAs reserved for routed tiles
  int d, T, G, M, k, B, dh;
  int expert_major;  // routed rows go to Qv[list entry] (token-list order)
};

__device__ __forceinline__ void store32_bf16(uint16_t* dst, const uint32_t (&v)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 o;
    o.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
    o.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
    o.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
    o.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
    d4[q] = o;
  }
}

template <int BN, bool GATHER>
__global__ void __launch_bounds__(192, 2)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
                const __grid_constant__ CUtensorMap tmB3, const __grid_constant__ Epi epi0,
                const __grid_constant__ Epi epi1, const __grid_constant__ Epi epi2,
                const __grid_constant__ Epi epi3,
                const Gather ga, const int K) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sp = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sA = sp;
  uint8_t* sB = sp + C::STAGES * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + C::STAGES * C::B_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* accb = empty + C::STAGES;
  uint64_t* drain = accb + 1;
  uint64_t* wfree = drain + 1;   // weighted slot: its stage is free (producer arrives)
  uint64_t* wready = wfree + 1;  // weighted slot: its tile is in shared memory (128 arrivals)
  uint32_t* tslot = reinterpret_cast<uint32_t*>(wready + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool z1 = blockIdx.z == 1 || (GATHER && blockIdx.x >= static_cast<unsigned>(ga.max_qtiles));
  // Output z of up to four (B operand, epilogue) pairs of one launch.
  const int zi = GATHER ? (z1 ? 1 : 0) : static_cast<int>(blockIdx.z);
  const CUtensorMap* tmB = zi == 0 ? &tmB0 : zi == 1 ? &tmB1 : zi == 2 ? &tmB2 : &tmB3;
  const Epi& epi = zi == 0 ? epi0 : zi == 1 ? epi1 : zi == 2 ? epi2 : epi3;

  const int nk = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], GATHER ? 129u : 1u);
      // With the weighted slot fused, the 128 epilogue threads read every
      // stage too and release it along with the UMMAs.
      mbar_init(&empty[s], (!GATHER && epi.kb_w >= 0) ? 129u : 1u);
    }
    mbar_init(accb, 1u);
    mbar_init(drain, 1u);
    mbar_init(wfree, 1u);
    mbar_init(wready, 128u);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    if (!GATHER) prefetch_tmap(&tmA);
    prefetch_tmap(tmB);
  }
  if (warp == 1) tmem_alloc(tslot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const bool late = !GATHER && epi.late_wait != 0;
  if (!late) pdl_wait();
  pdl_launch_dependents();

  // Tile of this CTA (read after pdl_wait: the routed tile table is produced
  // by the dispatch kernels).
  int m0 = 0, n0 = 0, e = 0, b = 0, list0 = 0, rows = 0;
  bool shared_tile = false, skip = false;
  if (GATHER) {
    const int q = blockIdx.x;
    if (q < ga.max_qtiles) {
      // Routed tile: up to 128 consecutive entries of one (expert, sequence)
      // token list; slots past the table's length have nothing to do.
      if (q >= *ga.n_qtiles) {
        skip = true;
      } else {
        const int4 qt = ga.qtiles[q];
        e = qt.x;
        b = qt.y;
        list0 = qt.z;
        rows = qt.w;
        n0 = e * ga.dh;
      }
    } else {
      // Shared-head tile: 128 consecutive rows of x (all tokens).
      shared_tile = true;
      m0 = (q - ga.max_qtiles) * BM;
      rows = min(BM, ga.B * ga.T - m0);
    }
  } else {
    m0 = blockIdx.x * BM;
    n0 = blockIdx.y * BN;
  }

  if (skip) {
    // nothing to compute: fall through to the teardown
  } else if (warp == 0) {
    if (lane == 0) {
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % C::STAGES;
        const uint32_t ph = (kb / C::STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) break;
        const bool wblk = !GATHER && kb == epi.kb_w;
        if (wblk) {  // A of this block is computed by the epilogue warps
          mbar_arrive(wfree);
          if (!mbar_wait(wready, 0, abort_flag)) break;
        }
        mbar_arrive_expect_tx(&full[s], (GATHER || wblk ? 0 : C::A_BYTES) + C::B_BYTES);
        if (!GATHER && !wblk) tma_load_2d(sA + s * C::A_BYTES, &tmA, &full[s], kb * BK, m0);
#pragma unroll
        for (int c = 0; c < BN / C::B_ATOM; ++c)
          tma_load_2d(sB + s * C::B_BYTES + c * (BK * C::B_SWB), tmB, &full[s],
                      n0 + c * C::B_ATOM, kb * BK);
      }
    }
  } else if (warp == 1) {
    // The whole warp runs the issue loop; elect.sync picks the issuing lane.
    constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, 0, 1);
    // Base descriptors built once; stage / k offsets are added to the
    // start-address field (units of 16 bytes; addresses stay below 2^18).
    const uint64_t dA = smem_desc(smem_u32(sA), 16, 1024, kLayoutSW128);
    const uint64_t dB = smem_desc(smem_u32(sB), BK * C::B_SWB, 8 * C::B_SWB, C::B_LAYOUT);
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % C::STAGES;
      const uint32_t ph = (kb / C::STAGES) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, abort_flag))) break;
      tc_fence_after();
      const uint64_t a0 = dA + static_cast<uint64_t>((s * C::A_BYTES) >> 4);
      const uint64_t b0 = dB + static_cast<uint64_t>((s * C::B_BYTES) >> 4);
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk)
        umma_bf16_ss_elect(tmem, a0 + 2 * kk, b0 + (kk * 16 * C::B_SWB) / 16, idesc,
                           (kb | kk) != 0 ? 1u : 0u);
      umma_commit_elect(&empty[s]);
    }
    umma_commit_elect(accb);
    umma_commit_elect(drain);
  } else {
    const int q = warp & 3;
    if (GATHER) {
      // 128 threads gather the A tile: in pass r, thread i copies 16-byte
      // chunk (i % 8) of row 16 r + i / 8, so each warp instruction moves four
      // whole 128-byte row segments. Rows past the tile's end are zero-filled.
      // A stage is published LA = STAGES - 2 blocks after its copies were
      // issued: with LA = STAGES - 1 the copy into a stage would wait for
      // the UMMAs of the stage published just before it (measured 12 % slower
      // at T = 32k).
      const int i = threadIdx.x - 64;
      const int chunk = i & 7;
      const uint16_t* src[8];
      uint32_t nbytes[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int row = r * 16 + (i >> 3);
        const bool valid = row < rows;
        size_t xrow = 0;
        if (valid) xrow = shared_tile ? static_cast<size_t>(m0 + row)
                                      : static_cast<size_t>(b) * ga.T + ga.tok[list0 + row];
        src[r] = ga.x + xrow * ga.d + chunk * 8;
        nbytes[r] = valid ? 16u : 0u;
      }
      const uint32_t a0 = smem_u32(sA);
      constexpr int LA = C::STAGES - 2;
      int kb = 0;
      for (; kb < nk; ++kb) {
        const int s = kb % C::STAGES;
        const uint32_t ph = (kb / C::STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) break;
        const uint32_t dst = a0 + s * C::A_BYTES;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const int row = r * 16 + (i >> 3);
          cp_async_16(dst + row * 128 + ((chunk ^ (row & 7)) << 4), src[r] + kb * BK, nbytes[r]);
        }
        cp_async_commit();
        if (kb >= LA) {
          cp_async_wait<LA>();
          fence_proxy_async_smem();
          mbar_arrive(&full[(kb - LA) % C::STAGES]);
        }
      }
      cp_async_wait<0>();
      fence_proxy_async_smem();
      for (int k2 = (kb - LA > 0 ? kb - LA : 0); k2 < kb; ++k2) mbar_arrive(&full[k2 % C::STAGES]);
    }
    if (!GATHER && epi.kb_w >= 0) {
      // Weighted slot: the same fp32 sum, in the same order, as the
      // stand-alone weighted-slot kernel, rounded to bf16. The kG routed
      // slots are the first K blocks of A, so the sum is taken from their
      // stages as they land: thread i takes 16-byte chunk i % 8 of rows
      // i / 8, i / 8 + 16, ... (8 threads read one slot row segment
      // together), and these threads release every stage along with the
      // UMMAs. The sum goes into the weighted block's stage once that stage
      // is free, and (first column tile) into the slot buffer. Rows past the
      // end are zero in the stages and get omega 0.
      const int i = threadIdx.x - 64;
      const int c = i & 7;
      float acc[8][8];
#pragma unroll
      for (int pass = 0; pass < 8; ++pass)
#pragma unroll
        for (int x = 0; x < 8; ++x) acc[pass][x] = 0.0f;
      // omega of this thread's rows for slot gs (read one block ahead).
      auto omega_of = [&](int gs, float (&w)[8]) {
#pragma unroll
        for (int pass = 0; pass < 8; ++pass) {
          const int row = m0 + pass * 16 + (i >> 3);
          w[pass] = (gs < epi.gk && row < epi.rows) ? __ldg(epi.omega + static_cast<size_t>(row) * epi.gk + gs)
                                                    : 0.0f;
        }
      };
      float wn[8];
      omega_of(0, wn);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % C::STAGES;
        const uint32_t ph = (kb / C::STAGES) & 1;
        if (kb == epi.kb_w) {
          uint4 o[8];
#pragma unroll
          for (int pass = 0; pass < 8; ++pass) {
            o[pass] = make_uint4(pack_bf16x2(acc[pass][0], acc[pass][1]), pack_bf16x2(acc[pass][2], acc[pass][3]),
                                 pack_bf16x2(acc[pass][4], acc[pass][5]), pack_bf16x2(acc[pass][6], acc[pass][7]));
            const int row = m0 + pass * 16 + (i >> 3);
            if (blockIdx.y == 0 && row < epi.rows)
              *reinterpret_cast<uint4*>(epi.wslots + static_cast<size_t>(row) * epi.lda + epi.kb_w * BK +
                                        c * 8) = o[pass];
          }
          if (!mbar_wait(wfree, 0, abort_flag)) break;
          uint8_t* stage = sA + s * C::A_BYTES;
#pragma unroll
          for (int pass = 0; pass < 8; ++pass) {
            const int r = pass * 16 + (i >> 3);
            *reinterpret_cast<uint4*>(stage + r * 128 + ((c ^ (r & 7)) << 4)) = o[pass];
          }
          fence_proxy_async_smem();
          mbar_arrive(wready);
        }
        if (!mbar_wait(&full[s], ph, abort_flag)) break;
        if (kb < epi.gk) {
          float w[8];
#pragma unroll
          for (int pass = 0; pass < 8; ++pass) w[pass] = wn[pass];
          omega_of(kb + 1, wn);
          const uint8_t* stage = sA + s * C::A_BYTES;
#pragma unroll
          for (int pass = 0; pass < 8; ++pass) {
            const int r = pass * 16 + (i >> 3);
            const uint4 v = *reinterpret_cast<const uint4*>(stage + r * 128 + ((c ^ (r & 7)) << 4));
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i2 = 0; i2 < 4; ++i2) {
              acc[pass][2 * i2] = fmaf(w[pass], __uint_as_float(u[i2] << 16), acc[pass][2 * i2]);
              acc[pass][2 * i2 + 1] = fmaf(w[pass], __uint_as_float(u[i2] & 0xffff0000u), acc[pass][2 * i2 + 1]);
            }
          }
        }
        mbar_arrive(&empty[s]);
      }
    }
    if (late) pdl_wait();
    const bool have = mbar_wait(accb, 0, abort_flag);
    tc_fence_after();
    const int r = q * 32 + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
    if (GATHER) {
      const bool valid = have && r < rows;
      size_t obase = 0;
      if (valid && shared_tile) {
        obase = static_cast<size_t>(m0 + r) * ga.dh;
      } else if (valid && ga.expert_major) {
        obase = static_cast<size_t>(list0 + r) * ga.dh;
      } else if (valid) {
        const int t = ga.tok[list0 + r];
        const int g = e / ga.M, j = e % ga.M;
        const int32_t* ip = ga.idx + ((static_cast<size_t>(b) * ga.T + t) * ga.G + g) * ga.k;
        int s = 0;
        for (int s2 = 0; s2 < ga.k; ++s2)
          if (ip[s2] == j) s = s2;
        obase = (((static_cast<size_t>(b) * ga.G + g) * ga.k + s) * ga.T + t) * ga.dh;
      }
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(trow + cc * 32, v);
        if (valid) store32_bf16((shared_tile ? ga.Qs : ga.Qv) + obase + cc * 32, v);
      }
    } else if (epi.outf != nullptr) {
      const int row = m0 + r;
      const bool valid = have && row < epi.rows;
      float* orow = epi.outf + static_cast<long long>(row) * epi.ldf;
#pragma unroll 1
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(trow + cc * 32, v);
        const int col0 = n0 + cc * 32;
        if (!valid || col0 >= epi.cols) continue;
        if (epi.fvec && col0 + 32 <= epi.cols) {
          float4* d4 = reinterpret_cast<float4*>(orow + col0);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            d4[q4] = make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                 __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (col0 + j < epi.cols) orow[col0 + j] = __uint_as_float(v[j]);
        }
      }
    } else {
      const int row = m0 + r;
      const bool valid = have && row < epi.rows;
      const int bb = row / epi.T, t = row % epi.T;
#pragma unroll 1
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(trow + cc * 32, v);
        const int col0 = n0 + cc * 32;
        if (valid && col0 < epi.cols) {
          const int h = col0 / epi.hd, c = col0 % epi.hd;
          if (epi.sel != nullptr) {
            const int g = (epi.h0 + h) / epi.M, j = epi.h0 + h - g * epi.M;
            const int32_t* ip = epi.sel + (static_cast<size_t>(row) * epi.G + g) * epi.k;
            for (int s2 = 0; s2 < epi.k; ++s2)
              if (__ldg(ip + s2) == j)
                store32_bf16(epi.out + ((static_cast<long long>(bb) * epi.G + g) * epi.k + s2) * epi.sh +
                                 t * epi.st + c, v);
          } else {
            store32_bf16(epi.out + bb * epi.sb + (epi.h0 + h) * epi.sh + t * epi.st + c, v);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (*abort_flag) {
      // Let every issued UMMA finish before the columns are released.
      volatile int none = 0;
      mbar_wait(drain, 0, &none, 500000000ull);
    }
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Routed + shared query projection with the expert's weights resident. The
// tile sequence (the routed tiles of the dispatch tile table, expert-major,
// then the shared-head tiles of 128 consecutive x rows) is cut into one
// contiguous range per CTA, one CTA per SM. A CTA keeps the W_q columns of
// its current expert (d x d_head, all K blocks) in shared memory and loads
// them again only when the expert changes, so per tile only the gathered A
// rows cross from L2; the accumulator alternates between two TMEM buffers,
// so one tile's epilogue overlaps the next tile's main loop.
//
// Warp roles (32 (2 + GW + 4) threads): warp 0 loads the expert's weights
// with TMA; warp 1 issues the UMMAs (one elected thread) and owns the TMEM
// allocation; GW warps gather the A rows with cp.async, with the next tile's
// row positions read while the current tile streams; 4 warps drain the
// accumulators (warp w reads TMEM lanes 32*(w%4)..+31) and write each row to
// its stream.
template <int DH>
struct QCfg {
  static constexpr int BN = DH;
  static constexpr int B_ATOM = DH >= 64 ? 64 : DH;
  static constexpr int B_SWB = B_ATOM * 2;
  static constexpr uint32_t B_LAYOUT = B_SWB == 128 ? kLayoutSW128 : kLayoutSW64;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BK * BN * 2;  // one K block of the weights
  static constexpr int W_MAX = 128 * 1024;     // resident weights: d * d_head * 2 bytes at most
  static constexpr int STAGES = 6;             // A ring
  static constexpr uint32_t TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;
  static constexpr size_t SMEM = 1024 + W_MAX + static_cast<size_t>(STAGES) * A_BYTES + 512;
};
constexpr int kQGatherWarps = 8;
constexpr int q_threads(int gw) { return 32 * (2 + gw + 4); }

// Entry v of the tile sequence as (expert, or -1 for a shared-head tile;
// sequence; first list entry, or first row of x; rows).
__device__ __forceinline__ int4 q_entry(const Gather& ga, int v, int n_routed) {
  if (v < n_routed) return ga.qtiles[v];
  const int m0 = (v - n_routed) * BM;
  return make_int4(-1, 0, m0, min(BM, ga.B * ga.T - m0));
}

// The x rows that gather thread i of GW warps copies for tile entry q: rows
// 4 GW r + i / 8 (r < 32 / GW), 16-byte chunk i % 8 of each K block; bit r
// of `valid` is set for rows inside the tile.
template <int GW>
__device__ __forceinline__ void q_rows(const Gather& ga, int4 q, int i, const uint16_t* (&src)[32 / GW],
                                       uint32_t& valid) {
  valid = 0;
#pragma unroll
  for (int r = 0; r < 32 / GW; ++r) {
    const int row = r * 4 * GW + (i >> 3);
    size_t xrow = 0;
    if (row < q.w) {
      xrow = q.x < 0 ? static_cast<size_t>(q.z + row)
                     : static_cast<size_t>(q.y) * ga.T + ga.tok[q.z + row];
      valid |= 1u << r;
    }
    src[r] = ga.x + xrow * ga.d + (i & 7) * 8;
  }
}

template <int DH, int GW>
__global__ void __launch_bounds__(q_threads(GW), 1)
    qgemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmWs,
                 const Gather ga, const int n_shared) {
  using C = QCfg<DH>;
  constexpr int BN = C::BN;
  constexpr int GT = 32 * GW;     // gather threads
  constexpr int NPASS = 32 / GW;  // 16-byte copies per gather thread per stage
  constexpr int EPI0 = 2 + GW;    // first epilogue warp
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sp = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sW = sp;                // [nk][B_BYTES]
  uint8_t* sA = sp + C::W_MAX;     // [STAGES][A_BYTES]
  uint64_t* full = reinterpret_cast<uint64_t*>(sA + C::STAGES * C::A_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;  // [2]: accumulator a holds a finished tile
  uint64_t* acc_empty = acc_full + 2;      // [2]: accumulator a was read (128 arrivals)
  uint64_t* w_full = acc_empty + 2;        // the current weights are in
  uint64_t* w_free = w_full + 1;           // every UMMA reading the current weights is done
  uint64_t* drain = w_free + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = (ga.d + BK - 1) / BK;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], GT);
      mbar_init(&empty[s], 1u);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1u);
      mbar_init(&acc_empty[a], 128u);
    }
    mbar_init(w_full, 1u);
    mbar_init(w_free, 1u);
    mbar_init(drain, 1u);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmWs);
  }
  if (warp == 1) tmem_alloc(tslot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  pdl_wait();  // the tile table and the token lists come from the dispatch kernels
  pdl_launch_dependents();
  const int n_routed = *ga.n_qtiles;
  const int nv = n_routed + n_shared;
  // This CTA's contiguous range of tiles [vb, ve).
  const int per = nv / static_cast<int>(gridDim.x), extra = nv % static_cast<int>(gridDim.x);
  const int c = static_cast<int>(blockIdx.x);
  const int vb = c * per + min(c, extra), ve = vb + per + (c < extra ? 1 : 0);

  if (warp == 0) {
    if (lane == 0) {
      int key = -2;     // expert whose weights are resident (-1: W_qs)
      uint32_t wl = 0;  // weight loads issued
      for (int v = vb; v < ve; ++v) {
        const int e = q_entry(ga, v, n_routed).x;
        if (e == key) continue;
        // The previous weights are released once every UMMA reading them is done.
        if (!mbar_wait(w_free, (wl & 1u) ^ 1u, abort_flag)) break;
        mbar_arrive_expect_tx(w_full, static_cast<uint32_t>(nk * C::B_BYTES));
        const CUtensorMap* tm = e < 0 ? &tmWs : &tmW;
        const int n0 = e < 0 ? 0 : e * ga.dh;
        for (int kb = 0; kb < nk; ++kb) {
#pragma unroll
          for (int cc = 0; cc < BN / C::B_ATOM; ++cc)
            tma_load_2d(sW + kb * C::B_BYTES + cc * (BK * C::B_SWB), tm, w_full, n0 + cc * C::B_ATOM,
                        kb * BK);
        }
        key = e;
        ++wl;
      }
    }
  } else if (warp == 1) {
    constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, 0, 1);
    const uint64_t dA = smem_desc(smem_u32(sA), 16, 1024, kLayoutSW128);
    const uint64_t dW = smem_desc(smem_u32(sW), BK * C::B_SWB, 8 * C::B_SWB, C::B_LAYOUT);
    uint32_t kbg = 0, wl = 0;
    bool ok = true;
    int it = 0, key = -2;
    int e_next = vb < ve ? q_entry(ga, vb, n_routed).x : -2;
    for (int v = vb; ok && v < ve; ++v, ++it) {
      const int e = e_next;
      e_next = v + 1 < ve ? q_entry(ga, v + 1, n_routed).x : -2;
      if (e != key) {
        if (!__all_sync(0xffffffffu, mbar_wait(w_full, wl & 1u, abort_flag))) break;
        key = e;
        ++wl;
      }
      const int a = it & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_empty[a], ((it >> 1) & 1) ^ 1u, abort_flag))) break;
      tc_fence_after();
      const uint32_t d = tmem + a * BN;
      for (int kb = 0; kb < nk; ++kb, ++kbg) {
        const int s = static_cast<int>(kbg % C::STAGES);
        const uint32_t ph = (kbg / C::STAGES) & 1u;
        if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t a0 = dA + static_cast<uint64_t>((s * C::A_BYTES) >> 4);
        const uint64_t b0 = dW + static_cast<uint64_t>((kb * C::B_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          umma_bf16_ss_elect(d, a0 + 2 * kk, b0 + (kk * 16 * C::B_SWB) / 16, idesc,
                             (kb | kk) != 0 ? 1u : 0u);
        umma_commit_elect(&empty[s]);
      }
      if (!ok) break;
      umma_commit_elect(&acc_full[a]);
      if (e_next != key) umma_commit_elect(w_free);  // the next tile needs other weights
    }
    umma_commit_elect(drain);
  } else if (warp < EPI0) {
    // Gather: in pass r, thread i copies 16-byte chunk (i % 8) of row
    // 4 GW r + i / 8 of the K block, so each warp instruction moves four whole
    // 128-byte row segments into the 128B-swizzled stage. Rows past the
    // tile's end are zero-filled. A stage is published (fence + arrival) once
    // this thread's copies into it have landed, LA blocks later; LA below the
    // ring depth leaves the stage that the next copy waits for already
    // published, so the copies never wait on the UMMAs they feed.
    const int i = threadIdx.x - 64;
    const int chunk = i & 7;
    constexpr uint32_t LA = C::STAGES / 2;
    const uint32_t a0 = smem_u32(sA);
    const uint16_t* src[NPASS];
    uint32_t valid = 0;
    int4 qn = make_int4(-1, 0, 0, 0);
    if (vb < ve) q_rows<GW>(ga, q_entry(ga, vb, n_routed), i, src, valid);
    if (vb + 1 < ve) qn = q_entry(ga, vb + 1, n_routed);
    uint32_t kbg = 0;
    bool ok = true;
    for (int v = vb; ok && v < ve; ++v) {
      // Row positions of the next tile (its entry was read one tile ago) and
      // the entry of the one after, read now and used a tile later.
      const uint16_t* nsrc[NPASS];
      uint32_t nvalid = 0;
      if (v + 1 < ve) q_rows<GW>(ga, qn, i, nsrc, nvalid);
      if (v + 2 < ve) qn = q_entry(ga, v + 2, n_routed);
      for (int kb = 0; kb < nk; ++kb, ++kbg) {
        const int s = static_cast<int>(kbg % C::STAGES);
        const uint32_t ph = (kbg / C::STAGES) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t dst = a0 + s * C::A_BYTES;
#pragma unroll
        for (int r = 0; r < NPASS; ++r) {
          const int row = r * 4 * GW + (i >> 3);
          cp_async_16(dst + row * 128 + ((chunk ^ (row & 7)) << 4), src[r] + kb * BK,
                      (valid >> r) & 1u ? 16u : 0u);
        }
        cp_async_commit();
        if (kbg >= LA) {
          cp_async_wait<LA>();
          fence_proxy_async_smem();
          mbar_arrive(&full[(kbg - LA) % C::STAGES]);
        }
      }
      if (v + 1 < ve) {
#pragma unroll
        for (int r = 0; r < NPASS; ++r) src[r] = nsrc[r];
        valid = nvalid;
      }
    }
    cp_async_wait<0>();
    fence_proxy_async_smem();
    for (uint32_t k2 = kbg > LA ? kbg - LA : 0u; k2 < kbg; ++k2) mbar_arrive(&full[k2 % C::STAGES]);
  } else {
    // Epilogue: the output row of each accumulator row is found while the
    // tile's main loop runs; the accumulator is released as soon as it has
    // been read into registers.
    const int qd = warp & 3;
    const int r = qd * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(qd * 32) << 16;
    int it = 0;
    for (int v = vb; v < ve; ++v, ++it) {
      const int4 q = q_entry(ga, v, n_routed);
      const bool valid = r < q.w;
      uint16_t* dst = nullptr;
      if (valid) {
        if (q.x < 0) {
          dst = ga.Qs + static_cast<size_t>(q.z + r) * ga.dh;
        } else if (ga.expert_major) {
          dst = ga.Qv + static_cast<size_t>(q.z + r) * ga.dh;
        } else {
          const int b = q.y, t = ga.tok[q.z + r];
          const int g = q.x / ga.M, j = q.x % ga.M;
          int s = 0;
          if (ga.k > 1) {
            const int32_t* ip = ga.idx + ((static_cast<size_t>(b) * ga.T + t) * ga.G + g) * ga.k;
            for (int s2 = 0; s2 < ga.k; ++s2)
              if (ip[s2] == j) s = s2;
          }
          dst = ga.Qv + (((static_cast<size_t>(b) * ga.G + g) * ga.k + s) * ga.T + t) * ga.dh;
        }
      }
      const int a = it & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[a], (it >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      uint32_t vals[BN / 32][32];
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) tmem_ld32(tmem + lane_off + a * BN + cc * 32, vals[cc]);
      tc_fence_before();
      mbar_arrive(&acc_empty[a]);
      if (valid) {
#pragma unroll
        for (int cc = 0; cc < BN / 32; ++cc) store32_bf16(dst + cc * 32, vals[cc]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (*abort_flag) {
      // Let every issued UMMA finish before the columns are released.
      volatile int none = 0;
      mbar_wait(drain, 0, &none, 500000000ull);
    }
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int BN, bool GATHER>
int launch(const CUtensorMap& A, const CUtensorMap& B0, const CUtensorMap& B1, const CUtensorMap& B2,
           const CUtensorMap& B3, const Epi& e0, const Epi& e1, const Epi& e2, const Epi& e3, const Gather& g,
           int K, dim3 grid, void* stream) {
  using C = GemmCfg<BN>;
  const int e = ensure_smem<gemm_kernel<BN, GATHER>>(static_cast<int>(C::SMEM));
  if (e != cudaSuccess) return e;
  return launch_pdl(gemm_kernel<BN, GATHER>, grid, dim3(192), C::SMEM, stream, A, B0, B1, B2, B3, e0, e1, e2, e3,
                    g, K);
}

template <int BN, bool GATHER>
int launch(const CUtensorMap& A, const CUtensorMap& B0, const CUtensorMap& B1, const Epi& e0,
           const Epi& e1, const Gather& g, int K, dim3 grid, void* stream) {
  return launch<BN, GATHER>(A, B0, B1, B1, B1, e0, e1, e1, e1, g, K, grid, stream);
}

template <int DH>
int launch_q(const CUtensorMap& W, const CUtensorMap& Ws, const Gather& g, int n_shared, dim3 grid,
             void* stream) {
  using C = QCfg<DH>;
  constexpr int GW = kQGatherWarps;
  const int e = ensure_smem<qgemm_kernel<DH, GW>>(static_cast<int>(C::SMEM));
  if (e != cudaSuccess) return e;
  return launch_pdl(qgemm_kernel<DH, GW>, grid, dim3(q_threads(GW)), C::SMEM, stream, W, Ws, g, n_shared);
}

// Dense GEMM with a head-split epilogue; chooses the tile width.
int dense_gemm(const uint16_t* A, int rows, int K, const uint16_t* W0, const uint16_t* W1, int N,
               const Epi& e0, const Epi& e1, int nz, void* stream) {
  int BN = 256;
  const long long mt = (rows + BM - 1) / BM;
  if (N % 256 != 0 || mt * (N / 256) * nz < 148) BN = 128;
  // Fewer 128-wide tiles than SMs: 64-wide ones (two CTAs per SM fit).
  if (N % 128 != 0 || mt * (N / 128) * nz < 148) BN = 64;
  if (N % 64 != 0) BN = 32;
  if (N % 32 != 0) return cudaErrorInvalidValue;
  CUtensorMap ta, tb0, tb1;
  const int batom = BN >= 64 ? 64 : BN;
  if (!make_tmap_bf16_2d(&ta, A, K, rows, K, 64, BM)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tb0, W0, N, K, N, batom, BK)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tb1, W1 ? W1 : W0, N, K, N, batom, BK)) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(mt), static_cast<unsigned>(N / BN), nz);
  Gather g{};
  switch (BN) {
    case 256: return launch<256, false>(ta, tb0, tb1, e0, e1, g, K, grid, stream);
    case 128: return launch<128, false>(ta, tb0, tb1, e0, e1, g, K, grid, stream);
    case 64: return launch<64, false>(ta, tb0, tb1, e0, e1, g, K, grid, stream);
    default: return launch<32, false>(ta, tb0, tb1, e0, e1, g, K, grid, stream);
  }
}

Epi head_split(uint16_t* out, int T, int H, int dh, int R) {
  Epi e;
  e.out = out;
  e.T = T;
  e.hd = dh;
  e.sb = static_cast<long long>(H) * T * dh;
  e.sh = static_cast<long long>(T) * dh;
  e.st = dh;
  e.rows = R;
  e.cols = H * dh;
  return e;
}

}  // namespace gemm_impl
using namespace gemm_impl;

// C[M, N] (fp32, row stride ldc) = A[M, K] B[K, N]: A bf16 with K contiguous
// (row stride lda), B bf16 with N contiguous (row stride ldb). Rows, columns
// and K blocks past the ends read as zero (TMA fill) and are not stored.
int gemm_f32out(const uint16_t* A, long long lda, int M, int K, const uint16_t* B, long long ldb, int N,
                float* C, long long ldc, void* stream) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  if (K <= 0 || ((lda | ldb) & 7) != 0 || ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B)) & 15u))
    return cudaErrorInvalidValue;
  const long long mt = (M + BM - 1) / BM;
  int BN = 128;
  if (N <= 32) BN = 32;
  else if (N <= 64 || mt * ((N + 127) / 128) < 148) BN = 64;
  const long long nt = (N + BN - 1) / BN;
  if (mt > 0x7fffffffll || nt > 65535) return cudaErrorInvalidConfiguration;
  // B's inner extent is rounded up to whole boxes: the caller's rows are at
  // least that long (columns past N only reach C columns that are not stored).
  const int batom = BN >= 64 ? 64 : BN;
  const long long nb = (N + batom - 1) / batom * batom;
  if (nb > ldb) return cudaErrorInvalidValue;
  CUtensorMap ta, tb;
  if (!make_tmap_bf16_2d(&ta, A, K, M, lda, 64, BM)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tb, B, nb, K, ldb, batom, BK)) return cudaErrorInvalidValue;
  Epi e;
  e.out = nullptr;
  e.T = M;
  e.hd = N;
  e.sb = e.sh = e.st = 0;
  e.rows = M;
  e.cols = N;
  e.outf = C;
  e.ldf = ldc;
  e.fvec = ((ldc & 3) == 0 && (reinterpret_cast<uintptr_t>(C) & 15u) == 0) ? 1 : 0;
  const dim3 grid(static_cast<unsigned>(mt), static_cast<unsigned>(nt), 1);
  Gather g{};
  switch (BN) {
    case 128: return launch<128, false>(ta, tb, tb, e, e, g, K, grid, stream);
    case 64: return launch<64, false>(ta, tb, tb, e, e, g, K, grid, stream);
    default: return launch<32, false>(ta, tb, tb, e, e, g, K, grid, stream);
  }
}

int gemm_kv(const gqe_config& c, const uint16_t* x, const uint16_t* W_k, const uint16_t* W_v,
            uint16_t* K, uint16_t* V, void* stream) {
  const int R = c.B * c.T;
  const Epi ek = head_split(K, c.T, c.G, c.d_head, R);
  const Epi ev = head_split(V, c.T, c.G, c.d_head, R);
  return dense_gemm(x, R, c.d_model, W_k, W_v, c.G * c.d_head, ek, ev, 2, stream);
}

int gemm_kv_at(const gqe_config& c1, const uint16_t* x, const uint16_t* W_k, const uint16_t* W_v,
               uint16_t* Kc, uint16_t* Vc, int cap, int pos, void* stream) {
  // Row b (one token of sequence b) -> cache[b][g][pos][:].
  const int B = c1.B;
  auto at = [&](uint16_t* cache) {
    Epi e;
    e.out = cache + static_cast<size_t>(pos) * c1.d_head;
    e.T = 1;
    e.hd = c1.d_head;
    e.sb = static_cast<long long>(c1.G) * cap * c1.d_head;
    e.sh = static_cast<long long>(cap) * c1.d_head;
    e.st = c1.d_head;
    e.rows = B;
    e.cols = c1.G * c1.d_head;
    return e;
  };
  return dense_gemm(x, B, c1.d_model, W_k, W_v, c1.G * c1.d_head, at(Kc), at(Vc), 2, stream);
}

int gemm_q_dense(const gqe_config& c, const uint16_t* x, const uint16_t* W_q, uint16_t* Q,
                 void* stream) {
  const int R = c.B * c.T;
  const int N = c.G * c.M;
  const Epi e = head_split(Q, c.T, N, c.d_head, R);
  return dense_gemm(x, R, c.d_model, W_q, nullptr, N * c.d_head, e, e, 1, stream);
}

int gemm_q_all_routed(const gqe_config& c, const uint16_t* x, const uint16_t* W_q, const int32_t* idx,
                      uint16_t* Qv, void* stream) {
  const int R = c.B * c.T;
  const int N = c.G * c.M;
  Epi e = head_split(Qv, c.T, N, c.d_head, R);
  e.sel = idx;
  e.G = c.G;
  e.M = c.M;
  e.k = c.k;
  return dense_gemm(x, R, c.d_model, W_q, nullptr, N * c.d_head, e, e, 1, stream);
}

int gemm_kvq(const gqe_config& c, const uint16_t* x, const uint16_t* W_k, const uint16_t* W_v,
             const uint16_t* W_q, const int32_t* idx, uint16_t* K, uint16_t* V, uint16_t* Q, void* stream) {
  const int R = c.B * c.T, dh = c.d_head;
  const int Nkv = c.G * dh, Nq = c.G * c.M * dh;
  if (Nq != 2 * Nkv || Nkv % 64 != 0) return cudaErrorInvalidValue;
  const int BN = Nkv % 128 == 0 ? 128 : 64;
  const long long mt = (R + BM - 1) / BM;
  CUtensorMap ta, tk, tv, tq0, tq1;
  if (!make_tmap_bf16_2d(&ta, x, c.d_model, R, c.d_model, 64, BM) ||
      !make_tmap_bf16_2d(&tk, W_k, Nkv, c.d_model, Nkv, 64, BK) ||
      !make_tmap_bf16_2d(&tv, W_v, Nkv, c.d_model, Nkv, 64, BK) ||
      !make_tmap_bf16_2d(&tq0, W_q, Nkv, c.d_model, Nq, 64, BK) ||
      !make_tmap_bf16_2d(&tq1, W_q + Nkv, Nkv, c.d_model, Nq, 64, BK))
    return cudaErrorInvalidValue;
  Epi ek = head_split(K, c.T, c.G, dh, R);
  Epi ev = head_split(V, c.T, c.G, dh, R);
  Epi eq0 = head_split(Q, c.T, c.G * c.M, dh, R);
  eq0.cols = Nkv;
  eq0.sel = idx;  // null: every expert's queries stored ([B][G*M][T][dh])
  eq0.G = c.G;
  eq0.M = c.M;
  eq0.k = c.k;
  Epi eq1 = eq0;
  eq1.h0 = c.G;  // the second half of the heads' columns
  if (idx != nullptr) {  // the main loop overlaps the router; the epilogues wait for it
    ek.late_wait = ev.late_wait = eq0.late_wait = eq1.late_wait = 1;
  }
  const dim3 grid(static_cast<unsigned>(mt), static_cast<unsigned>(Nkv / BN), 4);
  Gather g{};
  if (BN == 128) return launch<128, false>(ta, tk, tv, tq0, tq1, ek, ev, eq0, eq1, g, c.d_model, grid, stream);
  return launch<64, false>(ta, tk, tv, tq0, tq1, ek, ev, eq0, eq1, g, c.d_model, grid, stream);
}

int gemm_rowmajor(const uint16_t* A, int rows, int K, const uint16_t* W, int N, uint16_t* out,
                  void* stream) {
  Epi e;
  e.out = out;
  e.T = rows;
  e.hd = N;
  e.sb = 0;
  e.sh = 0;
  e.st = N;
  e.rows = rows;
  e.cols = N;
  return dense_gemm(A, rows, K, W, nullptr, N, e, e, 1, stream);
}

int gemm_output(const gqe_config& c, uint16_t* slots, const float* omega, const uint16_t* W_o,
                uint16_t* y, void* stream) {
  const int R = c.B * c.T;
  const int gk = c.G * c.k;
  const int K = n_slots(c) * c.d_head;
  if (!has_weighted_slot(c)) {  // ablation constructions: the kG routed slots only
    if (c.flags & GQE_FLAG_OUT_WEIGHTED_CONCAT) {
      const int e = launch_scale_slots(c, slots, omega, stream);
      if (e != cudaSuccess) return e;
    }
    return gemm_rowmajor(slots, R, K, W_o, c.d_model, y, stream);
  }
  if (c.d_head != BK) {  // the weighted slot is not one K block: separate kernel
    const int e = launch_weighted_slot(c, slots, omega, stream);
    if (e != cudaSuccess) return e;
    return gemm_rowmajor(slots, R, K, W_o, c.d_model, y, stream);
  }
  Epi e;
  e.out = y;
  e.T = R;
  e.hd = c.d_model;
  e.sb = 0;
  e.sh = 0;
  e.st = c.d_model;
  e.rows = R;
  e.cols = c.d_model;
  e.kb_w = n_slots(c) - 1;  // the weighted slot is the last one
  e.gk = gk;
  e.omega = omega;
  e.wslots = slots;
  e.lda = K;
  return dense_gemm(slots, R, K, W_o, nullptr, c.d_model, e, e, 1, stream);
}

int gemm_q_routed(const gqe_config& c, const uint16_t* x, const uint16_t* W_q, const uint16_t* W_qs,
                  const int32_t* idx, const int32_t* tok, const void* qtiles,
                  const int32_t* n_qtiles, int max_qtiles, uint16_t* Qv, uint16_t* Qs,
                  bool expert_major, void* stream) {
  const int N = c.G * c.M;
  const int dh = c.d_head;
  CUtensorMap tb, tbs;
  if (!make_tmap_bf16_2d(&tb, W_q, static_cast<uint64_t>(N) * dh, c.d_model,
                         static_cast<uint64_t>(N) * dh, dh, BK))
    return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tbs, W_qs, dh, c.d_model, dh, dh, BK)) return cudaErrorInvalidValue;
  Gather g;
  g.x = x;
  g.tok = tok;
  g.qtiles = static_cast<const int4*>(qtiles);
  g.n_qtiles = n_qtiles;
  g.idx = idx;
  g.Qv = Qv;
  g.Qs = Qs;
  g.max_qtiles = max_qtiles;
  g.d = c.d_model;
  g.T = c.T;
  g.G = c.G;
  g.M = c.M;
  g.k = c.k;
  g.B = c.B;
  g.dh = dh;
  g.expert_major = expert_major ? 1 : 0;
  const long long R = static_cast<long long>(c.B) * c.T;
  const long long shared_tiles = Qs != nullptr ? (R + BM - 1) / BM : 0;
  const long long tiles = max_qtiles + shared_tiles;  // upper bound; the table holds the count
  if (tiles == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (static_cast<long long>(c.d_model) * dh * 2 <= QCfg<64>::W_MAX && tiles >= 2ll * sms) {
    // Several tiles per SM and the expert's weights fit in shared memory:
    // one CTA per SM with the weights resident. (With about one tile per SM
    // the resident load only delays the first UMMA: measured 18.5 against
    // 17.1 us at T = 2048.)
    const dim3 grid(static_cast<unsigned>(sms));
    if (dh == 64) return launch_q<64>(tb, tbs, g, static_cast<int>(shared_tiles), grid, stream);
    return launch_q<32>(tb, tbs, g, static_cast<int>(shared_tiles), grid, stream);
  }
  // Otherwise one CTA per tile, the weights streamed with A.
  Epi e{};
  const dim3 grid(static_cast<unsigned>(tiles), 1, 1);
  if (dh == 64) return launch<64, true>(tb, tb, tbs, e, e, g, c.d_model, grid, stream);
  return launch<32, true>(tb, tb, tbs, e, e, g, c.d_model, grid, stream);
}

int gemm_q_shared(const gqe_config& c, const uint16_t* x, const uint16_t* W_qs, uint16_t* Qs,
                  void* stream) {
  const int R = c.B * c.T;
  const Epi e = head_split(Qs, c.T, 1, c.d_head, R);
  return dense_gemm(x, R, c.d_model, W_qs, nullptr, c.d_head, e, e, 1, stream);
}

}  // namespace gqe
