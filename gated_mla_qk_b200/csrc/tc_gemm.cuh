// bf16 GEMM on the 5th-generation tensor cores for the low-rank projections
// of the layer ("Kimi K3 · Gated MLA · OpenModelAtlas", "All 20 steps":
// c^Q = x W_DQ, q = c^Q W_UQ, [c^KV k^S] = x W_DKV, [k^C v] = c^KV W_UKV).
//
// C[M][N] = A[M][K] B[K][N], all row-major; fp32 accumulation in TMEM.
// Persistent: one CTA per SM walks the 128 x 256 output tiles (tile index
// advancing by the grid size).  A tiles (128 x 64, K-major) and B tiles
// (64 x 256, N contiguous = MN-major) stream through a 4-stage TMA ring that
// runs on across tile boundaries; one thread issues tcgen05.mma (M=128,
// N=256, K=16) into one of two 256-column TMEM accumulators, so the four
// epilogue warps read tile j back (tcgen05.ld) while the MMAs of tile j+1
// run.  Each epilogue warp stages 64-column chunks of its 32 rows in padded
// shared memory and stores them as whole 128-byte lines.  The epilogue either
// writes C row-major or, for the key/value up-projection, splits each
// 256-column tile (= one head) into K^C and V.
#pragma once

#include "sm100.cuh"

namespace gmla {
namespace tc_gemm {

using namespace sm100;

constexpr int BM = 128, BN = 256, BK = 64, NSTAGE = 4;
constexpr uint32_t A_BYTES = BM * BK * 2;                 // 16 KB
constexpr uint32_t BSUB = BK * 128;                       // one 64 (k) x 64 (n) sub-tile, 8 KB
constexpr uint32_t B_BYTES = 4 * BSUB;                    // 32 KB
constexpr uint32_t STAGE = A_BYTES + B_BYTES;             // 48 KB
constexpr uint32_t OFF_EPI = NSTAGE * STAGE;             // epilogue staging: 4 warps x [32 rows][64 cols + 8] bf16
constexpr int EPI_LD = 72;                                // padded row (144 B): conflict-free 16-byte stores
constexpr uint32_t EPI_WARP = 32 * EPI_LD * 2;            // 4.5 KB
constexpr uint32_t OFF_BAR = OFF_EPI + 4 * EPI_WARP;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 128 + 1024;

enum Bar { FULL = 0, EMPTY = NSTAGE, ACCF = 2 * NSTAGE, ACCE = ACCF + 2, DRAIN = ACCE + 2, NBAR = DRAIN + 1 };

struct Params {
  int M, N, K;
  __nv_bfloat16* C;          // [M][N] (mode 0)
  __nv_bfloat16* KC;         // [M][H][128] (mode 1)
  __nv_bfloat16* V;          // [M][H][128] (mode 1)
  int H;
  int mode;                  // 0: plain, 1: per-head split of [K^C_h | V_h] (N = H * 256)
  int N2;                    // pair kernel, mode 0: a second product A B2 [M][N2] in the same launch (0: none)
};

__global__ void __launch_bounds__(192, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, Params p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  volatile int* abort = &abort_flag;
  auto bar = [&](int i) { return sbase + OFF_BAR + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles_n = (p.N + BN - 1) / BN;
  const int n_tiles = n_tiles_n * ((p.M + BM - 1) / BM);
  const int nk = (p.K + BK - 1) / BK;

  if (threadIdx.x == 0) abort_flag = device_error_pending() ? 1 : 0;
  __syncthreads();
  if (abort_flag) return;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NBAR; ++i) mbar_init(bar(i), (i == ACCE || i == ACCE + 1) ? 128 : 1);
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(smem_u32(&tmem_slot), 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA); tma_prefetch_desc(&tmB);
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x) {
        const int tn = tile % n_tiles_n, tm = tile / n_tiles_n;
        for (int k = 0; k < nk; ++k, ++it) {
          const uint32_t s = it % NSTAGE, ph = (it / NSTAGE) & 1;
          if (!mbar_wait(bar(EMPTY + s), ph ^ 1u, abort)) { ok = false; break; }
          const uint32_t st = sbase + s * STAGE;
          mbar_arrive_expect_tx(bar(FULL + s), STAGE);
          tma_load_2d(st, &tmA, bar(FULL + s), k * BK, tm * BM);
          for (int c = 0; c < 4; ++c) tma_load_2d(st + A_BYTES + c * BSUB, &tmB, bar(FULL + s), tn * BN + 64 * c, k * BK);
        }
      }
      for (int q = (it > NSTAGE ? it - NSTAGE : 0); q < it; ++q)
        mbar_wait_drain(bar(FULL + q % NSTAGE), (q / NSTAGE) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, false, true);   // A K-major, B MN-major
      int it = 0, j = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x, ++j) {
        const int acc = j & 1;
        // Accumulator acc was last used by tile j-2: its epilogue must be done.
        if (j >= 2 && !(ok = mbar_wait(bar(ACCE + acc), ((uint32_t)(j >> 1) & 1u) ^ 1u, abort))) break;
        tc_fence_after();
        const uint32_t d = tmem + 256u * (uint32_t)acc;
        for (int k = 0; k < nk; ++k, ++it) {
          const uint32_t s = it % NSTAGE, ph = (it / NSTAGE) & 1;
          if (!(ok = mbar_wait(bar(FULL + s), ph, abort))) break;
          tc_fence_after();
          const uint32_t st = sbase + s * STAGE;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_ss(d, sdesc_sw128(st + kk * 32, 16, 1024), sdesc_sw128(st + A_BYTES + kk * 2048, BSUB, 1024), idesc,
                   (k > 0 || kk > 0));
          mma_commit(bar(EMPTY + s));
        }
        if (!ok) break;
        mma_commit(bar(ACCF + acc));
      }
      mma_commit(bar(DRAIN));
      mbar_wait_drain(bar(DRAIN), 0);
    }
    __syncwarp();
  } else {
    // epilogue warps 2..5: TMEM lanes 32 * (warp % 4) .. + 31
    const int sub = warp & 3;
    int j = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++j) {
      const int acc = j & 1;
      const bool w = mbar_wait(bar(ACCF + acc), (uint32_t)(j >> 1) & 1u, abort);
      if (!__all_sync(0xffffffffu, w)) break;
      tc_fence_after();
      const int tn = tile % n_tiles_n, tm = tile / n_tiles_n;
      const uint32_t taddr = tmem + ((uint32_t)(sub * 32) << 16) + 256u * (uint32_t)acc;
      // 64 columns at a time: thread `lane` stages row 32*sub + lane of the
      // chunk, then the warp writes the chunk out row by row, 8 lanes per
      // row (a full 128-byte line), 4 rows per store instruction.
      __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(smem_raw + (sbase - sraw) + OFF_EPI + sub * EPI_WARP);
#pragma unroll 1
      for (int q = 0; q < BN / 64; ++q) {
        float v[64];
        tmem_ld32(taddr + 64u * q, *reinterpret_cast<float(*)[32]>(&v[0]));
        tmem_ld32(taddr + 64u * q + 32u, *reinterpret_cast<float(*)[32]>(&v[32]));
        tmem_wait_ld_dep(*reinterpret_cast<float(*)[32]>(&v[0]));
        tmem_wait_ld_dep(*reinterpret_cast<float(*)[32]>(&v[32]));
        __syncwarp();
        uint4* srow = reinterpret_cast<uint4*>(stg + lane * EPI_LD);
#pragma unroll
        for (int c = 0; c < 8; ++c)
          srow[c] = make_uint4(pack_bf16x2(v[8 * c], v[8 * c + 1]), pack_bf16x2(v[8 * c + 2], v[8 * c + 3]),
                               pack_bf16x2(v[8 * c + 4], v[8 * c + 5]), pack_bf16x2(v[8 * c + 6], v[8 * c + 7]));
        __syncwarp();
        const int col = tn * BN + 64 * q + 8 * (lane & 7);      // this lane's 8 columns
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = 4 * i + (lane >> 3);
          const int row = tm * BM + sub * 32 + r;
          if (row >= p.M || col >= p.N) continue;
          const uint4 val = reinterpret_cast<const uint4*>(stg + r * EPI_LD)[lane & 7];
          __nv_bfloat16* dst;
          if (p.mode == 1) {
            const int h = col / 256, jj = col % 256;
            dst = (jj < 128) ? p.KC + ((size_t)row * p.H + h) * 128 + jj : p.V + ((size_t)row * p.H + h) * 128 + (jj - 128);
          } else {
            dst = p.C + (size_t)row * p.N + col;
          }
          if (col + 8 <= p.N) {
            *reinterpret_cast<uint4*>(dst) = val;
          } else {
            const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&val);
            for (int k = 0; col + k < p.N; ++k) dst[k] = e[k];
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(ACCE + acc));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ===========================================================================
// The same GEMM on CTA pairs (tcgen05 .cta_group::2): each pair of SMs owns a
// 256 x 256 output tile.  SM r of the pair loads rows [128 r, 128 r + 128) of
// the A tile and columns [128 r, 128 r + 128) of the B tile; the even CTA
// issues M = 256, N = 256, K = 16 MMAs that read A rows from both SMs and B
// columns from both halves, and each SM's TMEM receives its own 128 rows of
// all 256 columns.  Per SM and per 64-deep k-block that is 16 KB of A and
// 16 KB of B from L2 instead of 16 + 32 KB, for the same tensor work.
//   warp 0: TMA producer (both CTAs; the even CTA's full barrier counts both)
//   warp 1: TMEM allocation (both CTAs), MMA issue (even CTA)
//   warps 2-5: epilogue (both CTAs): TMEM -> bf16 in swizzled shared memory
//              -> TMA tile stores, the accumulator released after its last
//              TMEM read, before the stores complete
// Every wait is bounded; a pair has no early exit, so that both CTAs always
// reach the cluster barriers and the paired TMEM allocation and release.
// ===========================================================================
constexpr int PAIR_BM = 256, PAIR_NSTAGE = 6;              // pair tile rows; ring stages
constexpr uint32_t PAIR_A_BYTES = 128 * BK * 2;             // this SM's 128 rows: 16 KB
constexpr uint32_t PAIR_B_BYTES = 2 * BSUB;                 // this SM's 128 columns: 16 KB
constexpr uint32_t PAIR_STAGE = PAIR_A_BYTES + PAIR_B_BYTES;  // 32 KB
constexpr uint32_t PAIR_EPI_BUF = 32 * 128;                  // [32 rows][64 cols] bf16, 128-byte swizzle: 4 KB
constexpr uint32_t PAIR_OFF_EPI = PAIR_NSTAGE * PAIR_STAGE;  // 4 epilogue warps x 2 staging buffers
constexpr uint32_t PAIR_OFF_BAR = PAIR_OFF_EPI + 8 * PAIR_EPI_BUF;
constexpr uint32_t PAIR_SMEM_BYTES = PAIR_OFF_BAR + 256 + 1024;
static_assert(PAIR_SMEM_BYTES + 64 <= 232448, "pair GEMM shared memory exceeds the per-block limit");
enum PairBar { PFULL = 0, PEMPTY = PAIR_NSTAGE, PACCF = 2 * PAIR_NSTAGE, PACCE = PACCF + 2, PDRAIN = PACCE + 2,
               PNBAR = PDRAIN + 1 };

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmC0,
                 const __grid_constant__ CUtensorMap tmC1, Params p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  volatile int* abort = &abort_flag;
  auto bar = [&](int i) { return sbase + PAIR_OFF_BAR + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();                 // 0: issues the pair's MMAs
  const int n_pairs = (int)(gridDim.x / 2), pair_id = (int)(blockIdx.x / 2);
  // Column tiles of the first product, then (N2 > 0) of the second, which
  // shares A: one walk over both, so A is read once and the two products
  // share their last wave.
  const int n_tiles_n1 = (p.N + BN - 1) / BN;
  const int n_tiles_n = n_tiles_n1 + (p.N2 + BN - 1) / BN;
  const int n_tiles = n_tiles_n * ((p.M + PAIR_BM - 1) / PAIR_BM);
  const int nk = (p.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int i = 0; i < PNBAR; ++i) mbar_init(bar(i), (i == PACCE || i == PACCE + 1) ? 256 : 1);
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc_pair(smem_u32(&tmem_slot), 512); tmem_relinquish_pair(); }
  tc_fence_before();
  cluster_sync();                      // both CTAs' barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA); tma_prefetch_desc(&tmB);
      if (p.N2 > 0) tma_prefetch_desc(&tmB2);
      int it = 0;
      bool ok = true;
      for (int tile = pair_id; ok && tile < n_tiles; tile += n_pairs) {
        const int tn = tile % n_tiles_n, tm = tile / n_tiles_n;
        const bool second = tn >= n_tiles_n1;
        const CUtensorMap* mB = second ? &tmB2 : &tmB;
        const int bcol = (second ? tn - n_tiles_n1 : tn) * BN + 128 * (int)rank;
        for (int k = 0; k < nk; ++k, ++it) {
          const uint32_t s = it % PAIR_NSTAGE, ph = (it / PAIR_NSTAGE) & 1;
          if (!mbar_wait(bar(PEMPTY + s), ph ^ 1u, abort)) { ok = false; break; }
          const uint32_t st = sbase + s * PAIR_STAGE;
          const uint32_t full0 = map_to_cta(bar(PFULL + s), 0);          // the even CTA's full barrier
          if (rank == 0) mbar_arrive_expect_tx(bar(PFULL + s), 2 * PAIR_STAGE);
          tma_load_2d_pair(st, &tmA, full0, k * BK, tm * PAIR_BM + 128 * (int)rank);
          for (int c = 0; c < 2; ++c)
            tma_load_2d_pair(st + PAIR_A_BYTES + c * BSUB, mB, full0, bcol + 64 * c, k * BK);
        }
      }
      // Never leave with copies in flight into this CTA's shared memory: a
      // stage's copies have landed once the MMAs that read it have completed.
      for (int q = (it > PAIR_NSTAGE ? it - PAIR_NSTAGE : 0); q < it; ++q)
        mbar_wait_drain(bar(PEMPTY + q % PAIR_NSTAGE), (q / PAIR_NSTAGE) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(PAIR_BM, BN, false, true);   // A K-major, B MN-major
      int it = 0, j = 0;
      bool ok = true;
      for (int tile = pair_id; ok && tile < n_tiles; tile += n_pairs, ++j) {
        const int acc = j & 1;
        // Accumulator acc was last used by tile j-2: both epilogues must be done with it.
        if (j >= 2 && !(ok = mbar_wait(bar(PACCE + acc), ((uint32_t)(j >> 1) & 1u) ^ 1u, abort))) break;
        tc_fence_after();
        const uint32_t d = tmem + 256u * (uint32_t)acc;
        for (int k = 0; k < nk; ++k, ++it) {
          const uint32_t s = it % PAIR_NSTAGE, ph = (it / PAIR_NSTAGE) & 1;
          if (!(ok = mbar_wait(bar(PFULL + s), ph, abort))) break;
          tc_fence_after();
          const uint32_t st = sbase + s * PAIR_STAGE;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_ss_pair(d, sdesc_sw128(st + kk * 32, 16, 1024), sdesc_sw128(st + PAIR_A_BYTES + kk * 2048, BSUB, 1024), idesc,
                        (k > 0 || kk > 0));
          mma_commit_pair(bar(PEMPTY + s), 0x3);          // both CTAs may refill stage s
        }
        if (!ok) break;
        mma_commit_pair(bar(PACCF + acc), 0x3);           // both CTAs' epilogues may read accumulator acc
      }
      mma_commit_pair(bar(PDRAIN), 0x1);
      mbar_wait_drain(bar(PDRAIN), 0);
    }
    __syncwarp();
  } else {
    // epilogue warps 2..5: TMEM lanes 32 * (warp % 4) .. + 31 = this SM's rows.
    // Each 64-column chunk is rounded to bf16 into one of the warp's two
    // swizzled staging buffers and written by one TMA tile store (elements
    // past M or N are not written).  The accumulator is released as soon as
    // its last chunk has been read from TMEM; the stores run on behind it.
    const int sub = warp & 3;
    const uint32_t stg0 = sbase + PAIR_OFF_EPI + (uint32_t)sub * 2u * PAIR_EPI_BUF;
    if (lane == 0) { tma_prefetch_desc(&tmC0); tma_prefetch_desc(&tmC1); }
    int j = 0, chunk = 0;
    int last_buf = -1;                             // lane 0: staging buffer of the latest committed store
    for (int tile = pair_id; tile < n_tiles; tile += n_pairs, ++j) {
      const int acc = j & 1;
      const bool w = mbar_wait(bar(PACCF + acc), (uint32_t)(j >> 1) & 1u, abort);
      if (!__all_sync(0xffffffffu, w)) break;
      tc_fence_after();
      const int tn = tile % n_tiles_n, tm = tile / n_tiles_n;
      const uint32_t taddr = tmem + ((uint32_t)(sub * 32) << 16) + 256u * (uint32_t)acc;
      const int row0 = tm * PAIR_BM + 128 * (int)rank + sub * 32;
#pragma unroll 1
      for (int q = 0; q < BN / 64; ++q, ++chunk) {
        float v[64];
        tmem_ld32(taddr + 64u * q, *reinterpret_cast<float(*)[32]>(&v[0]));
        tmem_ld32(taddr + 64u * q + 32u, *reinterpret_cast<float(*)[32]>(&v[32]));
        tmem_wait_ld_dep(*reinterpret_cast<float(*)[32]>(&v[0]));
        tmem_wait_ld_dep(*reinterpret_cast<float(*)[32]>(&v[32]));
        if (q == BN / 64 - 1) {
          // Accumulator acc is free once both SMs' epilogues have read it (256 arrivals on the even CTA).
          tc_fence_before();
          if (rank == 0) mbar_arrive(bar(PACCE + acc));
          else mbar_arrive_cluster(map_to_cta(bar(PACCE + acc), 0));
        }
        const int b = chunk & 1;
        const uint32_t buf = stg0 + (uint32_t)b * PAIR_EPI_BUF;
        // Every store but the latest has finished reading its buffer; the
        // latest must have too if it read this one (chunks past N store nothing).
        if (lane == 0) {
          if (last_buf == b) bulk_wait_group_read<0>();
          else bulk_wait_group_read<1>();
        }
        __syncwarp();
        const uint32_t srow = buf + (uint32_t)lane * 128u;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(srow + ((uint32_t)(c ^ (lane & 7)) << 4), pack_bf16x2(v[8 * c], v[8 * c + 1]),
                       pack_bf16x2(v[8 * c + 2], v[8 * c + 3]), pack_bf16x2(v[8 * c + 4], v[8 * c + 5]),
                       pack_bf16x2(v[8 * c + 6], v[8 * c + 7]));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          // mode 1: chunks 0-1 of head tn's tile are K^C_tn, chunks 2-3 are
          // V_tn (tmC0, tmC1).  mode 0: C (tmC0), or the second product's C2 (tmC1).
          const bool second = tn >= n_tiles_n1;
          const CUtensorMap* m = ((p.mode == 1 && q >= 2) || second) ? &tmC1 : &tmC0;
          const int x = p.mode == 1 ? tn * 128 + 64 * (q & 1) : (second ? tn - n_tiles_n1 : tn) * BN + 64 * q;
          if (row0 < p.M && (p.mode == 1 || x < (second ? p.N2 : p.N))) {
            tma_store_2d(m, buf, x, row0);
            bulk_commit_group();
            last_buf = b;
          }
        }
      }
    }
    if (lane == 0) bulk_wait_group_all();          // every store has left shared memory and landed
    __syncwarp();
  }
  tc_fence_before();
  cluster_sync();                      // both CTAs done with the accumulators and the ring
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, 512);
}

}  // namespace tc_gemm
}  // namespace gmla
