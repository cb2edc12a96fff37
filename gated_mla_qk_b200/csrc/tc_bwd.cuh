// Backward of the causal gated MLA attention on the 5th-generation tensor
// cores (tcgen05 + TMEM + TMA), for Kimi K3's head widths (d_c = 128,
// d_s = 64, d_v = 128) in bf16.
//
// Gradients ("Kimi K3 · Gated MLA · OpenModelAtlas", "All 20 steps", taken
// back through each step; the row pass that forms dO~ = dO sigmoid(g) and
// D_t = sum_c dO o runs before these kernels):
//   P  = exp(S scale - lse),  S = Q_h K_h^T,  K_h = [K^C_h | k^S]
//   dP = dO~ V_h^T,  dS = P (dP - D)
//   dV_h = P^T dO~,  dK_h = scale dS^T Q_h,  dQ_h = scale dS K_h
// and k^S, shared by every head, gets the sum over heads of dK_h's last 64
// columns (fp32 atomic adds into a buffer the caller zeroes).
//
// Two kernels, each recomputing P from the forward's row log-sum-exp, so
// neither needs atomics apart from the cross-head k^S sum:
//   dkdv_kernel: one CTA per (128-key tile, head, batch); walks the 64-query
//     tiles at or after its keys.  Keys sit on the MMA's M side:
//       S^T  = K Q_i^T        (SS, M=128 N=64 K=192)     TMEM, double buffer
//       dP^T = V dO~_i^T      (SS, M=128 N=64 K=128)     TMEM
//       dV  += P^T dO~_i      (TS: P^T written back to TMEM over S^T)
//       dK  += dS^T Q_i       (SS: dS^T written to a swizzled shared tile)
//   dq_kernel: one CTA per (128-query tile, head, batch); walks the 64-key
//     tiles at or before its rows:
//       S = Q K_j^T, dP = dO~ V_j^T (SS, M=128 N=64), dQ += dS K_j (TS: dS
//       written back to TMEM over dP).
// Warp roles as in the forward: warps 0-3 compute P / dS (thread r owns
// TMEM lane r) and run the epilogue, warp 4 is the TMA producer, warp 5
// allocates TMEM and issues the MMAs.  Every wait is bounded (mbar_wait).
#pragma once

#include "sm100.cuh"

namespace gmla {
namespace tc_bwd {

using namespace sm100;

constexpr uint32_t SUB128 = 128 * 128;   // [128 rows x 64] bf16 sub-tile, 128B-swizzled
constexpr uint32_t SUB64 = 64 * 128;     // [64 rows x 64] bf16 sub-tile
constexpr int NS = 3;                    // ring slots
constexpr uint32_t SLOT = 5 * SUB64;     // 64 rows of a 192-wide and a 128-wide tensor: 40 KB

struct Params {
  int B, T, H;
  const float* lse;   // [B][T][H], natural log of the scaled logits' row sum
  const float* D;     // [B][T][H]
  float* dQ;          // [B][T][H][192]
  float* dKC;         // [B][T][H][128]
  float* dkS;         // [B][T][64]
  float* dV;          // [B][T][H][128]
  float scale;        // 1/sqrt(192)
  float scale_log2;   // log2(e)/sqrt(192)
};

constexpr float kLog2e = 1.4426950408889634f;

// ===========================================================================
// dK / dV
// ===========================================================================
namespace kv {
constexpr uint32_t OFF_K = 0;                       // K^C 0-63, K^C 64-127, k^S: 3 x [128 x 64]
constexpr uint32_t OFF_V = OFF_K + 3 * SUB128;      // V 0-63, V 64-127
constexpr uint32_t OFF_RING = OFF_V + 2 * SUB128;   // NS x (Q_i: 3 x [64 x 64], dO~_i: 2 x [64 x 64])
constexpr uint32_t OFF_DS = OFF_RING + NS * SLOT;   // dS^T [128 keys x 64 queries]
constexpr uint32_t OFF_LD = OFF_DS + SUB128;        // [2][2][64] floats: lse * log2(e), D
constexpr uint32_t OFF_BAR = OFF_LD + 1024;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
// TMEM columns
constexpr uint32_t TS = 0, TDP = 128, TDV = 192, TDK = 320;
enum Bar { KVFULL = 0, RFULL, REMPTY = RFULL + NS, SFULL = REMPTY + NS, DPFULL = SFULL + 2, DPFREE, PFULL, DKDONE,
           DRAIN, NBAR };
}  // namespace kv

__global__ void __launch_bounds__(192, 1)
dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
            const __grid_constant__ CUtensorMap tmKC, const __grid_constant__ CUtensorMap tmKS,
            const __grid_constant__ CUtensorMap tmV, Params p) {
  using namespace kv;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  float* sld = reinterpret_cast<float*>(smem_raw + (sbase - sraw) + OFF_LD);
  volatile int* abort = &abort_flag;
  auto bar = [&](int i) { return sbase + OFF_BAR + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int k0 = kt * 128;
  const int n_q = (p.T - k0 + 63) / 64;               // 64-query tiles from k0 to the end
  if (threadIdx.x == 0) abort_flag = device_error_pending() ? 1 : 0;
  __syncthreads();
  if (abort_flag) return;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 0; i < NBAR; ++i) mbar_init(bar(i), (i == PFULL || i == DPFREE) ? 128 : 1);
    fence_mbar_init();
  }
  if (warp == 5) { tmem_alloc(smem_u32(&tmem_slot), 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmDO); tma_prefetch_desc(&tmKC);
      tma_prefetch_desc(&tmKS); tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(bar(KVFULL), 5 * SUB128);
      tma_load_3d(sbase + OFF_K, &tmKC, bar(KVFULL), h * 128, k0, b);
      tma_load_3d(sbase + OFF_K + SUB128, &tmKC, bar(KVFULL), h * 128 + 64, k0, b);
      tma_load_3d(sbase + OFF_K + 2 * SUB128, &tmKS, bar(KVFULL), 0, k0, b);
      tma_load_3d(sbase + OFF_V, &tmV, bar(KVFULL), h * 128, k0, b);
      tma_load_3d(sbase + OFF_V + SUB128, &tmV, bar(KVFULL), h * 128 + 64, k0, b);
      bool ok = true;
      for (int i = 0; i < n_q && ok; ++i) {
        const int s = i % NS;
        if (!mbar_wait(bar(REMPTY + s), ((uint32_t)(i / NS) & 1u) ^ 1u, abort)) { ok = false; break; }
        const uint32_t dst = sbase + OFF_RING + (uint32_t)s * SLOT;
        const int q0 = k0 + 64 * i;
        mbar_arrive_expect_tx(bar(RFULL + s), SLOT);
        for (int c = 0; c < 3; ++c) tma_load_3d(dst + c * SUB64, &tmQ, bar(RFULL + s), h * 192 + 64 * c, q0, b);
        for (int c = 0; c < 2; ++c) tma_load_3d(dst + (3 + c) * SUB64, &tmDO, bar(RFULL + s), h * 128 + 64 * c, q0, b);
      }
      // Never leave with copies in flight into this CTA's shared memory.
      mbar_wait_drain(bar(KVFULL), 0);
      for (int i = (n_q > NS ? n_q - NS : 0); i < n_q; ++i)
        mbar_wait_drain(bar(RFULL + i % NS), (uint32_t)(i / NS) & 1u);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id64 = idesc_bf16_f32(128, 64, false, false);     // K-major x K-major, N = 64 queries
      constexpr uint32_t idDV = idesc_bf16_f32(128, 128, false, true);     // P^T (TMEM) x dO~ (MN-major)
      constexpr uint32_t idDK = idesc_bf16_f32(128, 192, false, true);     // dS^T (K-major) x Q (MN-major)
      bool ok = mbar_wait(bar(KVFULL), 0, abort);
      auto wait_ok = [&](int bi, uint32_t ph) {
        ok = ok && mbar_wait(bar(bi), ph, abort);
        if (ok) tc_fence_after();
        return ok;
      };
      auto slot_of = [&](int i) { return sbase + OFF_RING + (uint32_t)(i % NS) * SLOT; };
      auto issue_S = [&](int i) {                  // S^T(i) = K Q_i^T into buffer i & 1
        const uint32_t q = slot_of(i);
        const uint32_t d = tmem + TS + 64u * (uint32_t)(i & 1);
#pragma unroll
        for (int x = 0; x < 12; ++x)               // 3 sub-tiles of 64 dims x 4 steps of 16
          mma_ss(d, sdesc_sw128(sbase + OFF_K + (uint32_t)(x >> 2) * SUB128 + (uint32_t)(x & 3) * 32u, 16, 1024),
                 sdesc_sw128(q + (uint32_t)(x >> 2) * SUB64 + (uint32_t)(x & 3) * 32u, 16, 1024), id64, x > 0);
        mma_commit(bar(SFULL + (i & 1)));
      };
      auto issue_DP = [&](int i) {                 // dP^T(i) = V dO~_i^T
        const uint32_t q = slot_of(i);
#pragma unroll
        for (int x = 0; x < 8; ++x)
          mma_ss(tmem + TDP, sdesc_sw128(sbase + OFF_V + (uint32_t)(x >> 2) * SUB128 + (uint32_t)(x & 3) * 32u, 16, 1024),
                 sdesc_sw128(q + (3u + (uint32_t)(x >> 2)) * SUB64 + (uint32_t)(x & 3) * 32u, 16, 1024), id64, x > 0);
        mma_commit(bar(DPFULL));
      };
      if (ok && n_q > 0 && wait_ok(RFULL, 0)) {
        issue_S(0);
        issue_DP(0);
      }
      for (int i = 0; ok && i < n_q; ++i) {
        const int s = i % NS;
        if (i + 1 < n_q) {
          if (!wait_ok(RFULL + (i + 1) % NS, (uint32_t)((i + 1) / NS) & 1u)) break;
          // S^T buffer (i+1) & 1 held P^T(i-1), read by dV(i-1): issued earlier.
          issue_S(i + 1);
          // dP^T's buffer is free once the compute warps have loaded dP^T(i)
          // (they do that first), so dP^T(i+1) runs while they work on tile i.
          if (!wait_ok(DPFREE, (uint32_t)i & 1u)) break;
          issue_DP(i + 1);
        }
        if (!wait_ok(PFULL, (uint32_t)i & 1u)) break;
        const uint32_t q = slot_of(i);
        const uint32_t tP = tmem + TS + 64u * (uint32_t)(i & 1);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)             // dV += P^T dO~_i, 16 queries per step
          mma_ts(tmem + TDV, tP + 8u * (uint32_t)kk, sdesc_sw128(q + 3u * SUB64 + (uint32_t)kk * 2048u, SUB64, 1024), idDV,
                 (i > 0 || kk > 0));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)             // dK += dS^T Q_i
          mma_ss(tmem + TDK, sdesc_sw128(sbase + OFF_DS + (uint32_t)kk * 32u, 16, 1024),
                 sdesc_sw128(q + (uint32_t)kk * 2048u, SUB64, 1024), idDK, (i > 0 || kk > 0));
        mma_commit(bar(REMPTY + s));
        mma_commit(bar(DKDONE));
      }
      mma_commit(bar(DRAIN));
      mbar_wait_drain(bar(DRAIN), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ P^T, dS^T and the epilogue
    const int r = threadIdx.x;                   // key row inside the tile == TMEM lane
    const int key = k0 + r;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float c = p.scale_log2;
    bool ok = true;
    auto wait_warp = [&](int bi, uint32_t ph) {
      const bool w = mbar_wait(bar(bi), ph, abort);
      return __all_sync(0xffffffffu, w) != 0;
    };
    // lse * log2(e) and D of the queries of tile i, staged by threads 0-63
    // (lse) and 64-127 (D) one tile ahead.
    auto fetch = [&](int i) -> float {
      const int q = k0 + 64 * i + (r & 63);
      if (i >= n_q || q >= p.T) return 0.f;
      const size_t idx = ((size_t)b * p.T + q) * p.H + h;
      return r < 64 ? p.lse[idx] * kLog2e : p.D[idx];
    };
    sld[r] = fetch(0);                           // parity 0: [0][lse | D]
    float nxt = fetch(1);
    named_bar_sync(1, 128);
    for (int i = 0; i < n_q; ++i) {
      const float* lse2 = sld + (i & 1) * 128;
      const float* Dq = lse2 + 64;
      const int q0 = k0 + 64 * i;
      float s[64], dp[64];
      if (ok) ok = wait_warp(SFULL + (i & 1), (uint32_t)(i >> 1) & 1u);
      if (ok) ok = wait_warp(DPFULL, (uint32_t)i & 1u);
      if (ok) {
        tc_fence_after();
        const uint32_t ts = tmem + lane_off + TS + 64u * (uint32_t)(i & 1);
        tmem_ld32(ts, *reinterpret_cast<float(*)[32]>(&s[0]));
        tmem_ld32(ts + 32u, *reinterpret_cast<float(*)[32]>(&s[32]));
        tmem_ld32(tmem + lane_off + TDP, *reinterpret_cast<float(*)[32]>(&dp[0]));
        tmem_ld32(tmem + lane_off + TDP + 32u, *reinterpret_cast<float(*)[32]>(&dp[32]));
        tmem_wait_ld_dep(*reinterpret_cast<float(*)[32]>(&s[0]));
        tmem_wait_ld_dep(*reinterpret_cast<float(*)[32]>(&s[32]));
        tmem_wait_ld_dep(*reinterpret_cast<float(*)[32]>(&dp[0]));
        tmem_wait_ld_dep(*reinterpret_cast<float(*)[32]>(&dp[32]));
        tc_fence_before();
        mbar_arrive(bar(DPFREE));
        uint32_t pk[32], dk[32];
        // Query tiles from the third on lie wholly after the CTA's keys; only
        // those that reach past T (and the first two) need the mask.
        if (i >= 2 && q0 + 64 <= p.T) {
          // Two scores at a time on the FMA pipe (.f32x2): exponent argument,
          // dP - D and P (dP - D).
          const uint64_t c2 = f2(c, c);
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            float x0, x1, d0, d1;
            f2split(fma_f2(f2(s[e], s[e + 1]), c2, f2(-lse2[e], -lse2[e + 1])), x0, x1);
            const float p0 = ex2(x0), p1 = ex2(x1);
            pk[e >> 1] = pack_bf16x2(p0, p1);
            f2split(mul_f2(f2(p0, p1), sub_f2(f2(dp[e], dp[e + 1]), f2(Dq[e], Dq[e + 1]))), d0, d1);
            dk[e >> 1] = pack_bf16x2(d0, d1);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            float pv[2], dv[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int q = q0 + e + u;
              const bool live = q < p.T && key <= q;  // causal: the key is at or before the query
              pv[u] = live ? ex2(fmaf(s[e + u], c, -lse2[e + u])) : 0.f;
              dv[u] = pv[u] * (dp[e + u] - Dq[e + u]);
            }
            pk[e >> 1] = pack_bf16x2(pv[0], pv[1]);
            dk[e >> 1] = pack_bf16x2(dv[0], dv[1]);
          }
        }
        // P^T over the first 32 columns of its S^T buffer (read above).
        tmem_st32u(ts, pk);
        // dS^T into the shared tile once dK(i-1) has finished reading it.
        if (i > 0) ok = wait_warp(DKDONE, (uint32_t)(i - 1) & 1u);
        if (ok) {
          const uint32_t row = sbase + OFF_DS + (uint32_t)r * 128u;
#pragma unroll
          for (int cc = 0; cc < 8; ++cc)
            st_shared_v4(row + ((uint32_t)(cc ^ (r & 7)) << 4), dk[4 * cc], dk[4 * cc + 1], dk[4 * cc + 2], dk[4 * cc + 3]);
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        if (ok) mbar_arrive(bar(PFULL));
      }
      // Next tile's lse / D (every thread reaches this barrier each tile).
      sld[((i + 1) & 1) * 128 + r] = nxt;
      nxt = fetch(i + 2);
      named_bar_sync(1, 128);
    }
    if (ok && n_q > 0) ok = wait_warp(DKDONE, (uint32_t)(n_q - 1) & 1u);
    if (ok) {
      tc_fence_after();
      const bool valid = key < p.T;
      const size_t row = ((size_t)b * p.T + (valid ? key : 0)) * p.H + h;
#pragma unroll 1
      for (int k = 0; k < 4; ++k) {                // dV: 128 columns
        float v[32];
        tmem_ld32(tmem + lane_off + TDV + 32u * k, v);
        tmem_wait_ld_dep(v);
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(p.dV + row * 128 + 32 * k);
#pragma unroll
          for (int e = 0; e < 8; ++e) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
        }
      }
#pragma unroll 1
      for (int k = 0; k < 6; ++k) {                // dK: 128 K^C columns, then 64 k^S columns
        float v[32];
        tmem_ld32(tmem + lane_off + TDK + 32u * k, v);
        tmem_wait_ld_dep(v);
        if (valid) {
          if (k < 4) {
            float4* dst = reinterpret_cast<float4*>(p.dKC + row * 128 + 32 * k);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(v[4 * e] * p.scale, v[4 * e + 1] * p.scale, v[4 * e + 2] * p.scale,
                                   v[4 * e + 3] * p.scale);
          } else {
            float* dst = p.dkS + ((size_t)b * p.T + key) * 64 + 32 * (k - 4);
#pragma unroll
            for (int e = 0; e < 32; ++e) atomicAdd(dst + e, v[e] * p.scale);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ===========================================================================
// dQ
// ===========================================================================
namespace q {
constexpr uint32_t OFF_Q = 0;                       // 3 x [128 x 64]
constexpr uint32_t OFF_DO = OFF_Q + 3 * SUB128;     // 2 x [128 x 64]
constexpr uint32_t OFF_RING = OFF_DO + 2 * SUB128;  // NS x (K_j: K^C 0-63, K^C 64-127, k^S; V_j 0-63, 64-127) of 64 rows
constexpr uint32_t OFF_BAR = OFF_RING + NS * SLOT;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t TS = 0, TDP = 128, TDQ = 256;    // S, dP double buffers (64 columns each), dQ (192)
enum Bar { QFULL = 0, RFULL, REMPTY = RFULL + NS, SFULL = REMPTY + NS, DPFULL = SFULL + 2, PFULL = DPFULL + 2,
           DQDONE, DRAIN, NBAR };
}  // namespace q

__global__ void __launch_bounds__(192, 1)
dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
          const __grid_constant__ CUtensorMap tmKC, const __grid_constant__ CUtensorMap tmKS,
          const __grid_constant__ CUtensorMap tmV, Params p) {
  using namespace q;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  volatile int* abort = &abort_flag;
  auto bar = [&](int i) { return sbase + OFF_BAR + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Longest rows first: query tile n_qt - 1 - blockIdx.x.
  const int n_qt = (p.T + 127) / 128;
  const int qt = n_qt - 1 - (int)blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int q0 = qt * 128;
  const int n_k = (min(q0 + 128, p.T) + 63) / 64;     // 64-key tiles up to the diagonal
  if (threadIdx.x == 0) abort_flag = device_error_pending() ? 1 : 0;
  __syncthreads();
  if (abort_flag) return;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 0; i < NBAR; ++i) mbar_init(bar(i), i == PFULL ? 128 : 1);
    fence_mbar_init();
  }
  if (warp == 5) { tmem_alloc(smem_u32(&tmem_slot), 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmDO); tma_prefetch_desc(&tmKC);
      tma_prefetch_desc(&tmKS); tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(bar(QFULL), 5 * SUB128);
      for (int c = 0; c < 3; ++c) tma_load_3d(sbase + OFF_Q + c * SUB128, &tmQ, bar(QFULL), h * 192 + 64 * c, q0, b);
      for (int c = 0; c < 2; ++c) tma_load_3d(sbase + OFF_DO + c * SUB128, &tmDO, bar(QFULL), h * 128 + 64 * c, q0, b);
      bool ok = true;
      for (int j = 0; j < n_k && ok; ++j) {
        const int s = j % NS;
        if (!mbar_wait(bar(REMPTY + s), ((uint32_t)(j / NS) & 1u) ^ 1u, abort)) { ok = false; break; }
        const uint32_t dst = sbase + OFF_RING + (uint32_t)s * SLOT;
        const int kr = 64 * j;
        mbar_arrive_expect_tx(bar(RFULL + s), SLOT);
        tma_load_3d(dst, &tmKC, bar(RFULL + s), h * 128, kr, b);
        tma_load_3d(dst + SUB64, &tmKC, bar(RFULL + s), h * 128 + 64, kr, b);
        tma_load_3d(dst + 2 * SUB64, &tmKS, bar(RFULL + s), 0, kr, b);
        tma_load_3d(dst + 3 * SUB64, &tmV, bar(RFULL + s), h * 128, kr, b);
        tma_load_3d(dst + 4 * SUB64, &tmV, bar(RFULL + s), h * 128 + 64, kr, b);
      }
      mbar_wait_drain(bar(QFULL), 0);
      for (int j = (n_k > NS ? n_k - NS : 0); j < n_k; ++j)
        mbar_wait_drain(bar(RFULL + j % NS), (uint32_t)(j / NS) & 1u);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t id64 = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t idDQ = idesc_bf16_f32(128, 192, false, true);   // dS (TMEM) x K_j (MN-major)
      bool ok = mbar_wait(bar(QFULL), 0, abort);
      auto wait_ok = [&](int bi, uint32_t ph) {
        ok = ok && mbar_wait(bar(bi), ph, abort);
        if (ok) tc_fence_after();
        return ok;
      };
      auto slot_of = [&](int j) { return sbase + OFF_RING + (uint32_t)(j % NS) * SLOT; };
      auto issue_SDP = [&](int j) {                // S(j) = Q K_j^T, dP(j) = dO~ V_j^T into buffers j & 1
        const uint32_t k = slot_of(j);
        const uint32_t dS = tmem + TS + 64u * (uint32_t)(j & 1), dD = tmem + TDP + 64u * (uint32_t)(j & 1);
#pragma unroll
        for (int x = 0; x < 12; ++x)
          mma_ss(dS, sdesc_sw128(sbase + OFF_Q + (uint32_t)(x >> 2) * SUB128 + (uint32_t)(x & 3) * 32u, 16, 1024),
                 sdesc_sw128(k + (uint32_t)(x >> 2) * SUB64 + (uint32_t)(x & 3) * 32u, 16, 1024), id64, x > 0);
        mma_commit(bar(SFULL + (j & 1)));
#pragma unroll
        for (int x = 0; x < 8; ++x)
          mma_ss(dD, sdesc_sw128(sbase + OFF_DO + (uint32_t)(x >> 2) * SUB128 + (uint32_t)(x & 3) * 32u, 16, 1024),
                 sdesc_sw128(k + (3u + (uint32_t)(x >> 2)) * SUB64 + (uint32_t)(x & 3) * 32u, 16, 1024), id64, x > 0);
        mma_commit(bar(DPFULL + (j & 1)));
      };
      if (ok && n_k > 0 && wait_ok(RFULL, 0)) issue_SDP(0);
      for (int j = 0; ok && j < n_k; ++j) {
        if (j + 1 < n_k) {
          // Buffers (j+1) & 1: S(j-1) was loaded by the softmax warps before
          // PFULL(j-1), dS(j-1) (over dP) read by dQ(j-1): both done or issued.
          if (!wait_ok(RFULL + (j + 1) % NS, (uint32_t)((j + 1) / NS) & 1u)) break;
          issue_SDP(j + 1);
        }
        if (!wait_ok(PFULL, (uint32_t)j & 1u)) break;
        const uint32_t k = slot_of(j);
        const uint32_t tdS = tmem + TDP + 64u * (uint32_t)(j & 1);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)             // dQ += dS K_j, 16 keys per step
          mma_ts(tmem + TDQ, tdS + 8u * (uint32_t)kk, sdesc_sw128(k + (uint32_t)kk * 2048u, SUB64, 1024), idDQ,
                 (j > 0 || kk > 0));
        mma_commit(bar(REMPTY + j % NS));
      }
      mma_commit(bar(DQDONE));
      mma_commit(bar(DRAIN));
      mbar_wait_drain(bar(DRAIN), 0);
    }
    __syncwarp();
  } else {
    const int r = threadIdx.x;                   // query row == TMEM lane
    const int t = q0 + r;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float c = p.scale_log2;
    const bool valid = t < p.T;
    const size_t ridx = ((size_t)b * p.T + (valid ? t : 0)) * p.H + h;
    const float lse2 = valid ? p.lse[ridx] * kLog2e : 0.f;
    const float Dr = valid ? p.D[ridx] : 0.f;
    bool ok = true;
    auto wait_warp = [&](int bi, uint32_t ph) {
      const bool w = mbar_wait(bar(bi), ph, abort);
      return __all_sync(0xffffffffu, w) != 0;
    };
    // PFULL counts 128 arrivals per tile, and the S / dP of tile j+1 are
    // usually ready before every warp has finished tile j.  A warp that ran a
    // whole tile ahead would put its tile-(j+1) arrivals into tile j's phase,
    // and the dQ product would read the dS rows of a warp that has not
    // written them yet.  The vote at the end of each tile keeps the four warps
    // in step (and makes a failed wait end the loop in all of them at once).
    for (int j = 0; j < n_k; ++j) {
      const uint32_t par = (uint32_t)(j >> 1) & 1u;
      if (ok) ok = wait_warp(SFULL + (j & 1), par) && wait_warp(DPFULL + (j & 1), par);
      if (ok) {
        tc_fence_after();
        float s[64], dp[64];
        const uint32_t ts = tmem + lane_off + TS + 64u * (uint32_t)(j & 1);
        const uint32_t td = tmem + lane_off + TDP + 64u * (uint32_t)(j & 1);
        tmem_ld32(ts, *reinterpret_cast<float(*)[32]>(&s[0]));
        tmem_ld32(ts + 32u, *reinterpret_cast<float(*)[32]>(&s[32]));
        tmem_ld32(td, *reinterpret_cast<float(*)[32]>(&dp[0]));
        tmem_ld32(td + 32u, *reinterpret_cast<float(*)[32]>(&dp[32]));
        tmem_wait_ld_dep(*reinterpret_cast<float(*)[32]>(&s[0]));
        tmem_wait_ld_dep(*reinterpret_cast<float(*)[32]>(&s[32]));
        tmem_wait_ld_dep(*reinterpret_cast<float(*)[32]>(&dp[0]));
        tmem_wait_ld_dep(*reinterpret_cast<float(*)[32]>(&dp[32]));
        const int kb = 64 * j;
        uint32_t dk[32];
        // Only the key tiles that reach past the tile's first row (and a row
        // past T) need the mask.
        if (kb + 63 <= q0 && valid) {
          // Two scores at a time on the FMA pipe (.f32x2), as in dkdv_kernel.
          const uint64_t c2 = f2(c, c), n2 = f2(-lse2, -lse2), D2 = f2(Dr, Dr);
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            float x0, x1, d0, d1;
            f2split(fma_f2(f2(s[e], s[e + 1]), c2, n2), x0, x1);
            f2split(mul_f2(f2(ex2(x0), ex2(x1)), sub_f2(f2(dp[e], dp[e + 1]), D2)), d0, d1);
            dk[e >> 1] = pack_bf16x2(d0, d1);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            float dv[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const bool live = valid && kb + e + u <= t;   // causal (keys past T sit past every valid row)
              const float pv = live ? ex2(fmaf(s[e + u], c, -lse2)) : 0.f;
              dv[u] = pv * (dp[e + u] - Dr);
            }
            dk[e >> 1] = pack_bf16x2(dv[0], dv[1]);
          }
        }
        // dS over the first 32 columns of its dP buffer (this thread's dP row is in registers).
        tmem_st32u(td, dk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(PFULL));
      }
      ok = !bar_red_or(1, 128, !ok);
      if (!ok) break;
    }
    if (ok) ok = wait_warp(DQDONE, 0);
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int k = 0; k < 6; ++k) {
        float v[32];
        tmem_ld32(tmem + lane_off + TDQ + 32u * k, v);
        tmem_wait_ld_dep(v);
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(p.dQ + ridx * 192 + 32 * k);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(v[4 * e] * p.scale, v[4 * e + 1] * p.scale, v[4 * e + 2] * p.scale, v[4 * e + 3] * p.scale);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc_bwd
}  // namespace gmla
