// Causal gated MLA attention forward on the 5th-generation tensor cores
// (tcgen05 + TMEM + TMA), with the per-head max logit fused into the pass.
//
// Arithmetic ("Kimi K3 · Gated MLA · OpenModelAtlas", "All 20 steps"):
//   S_h = Q_h K_h^T / sqrt(192),  K_h = [K^C_h (128) | k^S (64, shared)]
//   A   = causal softmax (fp32),  O_h = A V_h (128),  o = sigmoid(g) * O
// plus maxlogit[h] = max over b, t, s <= t of S_h[t][s] (the statistic of
// "Anthology of the SOTA" SOTA-131's per-head max-logit check).
//
// One CTA = one 128-row query tile of one (batch, head), launched head-major;
// key/value tiles of 128 positions stream through a 3-slot TMA ring.  The shared key k^S is
// never broadcast in memory: S is two MMA groups (q^C.K^C over 128 dims and
// q^S.k^S over 64 dims) accumulating into the same TMEM tile.
//
// Warp roles (192 threads):
//   warps 0-3  softmax + epilogue; thread r owns query row r (= TMEM lane r)
//   warp  4    TMA producer (one lane)
//   warp  5    TMEM allocator and MMA issuer (one lane)
// TMEM (512 columns): S double buffer at columns [0,128) and [128,256),
// O accumulator at [256,384).
// Shared memory (1024-aligned, 128B-swizzled 16 KB sub-tiles of 128 x 64 bf16):
//   Q: 3 sub-tiles (q^C 0-63, q^C 64-127, q^S) | ring: 3 slots x 3 sub-tiles
//   (K slot = K^C 0-63, K^C 64-127, k^S; V slot = V 0-63, V 64-127).  P never
//   goes through shared memory: it is written into TMEM over its S buffer.
// Softmax uses base-2 exponentials of the scaled logits with a lazily
// updated reference max: O and l are rescaled only when a row's max grows by
// more than a factor 2^8, which keeps every exponential <= 256 and is exact
// once O is divided by l at the end.
#pragma once

#include "sm100.cuh"

namespace gmla {
namespace tc_attn {

using namespace sm100;

constexpr int BM = 128, BN = 128;
constexpr int NSTAGE = 3;
constexpr uint32_t SUB = 128 * 128;                       // bytes of one 128 x 64 bf16 sub-tile
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_RING = OFF_Q + 3 * SUB;
constexpr uint32_t OFF_BAR = OFF_RING + NSTAGE * 3 * SUB;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;     // + barriers + alignment slack

// P_j and the P.V product of tile j hand off through PFULL + (j & 1) and
// PVDONE + (j & 1): a softmax warp may run one tile ahead of the MMA issuer.
// QEMPTY (gated bf16 form): every S product of the tile is done, so the Q
// buffer is free for the gate tile (GFULL).  Without a gate the bf16 epilogue
// stages O there after the last P.V product, which completes after every S.
enum Bar { QFULL = 0, KVFULL = 1, KVEMPTY = KVFULL + NSTAGE, SFULL = KVEMPTY + NSTAGE, PFULL = SFULL + 2,
           PVDONE = PFULL + 2, QEMPTY = PVDONE + 2, GFULL, DRAIN, NBAR };

constexpr float kRescaleLog2 = 8.f;   // rescale O when the row max grows by > 2^8

struct Params {
  int B, T, H, n_qtiles;
  const __nv_bfloat16* g;   // [B][T][H*128] or nullptr
  void* O;                  // [B][T][H*128], bf16 or (training variant) fp32
  float* maxlogit;          // [H]
  float* lse;               // [B][T][H] row log-sum-exp of the scaled logits, or nullptr
  float scale;              // 1/sqrt(192)
  float scale_log2;         // log2(e)/sqrt(192)
};

__device__ __forceinline__ float sigmoidf_(float x) { return 1.f / (1.f + __expf(-x)); }

// OUT_F32: the output is kept in fp32 (the training variant of "Gated MLA
// et NoPE", "Un détail de précision numérique": no rounding of o to bf16);
// that epilogue stores straight from registers.  The bf16 epilogue goes
// through the Q buffer, free once the tile's last S product is done: the
// producer loads the gate tile there (tmG) during the last steps, each
// softmax thread turns its row of it into its row of o in place, and one
// thread writes the tile with two TMA stores (tmO; rows past T are not
// written).
template <bool OUT_F32>
__global__ void __launch_bounds__(192, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKC,
                const __grid_constant__ CUtensorMap tmKS, const __grid_constant__ CUtensorMap tmV,
                const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmO, Params p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  volatile int* abort = &abort_flag;
  auto bar = [&](int i) { return sbase + OFF_BAR + 8u * (uint32_t)i; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Head-major order: the CTAs in flight work on one or two heads, whose
  // K^C / V / k^S tiles then stay in L2 for every query tile that reads them;
  // inside a head the longest causal rows go first.
  const int QB = p.n_qtiles * p.B;
  const int h = (int)(blockIdx.x / QB);
  const int rem = (int)(blockIdx.x % QB);
  const int qt = p.n_qtiles - 1 - rem / p.B, b = rem % p.B;
  const int n_kv = qt + 1;

  // A CTA launched after another one gave up does no work (the error stays
  // recorded until the host reads it with gmla_device_status).
  if (threadIdx.x == 0) abort_flag = device_error_pending() ? 1 : 0;
  __syncthreads();
  if (abort_flag) return;
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_init(bar(QFULL), 1);
    for (int i = 0; i < NSTAGE; ++i) { mbar_init(bar(KVFULL + i), 1); mbar_init(bar(KVEMPTY + i), 1); }
    mbar_init(bar(SFULL), 1);
    mbar_init(bar(SFULL + 1), 1);
    mbar_init(bar(PFULL), 128);
    mbar_init(bar(PFULL + 1), 128);
    mbar_init(bar(PVDONE), 1);
    mbar_init(bar(PVDONE + 1), 1);
    mbar_init(bar(QEMPTY), 1);
    mbar_init(bar(GFULL), 1);
    mbar_init(bar(DRAIN), 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(&tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmKC); tma_prefetch_desc(&tmKS); tma_prefetch_desc(&tmV);
      const int qcol = h * 192, kcol = h * 128;
      mbar_arrive_expect_tx(bar(QFULL), 3 * SUB);
      tma_load_3d(sbase + OFF_Q, &tmQ, bar(QFULL), qcol, qt * BM, b);
      tma_load_3d(sbase + OFF_Q + SUB, &tmQ, bar(QFULL), qcol + 64, qt * BM, b);
      tma_load_3d(sbase + OFF_Q + 2 * SUB, &tmQ, bar(QFULL), qcol + 128, qt * BM, b);
      uint32_t u = 0;
      // Items in the order the MMA warp consumes them: K_0, then K_{j+1} (if any) and V_j for each j.
      auto load = [&](bool isK, int j) -> bool {
        const uint32_t slot = u % NSTAGE, ph = (u / NSTAGE) & 1u;
        if (!mbar_wait(bar(KVEMPTY + slot), ph ^ 1u, abort)) return false;
        const uint32_t dst = sbase + OFF_RING + slot * 3 * SUB;
        if (isK) {
          mbar_arrive_expect_tx(bar(KVFULL + slot), 3 * SUB);
          tma_load_3d(dst, &tmKC, bar(KVFULL + slot), kcol, j * BN, b);
          tma_load_3d(dst + SUB, &tmKC, bar(KVFULL + slot), kcol + 64, j * BN, b);
          tma_load_3d(dst + 2 * SUB, &tmKS, bar(KVFULL + slot), 0, j * BN, b);
        } else {
          mbar_arrive_expect_tx(bar(KVFULL + slot), 2 * SUB);
          tma_load_3d(dst, &tmV, bar(KVFULL + slot), kcol, j * BN, b);
          tma_load_3d(dst + SUB, &tmV, bar(KVFULL + slot), kcol + 64, j * BN, b);
        }
        ++u;
        return true;
      };
      bool ok = load(true, 0);
      for (int j = 0; ok && j < n_kv; ++j) {
        if (j + 1 < n_kv) ok = load(true, j + 1);
        if (ok) ok = load(false, j);
      }
      // bf16 epilogue: the gate tile into the Q buffer once Q is no longer read.
      bool g_issued = false;
      if constexpr (!OUT_F32) {
        if (ok && p.g != nullptr && mbar_wait(bar(QEMPTY), 0, abort)) {
          mbar_arrive_expect_tx(bar(GFULL), 2 * SUB);
          tma_load_3d(sbase + OFF_Q, &tmG, bar(GFULL), kcol, qt * BM, b);
          tma_load_3d(sbase + OFF_Q + SUB, &tmG, bar(GFULL), kcol + 64, qt * BM, b);
          g_issued = true;
        }
      }
      // Never leave with copies in flight into this CTA's shared memory.
      mbar_wait_drain(bar(QFULL), 0);
      if (g_issued) mbar_wait_drain(bar(GFULL), 0);
      for (uint32_t k = (u > NSTAGE ? u - NSTAGE : 0); k < u; ++k)
        mbar_wait_drain(bar(KVFULL + k % NSTAGE), (k / NSTAGE) & 1u);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);   // Q (K-major) x K (K-major)
      constexpr uint32_t idO = idesc_bf16_f32(128, 128, false, true);    // P (TMEM) x V (MN-major)
      const uint32_t tS0 = tmem, tO = tmem + 256;
      uint32_t u = 0;
      bool ok = mbar_wait(bar(QFULL), 0, abort);
      auto issue_S = [&](int buf, uint32_t slot) {
        const uint32_t kbase = sbase + OFF_RING + slot * 3 * SUB;
#pragma unroll
        for (int i = 0; i < 12; ++i) {
          const uint32_t qa = sbase + OFF_Q + (uint32_t)(i >> 2) * SUB + (uint32_t)(i & 3) * 32u;
          const uint32_t kb = kbase + (uint32_t)(i >> 2) * SUB + (uint32_t)(i & 3) * 32u;
          mma_ss(tS0 + (uint32_t)buf * 128u, sdesc_sw128(qa, 16, 1024), sdesc_sw128(kb, 16, 1024), idS, i > 0);
        }
        mma_commit(bar(SFULL + buf));
        mma_commit(bar(KVEMPTY + slot));
      };
      if (ok) {
        ok = mbar_wait(bar(KVFULL + 0), 0, abort);
        if (ok) {
          tc_fence_after();
          issue_S(0, 0);
          u = 1;
          if (!OUT_F32 && p.g && n_kv == 1) mma_commit(bar(QEMPTY));   // the tile's last S product (gate staging)
        }
      }
      for (int j = 0; ok && j < n_kv; ++j) {
        if (j + 1 < n_kv) {
          const uint32_t slot = u % NSTAGE, ph = (u / NSTAGE) & 1u;
          if (!mbar_wait(bar(KVFULL + slot), ph, abort)) { ok = false; break; }
          tc_fence_after();
          issue_S((j + 1) & 1, slot);
          ++u;
          if (!OUT_F32 && p.g && j + 2 == n_kv) mma_commit(bar(QEMPTY));   // the tile's last S product (gate staging)
        }
        if (!mbar_wait(bar(PFULL + (j & 1)), (uint32_t)(j >> 1) & 1u, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t slot = u % NSTAGE, ph = (u / NSTAGE) & 1u;
        if (!mbar_wait(bar(KVFULL + slot), ph, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t vbase = sbase + OFF_RING + slot * 3 * SUB;
        // P_j sits in the first 64 columns of S buffer (j & 1), two bf16 per column.
        const uint32_t tP = tS0 + (uint32_t)(j & 1) * 128u;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t vb = vbase + (uint32_t)i * 2048u;     // 16 keys x 128 B rows
          mma_ts(tO, tP + 8u * (uint32_t)i, sdesc_sw128(vb, SUB, 1024), idO, (j > 0 || i > 0));
        }
        mma_commit(bar(PVDONE + (j & 1)));
        mma_commit(bar(KVEMPTY + slot));
        ++u;
      }
      // Drain every MMA this thread issued before TMEM is released.
      mma_commit(bar(DRAIN));
      mbar_wait_drain(bar(DRAIN), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int r = threadIdx.x;                 // query row inside the tile == TMEM lane
    const int t = qt * BM + r;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t tS_row = tmem + lane_off, tO_row = tmem + lane_off + 256;
    const float c = p.scale_log2;
    float m_used = -INFINITY, l = 0.f, true_max = -INFINITY;
    bool ok = true;
    // Every lane waits; the outcome is made warp-uniform so that the
    // warp-collective TMEM accesses below are always executed by all lanes.
    auto wait_warp = [&](int i, uint32_t ph) {
      const bool w = mbar_wait(bar(i), ph, abort);
      return __all_sync(0xffffffffu, w) != 0;
    };
    for (int j = 0; j < n_kv; ++j) {
      const int buf = j & 1;
      if (!wait_warp(SFULL + buf, (uint32_t)(j >> 1) & 1u)) { ok = false; break; }
      tc_fence_after();
      float s[128];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float (&chunk)[32] = *reinterpret_cast<float(*)[32]>(&s[32 * k]);
        tmem_ld32(tS_row + (uint32_t)buf * 128u + 32u * k, chunk);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) tmem_wait_ld_dep(*reinterpret_cast<float(*)[32]>(&s[32 * k]));
      if (j == qt) {                           // diagonal tile: key column > query row is masked
#pragma unroll
        for (int k = 0; k < 128; ++k) s[k] = (k > r) ? -INFINITY : s[k];
      }
      // Row max with eight independent accumulators (a single chain would
      // serialise 127 dependent max operations).
      float pm[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) pm[q] = s[q];
#pragma unroll
      for (int k = 8; k < 128; ++k) pm[k & 7] = fmaxf(pm[k & 7], s[k]);
      const float mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])), fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
      true_max = fmaxf(true_max, mx);
      const bool need = (m_used == -INFINITY) || ((mx - m_used) * c > kRescaleLog2);
      const float m_new = need ? fmaxf(m_used, mx) : m_used;
      const float corr = need ? ex2((m_used - m_new) * c) : 1.f;
      const float neg = -m_new * c;
      uint32_t pk[64];
      // Exponent arguments and row-sum partials two at a time (.f32x2).
      const uint64_t c2 = f2(c, c), n2 = f2(neg, neg);
      uint64_t ps2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int e = 0; e < 128; e += 2) {
        float x0, x1;
        f2split(fma_f2(f2(s[e], s[e + 1]), c2, n2), x0, x1);
        const float a0 = ex2(x0), a1 = ex2(x1);
        ps2[(e >> 1) & 3] = add_f2(ps2[(e >> 1) & 3], f2(a0, a1));
        pk[e >> 1] = pack_bf16x2(a0, a1);
      }
      float ps[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) f2split(ps2[q], ps[2 * q], ps[2 * q + 1]);
      // P_j goes over P_{j-2} in this S buffer, whose P.V product completed
      // before S_j did (it was issued earlier).  Only a rescale of O waits,
      // for the P.V product of tile j-1, which O must hold before it is scaled.
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        if (!wait_warp(PVDONE + ((j - 1) & 1), (uint32_t)((j - 1) >> 1) & 1u)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float o[32];
          tmem_ld32(tO_row + 32u * k, o);
          tmem_wait_ld_dep(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= corr;
          tmem_st32(tO_row + 32u * k, o);
        }
        tmem_wait_st();
      }
      l = l * corr + (((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7])));
      m_used = m_new;
      // P into TMEM over the first 64 columns of its own S buffer.
      tmem_st32u(tS_row + (uint32_t)buf * 128u, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
      tmem_st32u(tS_row + (uint32_t)buf * 128u + 32u, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(PFULL + buf));
    }
    const bool ep = ok && wait_warp(PVDONE + ((n_kv - 1) & 1), (uint32_t)((n_kv - 1) >> 1) & 1u);
    const float inv_l = 1.f / l;
    const bool valid = t < p.T;
    if (ep) tc_fence_after();
    if constexpr (OUT_F32) {
      if (ep) {
        const size_t row_off = (((size_t)b * p.T + (valid ? t : 0)) * p.H + h) * 128;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float o[32];
          tmem_ld32(tO_row + 32u * k, o);
          tmem_wait_ld_dep(o);
          if (valid) {
            const uint4* gp = reinterpret_cast<const uint4*>(p.g + row_off + 32 * k);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              float gate[8];
              if (p.g) {
                uint4 gv = gp[v];
                const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float2 f = __bfloat1622float2(g2[e]);
                  gate[2 * e] = sigmoidf_(f.x);
                  gate[2 * e + 1] = sigmoidf_(f.y);
                }
              } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) gate[e] = 1.f;
              }
              float4* op = reinterpret_cast<float4*>(static_cast<float*>(p.O) + row_off + 32 * k) + 2 * v;
              op[0] = make_float4(o[8 * v] * inv_l * gate[0], o[8 * v + 1] * inv_l * gate[1],
                                  o[8 * v + 2] * inv_l * gate[2], o[8 * v + 3] * inv_l * gate[3]);
              op[1] = make_float4(o[8 * v + 4] * inv_l * gate[4], o[8 * v + 5] * inv_l * gate[5],
                                  o[8 * v + 6] * inv_l * gate[6], o[8 * v + 7] * inv_l * gate[7]);
            }
          }
        }
      }
    } else {
      // Row r of the staged tile: sub-tile k / 2 holds columns 64 (k / 2) ..,
      // 16-byte chunk c of the row at chunk c ^ (r & 7) (128-byte swizzle).
      const bool gated = p.g != nullptr;
      const bool staged = ep && (!gated || wait_warp(GFULL, 0));
      if (staged) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float o[32];
          tmem_ld32(tO_row + 32u * k, o);
          tmem_wait_ld_dep(o);
          const uint32_t rowb = sbase + OFF_Q + (uint32_t)(k >> 1) * SUB + (uint32_t)r * 128u;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint32_t addr = rowb + ((uint32_t)((((k & 1) << 2) + v) ^ (r & 7)) << 4);
            float gate[8];
            if (gated) {
              uint4 gv = ld_shared_v4(addr);
              const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(g2[e]);
                gate[2 * e] = sigmoidf_(f.x);
                gate[2 * e + 1] = sigmoidf_(f.y);
              }
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e) gate[e] = 1.f;
            }
            float y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] = o[8 * v + e] * inv_l * gate[e];
            st_shared_v4(addr, pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                         pack_bf16x2(y[6], y[7]));
          }
        }
        fence_proxy_async_smem();
      }
      // Every softmax thread reaches this vote once, whatever happened above.
      const bool all_staged = !bar_red_or(1, 128, !staged);
      if (all_staged && r == 0) {
        tma_store_3d(&tmO, sbase + OFF_Q, h * 128, qt * BM, b);
        tma_store_3d(&tmO, sbase + OFF_Q + SUB, h * 128 + 64, qt * BM, b);
        bulk_commit_group();
        bulk_wait_group_read<0>();               // the tile has left shared memory (it lands before the grid completes)
      }
    }
    if (ep) {
      if (p.lse && valid) p.lse[((size_t)b * p.T + t) * p.H + h] = fmaf(m_used, p.scale, __logf(l));
      float v = valid ? true_max * p.scale : -INFINITY;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
      if (lane == 0 && v > -INFINITY) atomic_max_float(p.maxlogit + h, v);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc_attn
}  // namespace gmla
