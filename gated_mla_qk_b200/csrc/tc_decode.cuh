// Absorbed-latent decode on tensor cores (bf16, H = 96, d_c = 128, d_s = 64,
// d_v = 128, kv_lora = 512).
//
// Arithmetic ("Kimi Qkclip" blog, section 3: decoding works on the cached
// latent; "Gated MLA et NoPE", "Le principe": 512 + 64 cached values per
// token).  For sequence i and head h, with W_UK,h / W_UV,h the K^C / V column
// blocks of W_UKV:
//   q~_h = [q^C_h W_UK,h^T | q^S_h]                          (absorb kernel)
//   s_j  = q~_h . cache_j / sqrt(192), p = softmax_j(s)
//   u_h  = sum_j p_j cache_j[0:512]                          (split kernel)
//   o_h  = (u_h / l) W_UV,h  (* sigmoid(g))                  (combine kernel)
//
// Split kernel: one CTA per (sequence, 1024-token chunk, half of the heads).
// The latent cache streams through two 72 KB TMA stages in tiles of 64
// tokens.  Per tile, two tcgen05 products share the same 128B-swizzled tile:
//   S^T [64 tokens x 48 heads] = cache_tile (K-major, K = 576) x q~^T
//   U^T [512 latent x 48 heads] += cache_tile^T (MN-major) x P^T
// so the cache is read from HBM once and never transposed.  Softmax runs per
// head, i.e. down a TMEM column (across token lanes), with a lazily updated
// per-head reference max: a cross-lane max is only taken when some logit
// exceeds the reference by more than 2^8 (always on a chunk's first tile).
// Each CTA writes its partial (reference max, sum, U) in fp32; the combine
// kernel merges the chunks of a sequence and applies W_UV.
#pragma once

#include "sm100.cuh"

namespace gmla {
namespace tc_dec {

using namespace sm100;

constexpr int HEADS = 96, HH = 48;        // heads, heads per CTA
constexpr int BT = 64;                     // tokens per tile
constexpr int CHUNK = 1024;                // tokens per split (work item)
constexpr int LAT = 512, WID = 576, NSUB = 9;
constexpr uint32_t QSUB = HH * 128;        // one [48 x 64] bf16 sub-tile of q~ (6 KB)
constexpr uint32_t CSUB = BT * 128;        // one [64 x 64] bf16 sub-tile of the cache (8 KB)
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_C = OFF_Q + NSUB * QSUB;             // 2 stages x 9 sub-tiles
constexpr uint32_t OFF_P = OFF_C + 2 * NSUB * CSUB;         // 2 P^T buffers [64 tokens x 128 B]
constexpr uint32_t OFF_RED = OFF_P + 2 * CSUB;              // float scratch for reductions
constexpr uint32_t OFF_BAR = OFF_RED + 2048;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t TMEM_S = 0, TMEM_U = 128;                // S^T buffers at 0 and 64; U^T blocks at 128 + 48b

enum Bar { QFULL = 0, CFULL = 1, CEMPTY = 3, SFULL = 5, PFULL = 7, PVDONE = 9, DRAIN = 11, NBAR = 12 };

constexpr float kRescaleLog2 = 8.f;
constexpr int kPrefetchAhead = 3;          // tiles brought into L2 beyond the two stages

struct SplitParams {
  int n_seq, NS;
  const int* offs;          // [n_seq + 1]
  float scale_log2;         // log2(e) / sqrt(192)
  float* part_ml;           // [n][NS][96][2]: reference max (raw logit units), sum
  float* part_u;            // [n][NS][96][512]
};

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])),
        "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
        "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
        "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
      : "memory");
}
// 48 consecutive TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld48(uint32_t taddr, float (&v)[48]) {
  tmem_ld16(taddr, v);
  tmem_ld16(taddr + 16, v + 16);
  tmem_ld16(taddr + 32, v + 32);
}
__device__ __forceinline__ void tmem_st48(uint32_t taddr, const float (&v)[48]) {
  tmem_st16(taddr, v);
  tmem_st16(taddr + 16, v + 16);
  tmem_st16(taddr + 32, v + 32);
}
// Named barrier over the four softmax warps only.
__device__ __forceinline__ void softmax_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__global__ void __launch_bounds__(192, 1)
decode_split_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmC, SplitParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  float* red = reinterpret_cast<float*>(smem_raw + (sbase - sraw) + OFF_RED);   // [4][48] + m[48] + corr[48] + flags
  float* sm_m = red + 4 * HH;
  float* sm_corr = sm_m + HH;
  int* sm_flag = reinterpret_cast<int*>(sm_corr + HH);
  volatile int* abort = &abort_flag;
  auto bar = [&](int i) { return sbase + OFF_BAR + 8u * (uint32_t)i; };

  const int hh = blockIdx.x, split = blockIdx.y, seq = blockIdx.z;
  const int beg = p.offs[seq], L = p.offs[seq + 1] - beg;
  const int t0 = split * CHUNK;
  if (t0 >= L) return;                                   // whole CTA: no work in this chunk
  const int len = min(CHUNK, L - t0);
  const int nt = (len + BT - 1) / BT;
  const int row0 = beg + t0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) abort_flag = device_error_pending() ? 1 : 0;
  __syncthreads();
  if (abort_flag) return;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NBAR; ++i) mbar_init(bar(i), (i == PFULL || i == PFULL + 1) ? 128 : 1);
    fence_mbar_init();
  }
  if (threadIdx.x < HH) sm_m[threadIdx.x] = -INFINITY;
  if (warp == 5) { tmem_alloc(smem_u32(&tmem_slot), 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  // Window of tile j inside the chunk: rows [ws, ws + 64) relative to row0,
  // shifted back for the last tile so that no row past the chunk's end is read.
  auto window = [&](int j) { return min(j * BT, len - BT); };

  if (warp == 4) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmC);
      mbar_arrive_expect_tx(bar(QFULL), NSUB * QSUB);
      for (int k = 0; k < NSUB; ++k)
        tma_load_2d(sbase + OFF_Q + k * QSUB, &tmQ, bar(QFULL), 64 * k, seq * HEADS + hh * HH);
      // Only two 72 KB stages fit next to q~, so the tiles after them are
      // pulled into L2 ahead of time: the stage loads then wait on L2, not HBM.
      auto prefetch = [&](int j) {
        if (j < nt)
          for (int k = 0; k < NSUB; ++k) tma_prefetch_l2_2d(&tmC, 64 * k, row0 + window(j));
      };
      for (int j = 2; j < 2 + kPrefetchAhead; ++j) prefetch(j);
      int issued = 0;
      for (int j = 0; j < nt; ++j) {
        const uint32_t st = j & 1, ph = (j >> 1) & 1;
        if (!mbar_wait(bar(CEMPTY + st), ph ^ 1u, abort)) break;
        prefetch(j + 2 + kPrefetchAhead);
        mbar_arrive_expect_tx(bar(CFULL + st), NSUB * CSUB);
        const int r = row0 + window(j);
        for (int k = 0; k < NSUB; ++k)
          tma_load_2d(sbase + OFF_C + st * NSUB * CSUB + k * CSUB, &tmC, bar(CFULL + st), 64 * k, r);
        ++issued;
      }
      mbar_wait_drain(bar(QFULL), 0);
      for (int j = (issued > 2 ? issued - 2 : 0); j < issued; ++j) mbar_wait_drain(bar(CFULL + (j & 1)), (j >> 1) & 1);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t idQK = idesc_bf16_f32(64, HH, false, false);   // cache (K-major) x q~ (K-major)
      constexpr uint32_t idPV = idesc_bf16_f32(128, HH, true, true);    // cache^T (MN-major) x P^T (MN-major)
      auto issue_qk = [&](int j) {
        const uint32_t cst = sbase + OFF_C + (j & 1) * NSUB * CSUB;
        const uint32_t d = tmem + TMEM_S + (uint32_t)(j & 1) * 64u;
#pragma unroll
        for (int k = 0; k < NSUB; ++k)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(d, sdesc_sw128(cst + k * CSUB + kk * 32, 16, 1024), sdesc_sw128(sbase + OFF_Q + k * QSUB + kk * 32, 16, 1024),
                   idQK, (k | kk) != 0);
        mma_commit(bar(SFULL + (j & 1)));
      };
      // Event loop: issue the score product of tile j+1 as soon as its data
      // lands and the P.V product of tile j as soon as its P^T is written,
      // in whichever order they become ready, so that a slow load of tile
      // j+1 never holds back P.V of tile j (which frees a stage for loads).
      bool ok = mbar_wait(bar(QFULL), 0, abort);
      if (ok) ok = mbar_wait(bar(CFULL), 0, abort);
      if (ok) { tc_fence_after(); issue_qk(0); }
      int next_qk = 1;                                  // next tile whose score product is pending
      uint64_t t_start = 0;
      for (int j = 0; ok && j < nt;) {
        bool progressed = false;
        if (next_qk < nt && next_qk <= j + 1 &&
            mbar_try_wait(bar(CFULL + (next_qk & 1)), (next_qk >> 1) & 1)) {
          tc_fence_after();
          issue_qk(next_qk++);
          progressed = true;
        }
        if (next_qk > j && mbar_try_wait(bar(PFULL + (j & 1)), (j >> 1) & 1)) {
          tc_fence_after();
          const uint32_t cst = sbase + OFF_C + (j & 1) * NSUB * CSUB;
          const uint32_t pb = sbase + OFF_P + (j & 1) * CSUB;
#pragma unroll
          for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tmem + TMEM_U + 48u * b, sdesc_sw128(cst + (2 * b) * CSUB + kk * 2048, CSUB, 1024),
                     sdesc_sw128(pb + kk * 2048, CSUB, 1024), idPV, (j > 0 || kk > 0));
          mma_commit(bar(PVDONE + (j & 1)));
          mma_commit(bar(CEMPTY + (j & 1)));
          ++j;
          progressed = true;
        }
        if (progressed) { t_start = 0; continue; }
        if (*abort || device_error_pending()) { *abort = 1; ok = false; break; }
        const uint64_t now = globaltimer_ns();
        if (t_start == 0) t_start = now;
        else if (now - t_start > kWaitLimitNs) { raise_device_error(GMLA_ETIMEOUT); *abort = 1; ok = false; }
      }
      mma_commit(bar(DRAIN));
      mbar_wait_drain(bar(DRAIN), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax (warps 0-3)
    const float c = p.scale_log2;
    const float thr_add = kRescaleLog2 / c;             // reference max may lag the true max by this much
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const int r = warp * 16 + lane;                     // token row of this thread (lanes 0-15)
    float lsum[HH];
#pragma unroll
    for (int h = 0; h < HH; ++h) lsum[h] = 0.f;
    // A failed (timed-out) wait turns `ok` off for the rest of the kernel; the
    // four warps still walk through every named barrier below in the same
    // order (they never leave the loop), so none is left waiting at one.
    bool ok = true;
    auto wait_warp = [&](int i, uint32_t ph) {
      const bool w = ok && mbar_wait(bar(i), ph, abort);
      ok = __all_sync(0xffffffffu, w) != 0;
      return ok;
    };
    for (int j = 0; j < nt; ++j) {
      float s[HH];
      if (wait_warp(SFULL + (j & 1), (j >> 1) & 1)) {
        tc_fence_after();
        tmem_ld48(tmem + lane_off + TMEM_S + (uint32_t)(j & 1) * 64u, s);
        tmem_wait_ld();
      }
      const int ws = window(j);
      const int tok = ws + r;                            // token index inside the chunk
      const bool valid = ok && lane < 16 && tok >= j * BT && tok < len;
      bool ex = false;
#pragma unroll
      for (int h = 0; h < HH; ++h) {
        s[h] = valid ? s[h] : -INFINITY;
        ex |= s[h] > sm_m[h] + thr_add;
      }
      const int vote = __any_sync(0xffffffffu, ex);
      if (lane == 0) sm_flag[warp] = vote;
      softmax_sync();
      const bool any = (sm_flag[0] | sm_flag[1] | sm_flag[2] | sm_flag[3]) != 0;
      softmax_sync();                                    // flags read before they are rewritten
      if (any) {
        // Exact per-head max of this tile (down the token lanes), then move
        // the reference of every head whose new logits passed it.
#pragma unroll
        for (int h = 0; h < HH; ++h) {
          float v = s[h];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
          if (lane == 0) red[warp * HH + h] = v;
        }
        softmax_sync();
        if (threadIdx.x < HH) {
          const int h = threadIdx.x;
          const float tmax = fmaxf(fmaxf(red[h], red[HH + h]), fmaxf(red[2 * HH + h], red[3 * HH + h]));
          const float m_old = sm_m[h];
          const float m_new = (tmax > m_old + thr_add) ? tmax : m_old;
          sm_corr[h] = (m_new == m_old) ? 1.f : ex2((m_old - m_new) * c);
          sm_m[h] = m_new;
        }
        softmax_sync();
        // U must hold every product issued so far before it is rescaled.
        if (j > 0 && wait_warp(PVDONE + ((j - 1) & 1), ((j - 1) >> 1) & 1)) {
          tc_fence_after();
#pragma unroll 1
          for (int b = 0; b < 4; ++b) {
            float u[HH];
            const uint32_t ua = tmem + lane_off + TMEM_U + 48u * b;
            tmem_ld48(ua, u);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < HH; ++h) u[h] *= sm_corr[h];
            tmem_st48(ua, u);
          }
          tmem_wait_st();
        }
#pragma unroll
        for (int h = 0; h < HH; ++h) lsum[h] *= sm_corr[h];
      }
      // P^T buffer (j & 1) was last read by the product of tile j - 2.
      const bool pfree = (j < 2) ? ok : wait_warp(PVDONE + (j & 1), ((j - 2) >> 1) & 1);
      if (pfree && lane < 16) {
        const uint32_t prow = sbase + OFF_P + (uint32_t)(j & 1) * CSUB + (uint32_t)r * 128u;
#pragma unroll
        for (int cc = 0; cc < HH / 8; ++cc) {
          float e[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int h = cc * 8 + q;
            e[q] = ex2(fmaf(s[h], c, -sm_m[h] * c));
            lsum[h] += e[q];
          }
          st_shared_v4(prow + ((uint32_t)(cc ^ (r & 7)) << 4), pack_bf16x2(e[0], e[1]), pack_bf16x2(e[2], e[3]),
                       pack_bf16x2(e[4], e[5]), pack_bf16x2(e[6], e[7]));
        }
      }
      if (ok) {
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(PFULL + (j & 1)));
      }
      softmax_sync();                                    // sm_m is reused by the next tile
    }
    const bool done = wait_warp(PVDONE + ((nt - 1) & 1), ((nt - 1) >> 1) & 1);
    tc_fence_after();
    // Sum of the exponentials per head over every token lane.
#pragma unroll
    for (int h = 0; h < HH; ++h) {
      float v = lsum[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) red[warp * HH + h] = v;
    }
    softmax_sync();
    const int all_done = (int)done;
    if (lane == 0) sm_flag[warp] = all_done;
    softmax_sync();
    if (sm_flag[0] & sm_flag[1] & sm_flag[2] & sm_flag[3]) {
      const size_t pbase = ((size_t)seq * p.NS + split) * HEADS + hh * HH;
      if (threadIdx.x < HH) {
        const int h = threadIdx.x;
        p.part_ml[(pbase + h) * 2 + 0] = sm_m[h];
        p.part_ml[(pbase + h) * 2 + 1] = red[h] + red[HH + h] + red[2 * HH + h] + red[3 * HH + h];
      }
#pragma unroll 1
      for (int b = 0; b < 4; ++b) {
        float u[HH];
        tmem_ld48(tmem + lane_off + TMEM_U + 48u * b, u);
        tmem_wait_ld();
        const int l = 128 * b + warp * 32 + lane;        // latent index of this lane
#pragma unroll
        for (int h = 0; h < HH; ++h) p.part_u[(pbase + h) * LAT + l] = u[h];
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

// ---------------------------------------------------------------------------
// Warp-level bf16 MMA (m16n8k16, fp32 accumulate) for the two small products
// around the split kernel: the absorbed query and the W_UV projection.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t ld_u32(const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); }
__device__ __forceinline__ uint32_t pack2(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}

__device__ __forceinline__ uint32_t lds32(const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); }
__device__ __forceinline__ void ldsm_x2_trans(uint32_t& r0, uint32_t& r1, const __nv_bfloat16* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1) : "r"(smem_u32(p)));
}

constexpr int ABS_SEQ = 64;                    // sequences per absorb block
constexpr int LDK = 136;                       // padded bf16 row of a 128-wide staged operand
constexpr size_t ABS_SMEM = (size_t)(LAT + ABS_SEQ) * LDK * 2;

// q~[i][h] = [q^C_h W_UK,h^T | q^S_h] in bf16.  Block = (head h, 64 sequences),
// 8 warps.  W_UK,h (512 x 128, one 256-byte row segment per latent index)
// and the block's q^C rows are staged in shared memory with 16-byte loads;
// warp w computes latent columns [64w, 64w + 64).
__global__ void __launch_bounds__(256) absorb_kernel(int n_seq, const __nv_bfloat16* __restrict__ q,
                                                     const __nv_bfloat16* __restrict__ W_UKV,
                                                     __nv_bfloat16* __restrict__ q_abs) {
  extern __shared__ __align__(16) uint8_t asm_[];
  __nv_bfloat16* Ws = reinterpret_cast<__nv_bfloat16*>(asm_);      // [512][LDK]: W_UK,h[latent][k]
  __nv_bfloat16* As = Ws + LAT * LDK;                               // [64][LDK]: q^C[i][k]
  const int h = blockIdx.x, i0 = blockIdx.y * ABS_SEQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  constexpr size_t ldw = (size_t)HEADS * 256;
  for (int e = threadIdx.x; e < LAT * 16; e += blockDim.x) {
    const int n = e >> 4, c = e & 15;
    cp_async16(Ws + n * LDK + c * 8, W_UKV + (size_t)n * ldw + (size_t)h * 256 + c * 8);
  }
  for (int e = threadIdx.x; e < ABS_SEQ * 16; e += blockDim.x) {
    const int r = e >> 4, c = e & 15, i = i0 + r;
    if (i < n_seq) cp_async16(As + r * LDK + c * 8, q + ((size_t)i * HEADS + h) * 192 + c * 8);
    else *reinterpret_cast<uint4*>(As + r * LDK + c * 8) = make_uint4(0u, 0u, 0u, 0u);
  }
  cp_async_wait_all();
  __syncthreads();
#pragma unroll 1
  for (int mt = 0; mt < ABS_SEQ / 16; ++mt) {
    float acc[8][4] = {};
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int k0 = kk * 16 + 2 * t;
      const __nv_bfloat16* ar = As + (mt * 16 + g) * LDK + k0;
      const uint32_t a[4] = {lds32(ar), lds32(ar + 8 * LDK), lds32(ar + 8), lds32(ar + 8 * LDK + 8)};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const __nv_bfloat16* br = Ws + (warp * 64 + nt * 8 + g) * LDK + k0;
        mma16816(acc[nt], a, lds32(br), lds32(br + 8));
      }
    }
    const int ra = i0 + mt * 16 + g, rb = ra + 8;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int col = warp * 64 + nt * 8 + 2 * t;
      if (ra < n_seq)
        *reinterpret_cast<__nv_bfloat162*>(q_abs + ((size_t)ra * HEADS + h) * WID + col) = __floats2bfloat162_rn(acc[nt][0], acc[nt][1]);
      if (rb < n_seq)
        *reinterpret_cast<__nv_bfloat162*>(q_abs + ((size_t)rb * HEADS + h) * WID + col) = __floats2bfloat162_rn(acc[nt][2], acc[nt][3]);
    }
  }
  // q^S passes through unchanged: 64 values = 8 x 16 bytes per sequence.
  for (int e = threadIdx.x; e < ABS_SEQ * 8; e += blockDim.x) {
    const int i = i0 + (e >> 3), c = e & 7;
    if (i < n_seq)
      *reinterpret_cast<uint4*>(q_abs + ((size_t)i * HEADS + h) * WID + LAT + c * 8) =
          *reinterpret_cast<const uint4*>(q + ((size_t)i * HEADS + h) * 192 + 128 + c * 8);
  }
}

constexpr int CMB_SEQ = 32;                    // sequences per combine block
constexpr int LDU = LAT + 8;                   // padded bf16 row of the merged latent tile

// Merge the chunks of each sequence for head h, normalise, and project with
// W_UV,h.  Block = (head h, 32 sequences), 8 warps; warp w owns output
// columns [16w, 16w + 16).  W_UV,h (512 x 128, row-major) is staged in shared
// memory and fed to the MMA through transposing matrix loads.
__global__ void __launch_bounds__(256) combine_kernel(int n_seq, int NS, const int* __restrict__ offs, float scale_log2,
                                                      const float* __restrict__ part_ml, const float* __restrict__ part_u,
                                                      const __nv_bfloat16* __restrict__ W_UKV,
                                                      const __nv_bfloat16* __restrict__ g, __nv_bfloat16* __restrict__ O) {
  extern __shared__ __align__(16) uint8_t csm[];
  __nv_bfloat16* Wv = reinterpret_cast<__nv_bfloat16*>(csm);                    // [512][LDK]
  __nv_bfloat16* U = Wv + LAT * LDK;                                             // [32][LDU]
  float* wsc = reinterpret_cast<float*>(U + CMB_SEQ * LDU);                      // [32][NS]
  int* nsv = reinterpret_cast<int*>(wsc + CMB_SEQ * NS);                         // [32]
  const int h = blockIdx.x, i0 = blockIdx.y * CMB_SEQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, t = lane & 3;
  constexpr size_t ldw = (size_t)HEADS * 256;
  for (int e = threadIdx.x; e < LAT * 16; e += blockDim.x) {
    const int k = e >> 4, c = e & 15;
    cp_async16(Wv + k * LDK + c * 8, W_UKV + (size_t)k * ldw + (size_t)h * 256 + 128 + c * 8);
  }
  // merge weights per (sequence, chunk): w_s = 2^((m_s - M) c) / sum_s l_s 2^((m_s - M) c)
  if (threadIdx.x < CMB_SEQ) {
    const int r = threadIdx.x, i = i0 + r;
    int ns = 0;
    if (i < n_seq) {
      ns = min(NS, (offs[i + 1] - offs[i] + CHUNK - 1) / CHUNK);
      float M = -INFINITY;
      for (int s = 0; s < ns; ++s) M = fmaxf(M, part_ml[(((size_t)i * NS + s) * HEADS + h) * 2]);
      float Ls = 0.f;
      for (int s = 0; s < ns; ++s) {
        const size_t k = (((size_t)i * NS + s) * HEADS + h) * 2;
        const float w = ex2((part_ml[k] - M) * scale_log2);
        wsc[r * NS + s] = w;
        Ls += part_ml[k + 1] * w;
      }
      const float inv = 1.f / Ls;
      for (int s = 0; s < ns; ++s) wsc[r * NS + s] *= inv;
    }
    nsv[r] = ns;
  }
  __syncthreads();
  // merged, normalised latent u[i][:] in bf16: each thread owns 16 groups of
  // four latents (rows r = tid/128 + 2k); the chunk loop is outermost so the
  // 16 loads of one chunk are independent and in flight together.
  constexpr int PER = CMB_SEQ * (LAT / 4) / 256;
  float4 u[PER];
  int maxns = 0;
#pragma unroll
  for (int k = 0; k < PER; ++k) { u[k] = make_float4(0.f, 0.f, 0.f, 0.f); maxns = max(maxns, nsv[(threadIdx.x + 256 * k) / (LAT / 4)]); }
  for (int s = 0; s < maxns; ++s) {
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int e = threadIdx.x + 256 * k, r = e / (LAT / 4), l = (e % (LAT / 4)) * 4, i = i0 + r;
      if (s < nsv[r]) {
        const float w = wsc[r * NS + s];
        const float4 v = *reinterpret_cast<const float4*>(part_u + (((size_t)i * NS + s) * HEADS + h) * LAT + l);
        u[k].x = fmaf(v.x, w, u[k].x); u[k].y = fmaf(v.y, w, u[k].y);
        u[k].z = fmaf(v.z, w, u[k].z); u[k].w = fmaf(v.w, w, u[k].w);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int e = threadIdx.x + 256 * k, r = e / (LAT / 4), l = (e % (LAT / 4)) * 4;
    __nv_bfloat162* d = reinterpret_cast<__nv_bfloat162*>(U + r * LDU + l);
    d[0] = __floats2bfloat162_rn(u[k].x, u[k].y);
    d[1] = __floats2bfloat162_rn(u[k].z, u[k].w);
  }
  cp_async_wait_all();
  __syncthreads();
  // O[i][h][:] = u W_UV,h  (M = 32 sequences, N = 128, K = 512)
  float acc[2][2][4] = {};
#pragma unroll 4
  for (int kk = 0; kk < LAT / 16; ++kk) {
    const int k0 = kk * 16;
    uint32_t bf[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
      ldsm_x2_trans(bf[nt][0], bf[nt][1], Wv + (k0 + (lane & 15)) * LDK + warp * 16 + nt * 8);
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      const __nv_bfloat16* ar = U + (mt * 16 + gq) * LDU + k0 + 2 * t;
      const uint32_t a[4] = {lds32(ar), lds32(ar + 8 * LDU), lds32(ar + 8), lds32(ar + 8 * LDU + 8)};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) mma16816(acc[mt][nt], a, bf[nt][0], bf[nt][1]);
    }
  }
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int i = i0 + mt * 16 + gq + 8 * hr;
        if (i >= n_seq) continue;
        const int col = warp * 16 + nt * 8 + 2 * t;
        const size_t idx = ((size_t)i * HEADS + h) * 128 + col;
        float o0 = acc[mt][nt][2 * hr], o1 = acc[mt][nt][2 * hr + 1];
        if (g) {
          const float2 gv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(g + idx));
          o0 *= 1.f / (1.f + __expf(-gv.x));
          o1 *= 1.f / (1.f + __expf(-gv.y));
        }
        *reinterpret_cast<__nv_bfloat162*>(O + idx) = __floats2bfloat162_rn(o0, o1);
      }
}

inline size_t combine_smem(int NS) { return (size_t)LAT * LDK * 2 + (size_t)CMB_SEQ * LDU * 2 + (size_t)CMB_SEQ * NS * 4 + CMB_SEQ * 4; }

inline int splits(int max_len) { return (max_len + CHUNK - 1) / CHUNK; }

inline size_t workspace_bytes(int n, int max_len) {
  auto al = [](size_t x) { return (x + 1023) & ~(size_t)1023; };
  const size_t ns = splits(max_len);
  return al((size_t)n * HEADS * WID * 2) + al((size_t)n * ns * HEADS * 2 * 4) + al((size_t)n * ns * HEADS * LAT * 4);
}

}  // namespace tc_dec
}  // namespace gmla
