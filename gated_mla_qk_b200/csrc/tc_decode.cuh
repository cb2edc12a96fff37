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
// Heads sit on the MMA's M side (48 heads as an M = 64 tile, half the TMEM
// lanes), tokens on N:
//   S [48 heads x 64 tokens] = q~ (A, resident in TMEM) x cache_tile^T (B, K-major)
//   U [48 heads x 512]      += P (A, smem) x cache_tile (B, MN-major)
// so the 64-token tile of the latent cache, streamed through three 72 KB TMA
// stages, is the only operand read from shared memory by the score product,
// and the same 128B-swizzled tile serves both products.  q~ and S live in the
// upper half of each TMEM sub-partition, U in the lower half.  Softmax is per
// row (one head per thread) with a lazily updated reference max; a row of U
// is rescaled only when its max grows by more than 2^8, and only while no
// product of this CTA is in flight.  Each CTA writes its partial (reference
// max, sum, U) in fp32; the combine kernel merges the chunks and applies W_UV.
#pragma once

#include "sm100.cuh"

namespace gmla {
namespace tc_dec {

using namespace sm100;

constexpr int HEADS = 96, HH = 48;        // heads, heads per CTA (an M = 64 tile with 16 idle rows)
constexpr int BT = 64;                     // tokens per tile (N of the score product)
constexpr int CHUNK = 1024;                // tokens per split (work item)
constexpr int LAT = 512, WID = 576, NSUB = 9, NSTAGE = 3;
constexpr uint32_t CSUB = BT * 128;        // one [64 tokens x 64] bf16 sub-tile of the cache (8 KB)
constexpr uint32_t STAGE = NSUB * CSUB;    // 72 KB
constexpr uint32_t OFF_C = 0;
constexpr uint32_t OFF_P = OFF_C + NSTAGE * STAGE;          // P [64 head rows x 128 B]
constexpr uint32_t OFF_BAR = OFF_P + CSUB;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
// TMEM columns.  Upper lanes (0-15 of each sub-partition): q~ as the A operand
// (576 bf16 = 288 columns) and two S buffers; lower lanes (16-31): U.
constexpr uint32_t TM_Q = 0, TM_S = 288, TM_U = 0;
constexpr uint32_t LANE_LO = 16u << 16;   // lane offset of the lower half

enum Bar { CFULL = 0, CEMPTY = CFULL + NSTAGE, SFULL = CEMPTY + NSTAGE, PFULL = SFULL + 2, PVDONE = PFULL + 1,
           QREADY = PVDONE + 1, DRAIN = QREADY + 1, NBAR = DRAIN + 1 };

constexpr float kRescaleLog2 = 8.f;
constexpr int kPrefetchAhead = 2;          // tiles brought into L2 beyond the stages

struct SplitParams {
  int n_seq, NS;
  const int* offs;                 // [n_seq + 1]
  const __nv_bfloat16* q_abs;      // [n][96][576]
  float scale_log2;                // log2(e) / sqrt(192)
  float* part_ml;                  // [n][NS][96][2]: reference max (raw logit units), sum
  float* part_u;                   // [n][NS][96][512]
};

__global__ void __launch_bounds__(192, 1)
decode_split_kernel(const __grid_constant__ CUtensorMap tmC, SplitParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
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
    for (int i = 0; i < NBAR; ++i) mbar_init(bar(i), (i == PFULL || i == QREADY) ? 128 : 1);
    fence_mbar_init();
  }
  if (warp == 5) { tmem_alloc(smem_u32(&tmem_slot), 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  // Rows [ws, ws + 64) of tile j relative to row0; the last tile is shifted
  // back so that no row past the chunk's end is read.
  auto window = [&](int j) { return min(j * BT, len - BT); };

  if (warp == 4) {
    if (lane == 0) {
      tma_prefetch_desc(&tmC);
      auto prefetch = [&](int j) {
        if (j < nt)
          for (int k = 0; k < NSUB; ++k) tma_prefetch_l2_2d(&tmC, 64 * k, row0 + window(j));
      };
      for (int j = NSTAGE; j < NSTAGE + kPrefetchAhead; ++j) prefetch(j);
      int issued = 0;
      for (int j = 0; j < nt; ++j) {
        const uint32_t st = j % NSTAGE, ph = (j / NSTAGE) & 1;
        if (!mbar_wait(bar(CEMPTY + st), ph ^ 1u, abort)) break;
        prefetch(j + NSTAGE + kPrefetchAhead);
        mbar_arrive_expect_tx(bar(CFULL + st), STAGE);
        const int r = row0 + window(j);
        for (int k = 0; k < NSUB; ++k)
          tma_load_2d(sbase + OFF_C + st * STAGE + k * CSUB, &tmC, bar(CFULL + st), 64 * k, r);
        ++issued;
      }
      for (int j = (issued > NSTAGE ? issued - NSTAGE : 0); j < issued; ++j)
        mbar_wait_drain(bar(CFULL + j % NSTAGE), (j / NSTAGE) & 1);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t idQK = idesc_bf16_f32(64, BT, false, false);    // q~ (TMEM) x cache tile (K-major)
      constexpr uint32_t idPV = idesc_bf16_f32(64, 256, false, true);    // P (K-major) x cache tile (MN-major)
      auto issue_qk = [&](int j) {
        const uint32_t cst = sbase + OFF_C + (j % NSTAGE) * STAGE;
        const uint32_t d = tmem + TM_S + (uint32_t)(j & 1) * 64u;
#pragma unroll
        for (int i = 0; i < 4 * NSUB; ++i)
          mma_ts(d, tmem + TM_Q + 8u * i, sdesc_sw128(cst + (i >> 2) * CSUB + (i & 3) * 32, 16, 1024), idQK, i != 0);
        mma_commit(bar(SFULL + (j & 1)));
      };
      // Event loop: issue the score product of a tile as soon as its data has
      // landed (and its S buffer is free), and the P.V product of tile j as
      // soon as P is written, in whichever order they become ready.
      bool ok = mbar_wait(bar(QREADY), 0, abort);
      int next_qk = 0;
      uint64_t t_start = 0;
      for (int j = 0; ok && j < nt;) {
        bool progressed = false;
        if (next_qk < nt && next_qk <= j + 1 &&
            mbar_test(bar(CFULL + next_qk % NSTAGE), (next_qk / NSTAGE) & 1)) {
          tc_fence_after();
          issue_qk(next_qk++);
          progressed = true;
        }
        if (next_qk > j && mbar_test(bar(PFULL), j & 1)) {
          tc_fence_after();
          const uint32_t cst = sbase + OFF_C + (j % NSTAGE) * STAGE;
#pragma unroll
          for (int kk = 0; kk < BT / 16; ++kk)
#pragma unroll
            for (int nh = 0; nh < 2; ++nh)
              mma_ss(tmem + LANE_LO + TM_U + 256u * nh, sdesc_sw128(sbase + OFF_P + kk * 32, 16, 1024),
                     sdesc_sw128(cst + (4 * nh) * CSUB + kk * 2048, CSUB, 1024), idPV, (j > 0 || kk > 0));
          mma_commit(bar(PVDONE));
          mma_commit(bar(CEMPTY + j % NSTAGE));
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
    // Lanes 0-15 of warp w own head rows 16w + lane (upper TMEM lanes: q~, S);
    // lanes 16-31 hold the U rows of the same heads (lower TMEM lanes).
    const float c = p.scale_log2;
    const float thr_add = kRescaleLog2 / c;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const bool upper = lane < 16;
    const int hr = warp * 16 + (lane & 15);              // head row inside the CTA (valid if < 48)
    const bool head_ok = hr < HH;
    // Load q~ into the upper TMEM lanes (the lower lanes write zeros into the
    // U columns, which the first P.V product overwrites).
    {
      const uint4* src = reinterpret_cast<const uint4*>(p.q_abs + ((size_t)seq * HEADS + hh * HH + (head_ok ? hr : 0)) * WID);
#pragma unroll 1
      for (int cch = 0; cch < 9; ++cch) {
        float v[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          uint4 x = make_uint4(0u, 0u, 0u, 0u);
          if (upper && head_ok) x = src[cch * 8 + q];
          v[4 * q + 0] = __uint_as_float(x.x); v[4 * q + 1] = __uint_as_float(x.y);
          v[4 * q + 2] = __uint_as_float(x.z); v[4 * q + 3] = __uint_as_float(x.w);
        }
        tmem_st32(tmem + lane_off + TM_Q + 32u * cch, v);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(QREADY));
    }
    float m_used = -INFINITY, lsum = 0.f;
    bool ok = true;
    auto wait_warp = [&](int i, uint32_t ph) {
      const bool w = ok && mbar_wait(bar(i), ph, abort);
      ok = __all_sync(0xffffffffu, w) != 0;
      return ok;
    };
    for (int j = 0; j < nt && ok; ++j) {
      if (!wait_warp(SFULL + (j & 1), (j >> 1) & 1)) break;
      tc_fence_after();
      float s[BT];
      tmem_ld32(tmem + lane_off + TM_S + (uint32_t)(j & 1) * 64u, *reinterpret_cast<float(*)[32]>(&s[0]));
      tmem_ld32(tmem + lane_off + TM_S + (uint32_t)(j & 1) * 64u + 32u, *reinterpret_cast<float(*)[32]>(&s[32]));
      tmem_wait_ld();
      const int ws = window(j);
      float pm[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) pm[q] = -INFINITY;
#pragma unroll
      for (int k = 0; k < BT; ++k) {
        const int tok = ws + k;
        s[k] = (upper && tok >= j * BT && tok < len) ? s[k] : -INFINITY;
        pm[k & 7] = fmaxf(pm[k & 7], s[k]);
      }
      const float mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])), fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
      const bool need = upper && head_ok && mx > m_used + thr_add;     // first tile: m_used = -inf
      const float m_new = need ? mx : m_used;
      const float corr = need ? ex2((m_used - m_new) * c) : 1.f;       // 0 on the first tile
      // P buffer and U: the previous product must have finished.
      if (j > 0 && !wait_warp(PVDONE, (j - 1) & 1)) break;
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // Rare: rescale this warp's U rows.  No product of this CTA is in
        // flight once the score product of tile j+1 (if issued) is done,
        // because P.V of tile j waits for this warp's arrival below.
        if (j + 1 < nt && !wait_warp(SFULL + ((j + 1) & 1), ((j + 1) >> 1) & 1)) break;
        tc_fence_after();
        const float f = __shfl_sync(0xffffffffu, corr, lane & 15);   // lower lane takes its head's factor
#pragma unroll 1
        for (int cch = 0; cch < LAT / 32; ++cch) {
          float u[32];
          tmem_ld32(tmem + lane_off + TM_U + 32u * cch, u);
          tmem_wait_ld();
          if (!upper) {
#pragma unroll
            for (int e = 0; e < 32; ++e) u[e] *= f;
          }
          tmem_st32(tmem + lane_off + TM_U + 32u * cch, u);
        }
        tmem_wait_st();
      }
      lsum *= corr;
      m_used = m_new;
      if (upper) {
        // Rows of the 16 idle heads (48-63) get P = 0.
        const float neg = head_ok ? -m_used * c : 0.f;
        const uint32_t prow = sbase + OFF_P + (uint32_t)hr * 128u;
        float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          float e[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            e[q] = head_ok ? ex2(fmaf(s[8 * cc + q], c, neg)) : 0.f;
            ps[q] += e[q];
          }
          st_shared_v4(prow + ((uint32_t)(cc ^ (hr & 7)) << 4), pack_bf16x2(e[0], e[1]), pack_bf16x2(e[2], e[3]),
                       pack_bf16x2(e[4], e[5]), pack_bf16x2(e[6], e[7]));
        }
        lsum += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(PFULL));
    }
    if (ok && wait_warp(PVDONE, (nt - 1) & 1)) {
      tc_fence_after();
      const size_t pbase = ((size_t)seq * p.NS + split) * HEADS + hh * HH;
      if (upper && head_ok) {
        p.part_ml[(pbase + hr) * 2 + 0] = m_used;
        p.part_ml[(pbase + hr) * 2 + 1] = lsum;
      }
      float* dst = p.part_u + (pbase + (head_ok ? hr : 0)) * LAT;
#pragma unroll 1
      for (int cch = 0; cch < LAT / 32; ++cch) {
        float u[32];
        tmem_ld32(tmem + lane_off + TM_U + 32u * cch, u);
        tmem_wait_ld();
        if (!upper && head_ok) {
          float4* d4 = reinterpret_cast<float4*>(dst + 32 * cch);
#pragma unroll
          for (int q = 0; q < 8; ++q) d4[q] = make_float4(u[4 * q], u[4 * q + 1], u[4 * q + 2], u[4 * q + 3]);
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

// Merge the chunks of each (sequence, head): one warp per pair, 16 latents per
// lane.  u = sum_s U_s 2^((m_s - M) c) / sum_s l_s 2^((m_s - M) c), in bf16.
__global__ void __launch_bounds__(256) merge_kernel(int n_seq, int NS, const int* __restrict__ offs, float scale_log2,
                                                    const float* __restrict__ part_ml, const float* __restrict__ part_u,
                                                    __nv_bfloat16* __restrict__ u_out) {
  const int pair = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (pair >= n_seq * HEADS) return;
  const int i = pair / HEADS, h = pair % HEADS;
  const int ns = min(NS, (offs[i + 1] - offs[i] + CHUNK - 1) / CHUNK);
  float M = -INFINITY;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, part_ml[(((size_t)i * NS + s) * HEADS + h) * 2]);
  float4 acc[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  float Ls = 0.f;
  for (int s = 0; s < ns; ++s) {
    const size_t k = ((size_t)i * NS + s) * HEADS + h;
    const float w = ex2((part_ml[2 * k] - M) * scale_log2);
    Ls += part_ml[2 * k + 1] * w;
    const float4* src = reinterpret_cast<const float4*>(part_u + k * LAT);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = src[lane + 32 * q];
      acc[q].x = fmaf(v.x, w, acc[q].x); acc[q].y = fmaf(v.y, w, acc[q].y);
      acc[q].z = fmaf(v.z, w, acc[q].z); acc[q].w = fmaf(v.w, w, acc[q].w);
    }
  }
  const float inv = 1.f / Ls;
  __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(u_out + ((size_t)i * HEADS + h) * LAT);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int l4 = lane + 32 * q;
    dst[2 * l4] = __floats2bfloat162_rn(acc[q].x * inv, acc[q].y * inv);
    dst[2 * l4 + 1] = __floats2bfloat162_rn(acc[q].z * inv, acc[q].w * inv);
  }
}

constexpr int PRJ_SEQ = 64;                    // sequences per projection block
constexpr int LDU = LAT + 8;                   // padded bf16 row of the staged latent tile
constexpr size_t PRJ_SMEM = (size_t)LAT * LDK * 2 + (size_t)PRJ_SEQ * LDU * 2;

// o[i][h] = u[i][h] W_UV,h (* sigmoid(g)).  Block = (head h, 64 sequences),
// 8 warps; warp w owns output columns [16w, 16w + 16).  W_UV,h (512 x 128,
// row-major) and the block's merged latents are staged with cp.async; W_UV,h
// feeds the MMA through transposing matrix loads.
__global__ void __launch_bounds__(256) project_kernel(int n_seq, const __nv_bfloat16* __restrict__ u_in,
                                                      const __nv_bfloat16* __restrict__ W_UKV,
                                                      const __nv_bfloat16* __restrict__ g, __nv_bfloat16* __restrict__ O) {
  extern __shared__ __align__(16) uint8_t csm[];
  __nv_bfloat16* Wv = reinterpret_cast<__nv_bfloat16*>(csm);                    // [512][LDK]
  __nv_bfloat16* U = Wv + LAT * LDK;                                             // [64][LDU]
  const int h = blockIdx.x, i0 = blockIdx.y * PRJ_SEQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, t = lane & 3;
  constexpr size_t ldw = (size_t)HEADS * 256;
  for (int e = threadIdx.x; e < LAT * 16; e += blockDim.x) {
    const int k = e >> 4, c = e & 15;
    cp_async16(Wv + k * LDK + c * 8, W_UKV + (size_t)k * ldw + (size_t)h * 256 + 128 + c * 8);
  }
  for (int e = threadIdx.x; e < PRJ_SEQ * (LAT / 8); e += blockDim.x) {
    const int r = e / (LAT / 8), c = e % (LAT / 8), i = i0 + r;
    if (i < n_seq) cp_async16(U + r * LDU + c * 8, u_in + ((size_t)i * HEADS + h) * LAT + c * 8);
    else *reinterpret_cast<uint4*>(U + r * LDU + c * 8) = make_uint4(0u, 0u, 0u, 0u);
  }
  cp_async_wait_all();
  __syncthreads();
  float acc[4][2][4] = {};
#pragma unroll 4
  for (int kk = 0; kk < LAT / 16; ++kk) {
    const int k0 = kk * 16;
    uint32_t bf[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
      ldsm_x2_trans(bf[nt][0], bf[nt][1], Wv + (k0 + (lane & 15)) * LDK + warp * 16 + nt * 8);
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      const __nv_bfloat16* ar = U + (mt * 16 + gq) * LDU + k0 + 2 * t;
      const uint32_t a[4] = {lds32(ar), lds32(ar + 8 * LDU), lds32(ar + 8), lds32(ar + 8 * LDU + 8)};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) mma16816(acc[mt][nt], a, bf[nt][0], bf[nt][1]);
    }
  }
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
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


inline int splits(int max_len) { return (max_len + CHUNK - 1) / CHUNK; }

inline size_t workspace_bytes(int n, int max_len) {
  auto al = [](size_t x) { return (x + 1023) & ~(size_t)1023; };
  const size_t ns = splits(max_len);
  return al((size_t)n * HEADS * WID * 2) + al((size_t)n * ns * HEADS * 2 * 4) + al((size_t)n * ns * HEADS * LAT * 4) +
         al((size_t)n * HEADS * LAT * 2);
}

}  // namespace tc_dec
}  // namespace gmla
