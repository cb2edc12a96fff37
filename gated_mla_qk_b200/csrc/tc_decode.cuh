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
//   o_h  = (u_h / l) W_UV,h  (* sigmoid(g))                  (merge + projection kernel)
//
// Split kernel: a persistent grid of one CTA per SM.  The 96-token tiles of
// all sequences, laid end to end, are cut into equal ranges, one per CTA, so
// every SM streams the same number of cache bytes whatever the length mix; a
// range may end in the middle of one sequence and start in the middle of
// another.  Each (CTA, sequence) piece of a range writes one partial (the
// reference max, sum and U of every head) that the merge kernel combines.
//
// Per 96-token tile, both products run on the tensor core at M = 128:
//   S   [96(+32) heads x 96 tokens] = q~ (A, smem, K-major) x tile^T (B, K-major)
//   U^T [512 latent x 96 heads]    += tile^T (A, smem, MN-major) x P^T (B, K-major)
// All 96 heads share one read of the tile from HBM.  Heads sit on M for the
// score product (one softmax row per thread), the latent sits on M for the
// value product, so U^T takes 4 x 96 TMEM columns beside the 96-column S.
// q~ (108 KB) stays in shared memory for the whole sequence.  The tile's
// latent streams through a ring of four 24 KB slots twice: once, as 128-wide
// latent pairs, for the score product, and once more (from L2, where the
// first pass left it under an evict-last policy) for the value product after
// the softmax, so no slot is held across the softmax and the ring stays short.  The 64 shared-key dims
// are a fifth score-product item of the same ring (in the first half of a
// slot).  P^T's last 32 tokens use a 64-byte swizzle (6 KB instead of 12),
// which is what makes room for the fourth slot.  The score product of tile
// t+1 runs while the softmax of tile t runs; S is released as soon as the
// softmax has loaded it.
// Softmax: base-2 exponentials against a lazily updated reference max per
// head; U^T's column of a head is rescaled only when the head's max grows by
// more than 2^8 (all four softmax warps take part, since a head's column
// spans every TMEM lane).
#pragma once

#include "sm100.cuh"

namespace gmla {
namespace tc_dec {

using namespace sm100;

constexpr int HEADS = 96, BT = 96, LAT = 512, WID = 576;
constexpr int NPS = 4;                     // ring slots (latent pairs; the shared-key dims in half a slot)
constexpr int G_CAP = 256;                 // most split CTAs (one per SM)
constexpr uint32_t CSUB = BT * 128;        // [96 tokens x 64 dims] bf16, 12 KB
constexpr uint32_t PAIR = 2 * CSUB;        // one 128-wide latent pair, 24 KB
constexpr uint32_t QCH = HEADS * 128;      // [96 heads x 64 dims] bf16, 12 KB
constexpr uint32_t OFF_Q = 0;              // q~: 9 chunks of 64 dims
constexpr uint32_t OFF_P = OFF_Q + 9 * QCH;                 // P^T tokens 0-63: [96 heads x 64] 128-byte swizzle
constexpr uint32_t OFF_P2 = OFF_P + QCH;                    // P^T tokens 64-95: [96 heads x 32] 64-byte swizzle
constexpr uint32_t P2_BYTES = HEADS * 64;                   // 6 KB
static_assert(BT == 96, "P^T is laid out as 64 + 32 tokens");
constexpr uint32_t OFF_PAIR = OFF_P2 + P2_BYTES;
constexpr uint32_t OFF_CORR = OFF_PAIR + NPS * PAIR;        // 96 rescale factors
constexpr uint32_t OFF_BAR = OFF_CORR + 512;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t TM_S = 0, TM_U = 128;   // TMEM columns: S (96), U^T 4 x 96
static_assert(OFF_PAIR % 1024 == 0, "ring slots must be 1024-byte aligned (128-byte swizzle)");
static_assert(OFF_P2 % 512 == 0, "the 64-byte swizzled P^T part must be 512-byte aligned");
static_assert(SMEM_BYTES + 64 <= 232448, "decode shared memory exceeds the per-block limit");
// The score product reads 128 rows of each q~ chunk: rows 96-127 fall on the
// next chunk (or on P^T for the last one), and the S rows they give are never
// read.

enum Bar { QFULL = 0, QEMPTY, LFULL, LEMPTY = LFULL + NPS, SFULL = LEMPTY + NPS, SFREE, PFULL, PVDONE, UFREE,
           DRAIN, NBAR };

constexpr float kRescaleLog2 = 8.f;
// Tiles brought into L2 ahead of their first ring load.  One is enough; at
// three the prefetched lines evicted the ones the second pass over a tile re-reads.
constexpr int kPrefetchAhead = 1;

// The cache rows each query attends to.  Decode: sequence i owns the packed
// rows offs[i] .. offs[i+1]-1.  Prefill on the latent cache (prefix_T > 0):
// query i = b * prefix_T + t attends to rows b * prefix_T .. b * prefix_T + t,
// its own causal prefix.
struct Windows {
  const int* offs;                 // [n_seq + 1] (decode)
  int prefix_T;                    // > 0: prefill, sequence length
  __device__ int start(int i) const { return prefix_T > 0 ? (i / prefix_T) * prefix_T : offs[i]; }
  __device__ int len(int i) const { return prefix_T > 0 ? i % prefix_T + 1 : offs[i + 1] - offs[i]; }
};

struct SplitParams {
  int n_seq, G;
  Windows win;
  const __nv_bfloat16* cache;      // [rows][576]
  const int* plan;                 // [n_seq + 1] tile prefix, then [G] first sequence of each CTA
  float scale_log2;                // log2(e) / sqrt(192)
  float* part_ml;                  // [G + n_seq][96][2]: reference max (raw logit units), sum
  float* part_u;                   // [G + n_seq][96][512]
  float* maxlogit;                 // [96] or nullptr: per-head max of the scaled logits (atomic max)
  float scale;                     // 1 / sqrt(192)
};

// Walks the tiles of a CTA's range: sequence i, tile k of it.  The tile's
// BT-row window ends at the sequence's end when the tile is the last one, so
// no row past the sequence (or the cache) is read; rows before the sequence
// are masked (and rows before the cache read as zero).  A sequence with an
// empty cache has no tiles and is stepped over (the merge writes its zeros).
struct TileCursor {
  Windows win;
  int n, i, k, nti, L, start;
  __device__ void load(int seq) {
    while (seq < n && win.len(seq) == 0) ++seq;
    i = seq;
    if (seq < n) { start = win.start(seq); L = win.len(seq); nti = (L + BT - 1) / BT; }
  }
  __device__ void next() {
    if (++k == nti) { k = 0; load(i + 1); }
  }
  __device__ int wrel() const { return min(k * BT, L - BT); }
  __device__ int row() const { return start + wrel(); }
  __device__ bool last_of_seq() const { return k == nti - 1; }
};

__device__ __forceinline__ void cta_range(const int* plan, int n, int G, int c, int& nt, int& i0, int& k0) {
  const long long N = plan[n];
  const long long t0 = (long long)c * N / G, t1 = (long long)(c + 1) * N / G;
  nt = (int)(t1 - t0);
  i0 = nt > 0 ? plan[n + 1 + c] : 0;
  k0 = nt > 0 ? (int)(t0 - plan[i0]) : 0;
}

__global__ void __launch_bounds__(192, 1)
decode_split_kernel(const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmQ, SplitParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  float* corr_sm = reinterpret_cast<float*>(smem_raw + (sbase - sraw) + OFF_CORR);
  volatile int* abort = &abort_flag;
  auto bar = [&](int i) { return sbase + OFF_BAR + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;

  if (threadIdx.x == 0) abort_flag = device_error_pending() ? 1 : 0;
  __syncthreads();
  if (abort_flag) return;
  __syncthreads();
  // Set-up that reads nothing of the absorb kernel's results, done while that
  // kernel finishes (this grid is launched behind it).
  if (threadIdx.x == 0) {
    for (int i = 0; i < NBAR; ++i) mbar_init(bar(i), (i == PFULL || i == UFREE || i == SFREE) ? 128 : 1);
    fence_mbar_init();
  }
  if (warp == 5) { tmem_alloc(smem_u32(&tmem_slot), 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // q~ and the work plan are the absorb kernel's results.
  griddep_wait();
  griddep_launch_dependents();
  int nt, i0, k0;
  cta_range(p.plan, p.n_seq, p.G, cta, nt, i0, k0);
  if (nt == 0) {                                         // whole CTA: empty range
    if (warp == 5) tmem_dealloc(tmem, 512);
    return;
  }
  auto cursor = [&]() {
    TileCursor cur;
    cur.win = p.win; cur.n = p.n_seq; cur.k = k0;
    cur.load(i0);
    return cur;
  };

  // Ring order (producer and MMA thread walk it alike): the score-product
  // items of tile 0 (four latent pairs, then the shared-key dims); then, per
  // tile t, the score-product items of tile t+1 followed by the value-product
  // pairs of tile t.
  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmC); tma_prefetch_desc(&tmQ);
      TileCursor cq = cursor(), cp = cursor(), pf = cursor();
      int pf_t = 0;
      auto prefetch_upto = [&](int upto) {
        for (; pf_t < upto && pf_t < nt; ++pf_t) {
          // A tile's rows are contiguous in the cache: bulk prefetches.
          const int r0 = max(pf.row(), 0), r1 = pf.row() + BT;
          const uint8_t* src = reinterpret_cast<const uint8_t*>(p.cache + (size_t)r0 * WID);
          for (uint32_t off = 0, n = (uint32_t)(r1 - r0) * WID * 2u; off < n; off += 16384u)
            bulk_prefetch_l2(src + off, min(16384u, n - off));
          pf.next();
        }
      };
      int u = 0, seg = 0;
      bool ok = true;
      // The first pass over a tile keeps its lines in L2 for the second; the
      // second pass is their last use.
      const uint64_t pol_keep = l2_policy_evict_last(), pol_drop = l2_policy_evict_first();
      auto load_pair = [&](int row, int pr, bool second) {
        const uint32_t slot = (uint32_t)(u % NPS);
        if (!mbar_wait(bar(LEMPTY + slot), ((uint32_t)(u / NPS) & 1u) ^ 1u, abort)) { ok = false; return; }
        const uint32_t dst = sbase + OFF_PAIR + slot * PAIR;
        mbar_arrive_expect_tx(bar(LFULL + slot), PAIR);
        const uint64_t pol = second ? pol_drop : pol_keep;
        tma_load_2d_hint(dst, &tmC, bar(LFULL + slot), 128 * pr, row, pol);
        tma_load_2d_hint(dst + CSUB, &tmC, bar(LFULL + slot), 128 * pr + 64, row, pol);
        ++u;
      };
      auto load_rope = [&](int row) {       // the 64 shared-key dims, first half of a slot
        const uint32_t slot = (uint32_t)(u % NPS);
        if (!mbar_wait(bar(LEMPTY + slot), ((uint32_t)(u / NPS) & 1u) ^ 1u, abort)) { ok = false; return; }
        mbar_arrive_expect_tx(bar(LFULL + slot), CSUB);
        tma_load_2d_hint(sbase + OFF_PAIR + slot * PAIR, &tmC, bar(LFULL + slot), LAT, row, pol_drop);   // read once
        ++u;
      };
      auto load_qk = [&](int t) {           // score-product items of tile t (cursor cq at t)
        (void)t;
        const int row = cq.row();
        for (int pr = 0; pr < 4 && ok; ++pr) load_pair(row, pr, false);
        if (ok) load_rope(row);
      };
      prefetch_upto(kPrefetchAhead);
      mbar_arrive_expect_tx(bar(QFULL), 9 * QCH);
      for (int c = 0; c < 9; ++c) tma_load_2d(sbase + OFF_Q + c * QCH, &tmQ, bar(QFULL), 64 * c, cq.i * HEADS);
      load_qk(0);
      for (int t = 0; ok && t < nt; ++t) {
        const bool last = (t == nt - 1) || cq.last_of_seq();      // cq at tile t here
        cq.next();
        if (t + 1 < nt) {
          if (last) {                        // tile t+1 starts another sequence: its q~
            ++seg;
            if (!mbar_wait(bar(QEMPTY), (uint32_t)(seg - 1) & 1u, abort)) { ok = false; break; }
            mbar_arrive_expect_tx(bar(QFULL), 9 * QCH);
            for (int c = 0; c < 9; ++c) tma_load_2d(sbase + OFF_Q + c * QCH, &tmQ, bar(QFULL), 64 * c, cq.i * HEADS);
          }
          load_qk(t + 1);
        }
        const int row = cp.row();
        for (int pr = 0; pr < 4 && ok; ++pr) load_pair(row, pr, true);
        cp.next();
        prefetch_upto(t + 2 + kPrefetchAhead);
      }
      // Never leave with copies in flight into this CTA's shared memory.
      mbar_wait_drain(bar(QFULL), (uint32_t)seg & 1u);
      for (int v = (u > NPS ? u - NPS : 0); v < u; ++v) mbar_wait_drain(bar(LFULL + v % NPS), (uint32_t)(v / NPS) & 1u);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idQK = idesc_bf16_f32(128, BT, false, false);      // q~ (K-major) x tile (K-major)
      constexpr uint32_t idPV = idesc_bf16_f32(128, HEADS, true, false);    // tile^T (MN-major) x P^T (K-major)
      bool ok = true;
      int u = 0;
      auto wait_ok = [&](int b, uint32_t ph) {
        ok = ok && mbar_wait_lean(bar(b), ph, abort);
        if (ok) tc_fence_after();
        return ok;
      };
      // Base descriptors, built once: every MMA below steps one of them by a
      // compile-time byte offset (or picks a ring slot's).
      const uint64_t dQ = sdesc_sw128(sbase + OFF_Q, 16, 1024);
      const uint64_t dP = sdesc_sw128(sbase + OFF_P, 16, 1024);
      const uint64_t dP2 = sdesc_sw64_kmajor(sbase + OFF_P2);
      const uint64_t dRingK = sdesc_sw128(sbase + OFF_PAIR, 16, 1024);     // slot 0, K-major (score B)
      const uint64_t dRingM = sdesc_sw128(sbase + OFF_PAIR, CSUB, 1024);   // slot 0, MN-major (value A)
      int slot_u = 0;                          // u % NPS and (u / NPS) & 1, kept incrementally
      uint32_t ph_u = 0;
      auto next_pair = [&]() -> bool {         // wait for ring item u
        return wait_ok(LFULL + slot_u, ph_u);
      };
      auto release_pair = [&]() {
        mma_commit(bar(LEMPTY + slot_u));
        ++u;
        if (++slot_u == NPS) { slot_u = 0; ph_u ^= 1u; }
      };
      auto qk = [&](int t) {
        const uint32_t d = tmem + TM_S;
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          if (!next_pair()) return;
          const uint64_t sb = sdesc_add(dRingK, (uint32_t)slot_u * PAIR);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(d, sdesc_add(dQ, (uint32_t)(2 * q + hf) * QCH + kk * 32u), sdesc_add(sb, hf * CSUB + kk * 32u), idQK,
                     (q | hf | kk) != 0);
          release_pair();
        }
        (void)t;
        if (!next_pair()) return;              // the shared-key dims
        {
          const uint64_t sb = sdesc_add(dRingK, (uint32_t)slot_u * PAIR);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(d, sdesc_add(dQ, 8u * QCH + kk * 32u), sdesc_add(sb, kk * 32u), idQK, true);
        }
        release_pair();
        mma_commit(bar(SFULL));
      };
      auto pv = [&](bool fresh) {
#pragma unroll 1
        for (int b = 0; b < 4; ++b) {
          if (!next_pair()) return;
          const uint64_t sb = sdesc_add(dRingM, (uint32_t)slot_u * PAIR);
#pragma unroll
          for (int kk = 0; kk < BT / 16; ++kk)     // tokens 16 kk .. 16 kk + 15 of P^T
            mma_ss(tmem + TM_U + (uint32_t)b * HEADS, sdesc_add(sb, kk * 2048u),
                   kk < 4 ? sdesc_add(dP, (uint32_t)kk * 32u) : sdesc_add(dP2, (uint32_t)(kk - 4) * 32u), idPV,
                   !(fresh && kk == 0));
          release_pair();
        }
        mma_commit(bar(PVDONE));
      };
      TileCursor cur = cursor();
      int seg = 0;
      if (wait_ok(QFULL, 0)) {
        qk(0);
        if (ok && ((nt == 1) || cur.last_of_seq())) mma_commit(bar(QEMPTY));
      }
      for (int t = 0; ok && t < nt; ++t) {
        const bool first = (t == 0) || cur.k == 0;
        const bool last = (t == nt - 1) || cur.last_of_seq();
        cur.next();                          // now at tile t+1
        if (t + 1 < nt) {
          if (last && !wait_ok(QFULL, (uint32_t)(seg + 1) & 1u)) break;
          // S is single-buffered: the softmax of tile t must have loaded it.
          if (!wait_ok(SFREE, (uint32_t)t & 1u)) break;
          qk(t + 1);
          if (ok && ((t + 2 == nt) || cur.last_of_seq())) mma_commit(bar(QEMPTY));
        }
        if (!wait_ok(PFULL, (uint32_t)t & 1u)) break;
        if (first && seg > 0 && !wait_ok(UFREE, (uint32_t)(seg - 1) & 1u)) break;
        pv(first);
        if (last) ++seg;
      }
      // Drain every MMA this thread issued before TMEM is released.
      mma_commit(bar(DRAIN));
      mbar_wait_drain(bar(DRAIN), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + partials (warps 0-3)
    // Thread x owns head row x of S (x < 96) and latent row x of each U^T block.
    const int x = threadIdx.x;
    const bool head = x < HEADS;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float c = p.scale_log2;
    const float thr_add = kRescaleLog2 / c;
    float m_used = -INFINITY, l = 0.f, piece_max = -INFINITY;
    bool ok = true;
    TileCursor cur = cursor();
    // The loop runs the same named barriers in every thread whatever
    // happens, so a failed wait can never strand a warp in a barrier.
    for (int t = 0; t < nt; ++t) {
      const bool first = (t == 0) || cur.k == 0;
      const bool last = (t == nt - 1) || cur.last_of_seq();
      if (ok) ok = mbar_wait(bar(SFULL), (uint32_t)t & 1u, abort);
      ok = !bar_red_or(1, 128, !ok);
      float s[BT];
      bool need = false;
      float corr = 1.f, m_new = m_used;
      if (ok) {
        tc_fence_after();
        const uint32_t ts = tmem + lane_off + TM_S;
        static_assert(BT % 32 == 0, "S is loaded in 32-column pieces");
#pragma unroll
        for (int k = 0; k < BT / 32; ++k) tmem_ld32(ts + 32u * k, *reinterpret_cast<float(*)[32]>(&s[32 * k]));
#pragma unroll
        for (int k = 0; k < BT / 32; ++k) tmem_wait_ld_dep(*reinterpret_cast<float(*)[32]>(&s[32 * k]));
        tc_fence_before();
        mbar_arrive(bar(SFREE));             // S may now be overwritten by the next tile's score product
        if (head) {
          const int w = cur.wrel();
          const int lo = cur.k * BT - w, hi = cur.L - w;   // valid columns [lo, hi)
          float pm[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) pm[q] = -INFINITY;
          if (lo == 0 && hi >= BT) {
#pragma unroll
            for (int e = 0; e < BT; ++e) pm[e & 7] = fmaxf(pm[e & 7], s[e]);
          } else {
#pragma unroll
            for (int e = 0; e < BT; ++e) {
              s[e] = (e >= lo && e < hi) ? s[e] : -INFINITY;
              pm[e & 7] = fmaxf(pm[e & 7], s[e]);
            }
          }
          const float mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])), fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
          piece_max = fmaxf(piece_max, mx);
          need = mx > m_used + thr_add;                     // always on a piece's first tile
          m_new = need ? mx : m_used;
          corr = need ? ex2((m_used - m_new) * c) : 1.f;    // 0 on a piece's first tile
          if (!first) corr_sm[x] = corr;
        }
      }
      const bool resc = bar_red_or(1, 128, ok && head && need && !first);
      // Probabilities first, into registers; P^T and U^T are touched only
      // once the value product of tile t-1 has finished with them.
      uint32_t pk[BT / 2];
      if (ok && head) {
        l *= corr;
        m_used = m_new;
        const float neg = -m_used * c;
        float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int e = 0; e < BT; e += 2) {
          const float a0 = ex2(fmaf(s[e], c, neg)), a1 = ex2(fmaf(s[e + 1], c, neg));
          ps[(e >> 1) & 7] += a0 + a1;
          pk[e >> 1] = pack_bf16x2(a0, a1);
        }
        l += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      }
      if (ok && t > 0) {
        bool w = mbar_wait(bar(PVDONE), (uint32_t)(t - 1) & 1u, abort);
        ok = __all_sync(0xffffffffu, w) != 0;
        if (ok) tc_fence_after();
      }
      if (ok && resc) {
        // Rare: scale the U^T columns of the heads whose max moved (the
        // value product of tile t waits for this thread's arrival below).
#pragma unroll 1
        for (int b = 0; b < 4; ++b)
#pragma unroll 1
          for (int cc = 0; cc < 3; ++cc) {
            const uint32_t tu = tmem + lane_off + TM_U + (uint32_t)(b * HEADS + 32 * cc);
            float u[32];
            tmem_ld32(tu, u);
            tmem_wait_ld_dep(u);
#pragma unroll
            for (int e = 0; e < 32; ++e) u[e] *= corr_sm[32 * cc + e];
            tmem_st32(tu, u);
          }
        tmem_wait_st();
      }
      if (ok && head) {
        // P^T row x: tokens 0-63 as a 128-byte row (128-byte swizzle), tokens
        // 64-95 as a 64-byte row (64-byte swizzle).
        const uint32_t prow = sbase + OFF_P + (uint32_t)x * 128u, prow2 = sbase + OFF_P2 + (uint32_t)x * 64u;
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
          st_shared_v4(prow + ((uint32_t)(cc ^ (x & 7)) << 4), pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          st_shared_v4(prow2 + ((uint32_t)(cc ^ ((x >> 1) & 3)) << 4), pk[32 + 4 * cc], pk[33 + 4 * cc], pk[34 + 4 * cc],
                       pk[35 + 4 * cc]);
      }
      if (ok) {
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(PFULL));
      }
      if (last) {
        // End of this CTA's piece of sequence cur.i: write its partial once
        // the value product of tile t has finished.
        bool w_ok = ok && mbar_wait(bar(PVDONE), (uint32_t)t & 1u, abort);
        w_ok = __all_sync(0xffffffffu, w_ok) != 0;
        ok = ok && w_ok;
        if (ok) {
          tc_fence_after();
          const size_t id = (size_t)cta + (size_t)cur.i;
          float* dst = p.part_u + id * HEADS * LAT + x;
          // The merge kernel reads the partials right after this kernel: keep
          // them in L2 while the cache streams past under its own policies.
          const uint64_t keep = l2_policy_evict_last();
#pragma unroll 1
          for (int b = 0; b < 4; ++b)
#pragma unroll 1
            for (int cc = 0; cc < 3; ++cc) {
              float u[32];
              tmem_ld32(tmem + lane_off + TM_U + (uint32_t)(b * HEADS + 32 * cc), u);
              tmem_wait_ld_dep(u);
#pragma unroll
              for (int e = 0; e < 32; ++e) st_global_hint(dst + (size_t)(32 * cc + e) * LAT + 128 * b, u[e], keep);
            }
          if (head) {
            st_global_hint(p.part_ml + (id * HEADS + x) * 2 + 0, m_used, keep);
            st_global_hint(p.part_ml + (id * HEADS + x) * 2 + 1, l, keep);
            // Prefill: the head's largest scaled logit (order-independent atomic max).
            if (p.maxlogit && piece_max > -INFINITY) atomic_max_float(p.maxlogit + x, piece_max * p.scale);
          }
          tc_fence_before();
          mbar_arrive(bar(UFREE));
        }
        m_used = -INFINITY;
        l = 0.f;
        piece_max = -INFINITY;
      }
      cur.next();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Work plan of the split kernel, built by one block of 256 threads:
//   plan[0..n]        P_i = number of BT-token tiles of sequences 0..i-1
//   plan[n+1+c]       the sequence holding tile floor(c P_n / G), c < G
__device__ void build_plan(int n_seq, Windows win, int G, int* __restrict__ plan) {
  __shared__ int wsum[8];
  __shared__ int carry;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) { carry = 0; plan[0] = 0; }
  __syncthreads();
  for (int base = 0; base < n_seq; base += 256) {
    const int i = base + (int)threadIdx.x;
    int x = i < n_seq ? (win.len(i) + BT - 1) / BT : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    int pre = carry;
    for (int w = 0; w < warp; ++w) pre += wsum[w];
    const int incl = pre + x;
    if (i < n_seq) plan[i + 1] = incl;
    __syncthreads();
    if (threadIdx.x == 255) carry = incl;
    __syncthreads();
  }
  const long long N = carry;
  for (int c = threadIdx.x; c < G; c += 256) {
    const long long t = (long long)c * N / G;
    int lo = 0, hi = n_seq - 1;                  // largest i with P_i <= t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (plan[mid] <= t) lo = mid; else hi = mid - 1;
    }
    plan[n_seq + 1 + c] = lo;
  }
}

constexpr int ABS_SEQ = 64;                    // sequences per absorb block
constexpr int ABS_Q = 128;                     // latent columns per absorb block
constexpr int LDK = 136;                       // padded bf16 row of a 128-wide staged operand
constexpr size_t ABS_SMEM = (size_t)(ABS_Q + ABS_SEQ) * LDK * 2;

// q~[i][h] = [q^C_h W_UK,h^T | q^S_h] in bf16.  Block = (head h, 128 latent
// columns, 64 sequences), 8 warps.  The block's rows of W_UK,h (128 x 128,
// one 256-byte row segment per latent index) and its q^C rows are staged in
// shared memory with 16-byte loads; warp w computes 16 latent columns.
// Block (HEADS, 0, 0) builds the split kernel's work plan meanwhile.
__global__ void __launch_bounds__(256) absorb_kernel(int n_seq, const __nv_bfloat16* __restrict__ q,
                                                     const __nv_bfloat16* __restrict__ W_UKV,
                                                     __nv_bfloat16* __restrict__ q_abs, Windows win,
                                                     int G, int* __restrict__ plan) {
  extern __shared__ __align__(16) uint8_t asm_[];
  __nv_bfloat16* Ws = reinterpret_cast<__nv_bfloat16*>(asm_);      // [128][LDK]: W_UK,h[latent][k]
  __nv_bfloat16* As = Ws + ABS_Q * LDK;                             // [64][LDK]: q^C[i][k]
  const int h = blockIdx.x, n0 = blockIdx.y * ABS_Q, i0 = blockIdx.z * ABS_SEQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  constexpr size_t ldw = (size_t)HEADS * 256;
  griddep_launch_dependents();                 // the split kernel may be scheduled (it waits for this grid)
  if (h == HEADS) {                            // the extra column of blocks: one of them builds the plan
    if (blockIdx.y == 0 && blockIdx.z == 0) build_plan(n_seq, win, G, plan);
    return;
  }
  for (int e = threadIdx.x; e < ABS_Q * 16; e += blockDim.x) {
    const int n = e >> 4, c = e & 15;
    cp_async16(Ws + n * LDK + c * 8, W_UKV + (size_t)(n0 + n) * ldw + (size_t)h * 256 + c * 8);
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
    float acc[2][4] = {};
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int k0 = kk * 16 + 2 * t;
      const __nv_bfloat16* ar = As + (mt * 16 + g) * LDK + k0;
      const uint32_t a[4] = {lds32(ar), lds32(ar + 8 * LDK), lds32(ar + 8), lds32(ar + 8 * LDK + 8)};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const __nv_bfloat16* br = Ws + (warp * 16 + nt * 8 + g) * LDK + k0;
        mma16816(acc[nt], a, lds32(br), lds32(br + 8));
      }
    }
    const int ra = i0 + mt * 16 + g, rb = ra + 8;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int col = n0 + warp * 16 + nt * 8 + 2 * t;
      if (ra < n_seq)
        *reinterpret_cast<__nv_bfloat162*>(q_abs + ((size_t)ra * HEADS + h) * WID + col) = __floats2bfloat162_rn(acc[nt][0], acc[nt][1]);
      if (rb < n_seq)
        *reinterpret_cast<__nv_bfloat162*>(q_abs + ((size_t)rb * HEADS + h) * WID + col) = __floats2bfloat162_rn(acc[nt][2], acc[nt][3]);
    }
  }
  // q^S passes through unchanged: 64 values = 8 x 16 bytes per sequence.
  if (blockIdx.y != 0) return;
  for (int e = threadIdx.x; e < ABS_SEQ * 8; e += blockDim.x) {
    const int i = i0 + (e >> 3), c = e & 7;
    if (i < n_seq)
      *reinterpret_cast<uint4*>(q_abs + ((size_t)i * HEADS + h) * WID + LAT + c * 8) =
          *reinterpret_cast<const uint4*>(q + ((size_t)i * HEADS + h) * 192 + 128 + c * 8);
  }
}

constexpr int MP_SEQ = 64;                     // sequences per merge + projection block
constexpr int MP_THREADS = 512;
constexpr int MP_MAXP = 32;                    // pieces per sequence merged in one batch
constexpr int LDU = LAT + 8;                   // padded bf16 row of a staged merged latent
constexpr int LDWV = 128 + 8;                  // padded bf16 row of the staged W_UV,h
constexpr size_t MP_SMEM = (size_t)LAT * LDWV * 2 + (size_t)MP_SEQ * LDU * 2;

// Pieces of one sequence for the merge: CTA c's piece of sequence i is
// partial c + i, for the CTAs c in [c_lo, c_hi] whose tile ranges meet the
// sequence's tiles (empty ranges write nothing and are skipped).
struct MergeSeq {
  int i, c_lo, n;                              // n = 0: no tiles (zeros)
  __device__ void init(int seq, int n_seq, int G, const int* plan, long long N) {
    i = seq;
    n = 0;
    c_lo = 0;
    if (seq >= n_seq) return;
    const long long t_lo = plan[seq], t_hi = plan[seq + 1] - 1;
    if (t_hi < t_lo) return;
    // CTA holding tile t: the largest c with floor(c N / G) <= t.
    c_lo = (int)(((t_lo + 1) * G - 1) / N);
    n = (int)(((t_hi + 1) * G - 1) / N) - c_lo + 1;
  }
};

// Merge + un-absorb, one block per (head h, 64 sequences), 16 warps.
//   1. W_UV,h (512 x 128) is staged in shared memory with cp.async; it does
//      not depend on the split kernel, so with a programmatic launch it is
//      fetched while the split kernel finishes.
//   2. Merge: u = sum_s U_s 2^((m_s - M) c) / sum_s l_s 2^((m_s - M) c) over
//      the pieces s of a sequence, rounded to bf16 into shared memory.  A warp
//      merges two sequences at a time: lane j reads piece j's (m, l) of both,
//      then the pieces' U rows (16 latents per lane) of both sequences are
//      loaded together, so each pair costs two dependent global round trips.
//   3. o = u W_UV,h (* sigmoid(g)) with mma.sync: warp w owns 16 sequences
//      (w mod 4) and 32 output columns (w / 4).
__global__ void __launch_bounds__(MP_THREADS, 1)
merge_project_kernel(int n_seq, int G, const int* __restrict__ plan, float scale_log2,
                     const float* __restrict__ part_ml, const float* __restrict__ part_u,
                     const __nv_bfloat16* __restrict__ W_UKV, const __nv_bfloat16* __restrict__ g,
                     __nv_bfloat16* __restrict__ O) {
  extern __shared__ __align__(16) uint8_t mps[];
  __nv_bfloat16* Wv = reinterpret_cast<__nv_bfloat16*>(mps);                     // [512][LDWV]
  __nv_bfloat16* Us = Wv + LAT * LDWV;                                             // [64][LDU]
  const int h = blockIdx.x, i0 = blockIdx.y * MP_SEQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr size_t ldw = (size_t)HEADS * 256;
  for (int e = threadIdx.x; e < LAT * 16; e += MP_THREADS) {
    const int k = e >> 4, c = e & 15;
    cp_async16(Wv + k * LDWV + c * 8, W_UKV + (size_t)k * ldw + (size_t)h * 256 + 128 + c * 8);
  }
  griddep_wait();                                // the split kernel's partials
  const long long N = plan[n_seq];
  auto empty = [&](int cc) { return (long long)cc * N / G == (long long)(cc + 1) * N / G; };
  for (int r0 = warp; r0 < MP_SEQ; r0 += 2 * (MP_THREADS / 32)) {
    MergeSeq sq[2];
    sq[0].init(i0 + r0, n_seq, G, plan, N);
    sq[1].init(i0 + r0 + MP_THREADS / 32, n_seq, G, plan, N);
    float4 acc[2][4];
    float Ls[2] = {0.f, 0.f};
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[a][q] = make_float4(0.f, 0.f, 0.f, 0.f);
    const int nmax = max(sq[0].n, sq[1].n);
    for (int base = 0; base < nmax; base += MP_MAXP) {
      // Lane j: (m, l) of piece base + j of both sequences, one round trip.
      float ml[2], ll[2], M[2], w[2];
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        ml[a] = -INFINITY; ll[a] = 0.f;
        const int cc = sq[a].c_lo + base + lane;
        if (base + lane < sq[a].n && !empty(cc)) {
          const size_t k = (size_t)(cc + sq[a].i) * HEADS + h;
          ml[a] = part_ml[2 * k];
          ll[a] = part_ml[2 * k + 1];
        }
      }
      // A sequence with more than MP_MAXP pieces needs the max over all of
      // them before any weight: take it from a first pass in that case.
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        M[a] = ml[a];
        if (sq[a].n > MP_MAXP)
          for (int cc = sq[a].c_lo + lane; cc < sq[a].c_lo + sq[a].n; cc += 32)
            if (!empty(cc)) M[a] = fmaxf(M[a], part_ml[((size_t)(cc + sq[a].i) * HEADS + h) * 2]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M[a] = fmaxf(M[a], __shfl_xor_sync(0xffffffffu, M[a], o));
        // Empty or missing pieces have m = -inf, hence weight 0.
        w[a] = ml[a] == -INFINITY ? 0.f : ex2((ml[a] - M[a]) * scale_log2);
        float lw = ll[a] * w[a];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
        Ls[a] += lw;
      }
      const int cnt = min(MP_MAXP, nmax - base);
#pragma unroll 2
      for (int j = 0; j < cnt; ++j) {
        float4 v[2][4];
        float wj[2];
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          wj[a] = __shfl_sync(0xffffffffu, w[a], j);
          // A piece with weight 0 (empty, or past this sequence's pieces) is not read.
          const float4* src = reinterpret_cast<const float4*>(
              part_u + ((size_t)(sq[a].c_lo + base + j + sq[a].i) * HEADS + h) * LAT);
#pragma unroll
          for (int q = 0; q < 4; ++q) v[a][q] = wj[a] != 0.f ? src[lane + 32 * q] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc[a][q].x = fmaf(v[a][q].x, wj[a], acc[a][q].x); acc[a][q].y = fmaf(v[a][q].y, wj[a], acc[a][q].y);
            acc[a][q].z = fmaf(v[a][q].z, wj[a], acc[a][q].z); acc[a][q].w = fmaf(v[a][q].w, wj[a], acc[a][q].w);
          }
      }
      // With more than MP_MAXP pieces, later batches must use the same M:
      // the first pass above already took the max over all pieces.
    }
#pragma unroll
    for (int a = 0; a < 2; ++a) {
      const int r = r0 + a * (MP_THREADS / 32);
      uint2* dst = reinterpret_cast<uint2*>(Us + r * LDU);
      const float inv = sq[a].n > 0 ? 1.f / Ls[a] : 0.f;   // no tiles: zeros
#pragma unroll
      for (int q = 0; q < 4; ++q)
        dst[lane + 32 * q] = make_uint2(pack_bf16x2(acc[a][q].x * inv, acc[a][q].y * inv),
                                        pack_bf16x2(acc[a][q].z * inv, acc[a][q].w * inv));
    }
  }
  cp_async_wait_all();
  __syncthreads();
  const int gq = lane >> 2, t = lane & 3;
  const int mt = warp & 3, c0 = (warp >> 2) * 32;
  float acc[4][4] = {};
#pragma unroll 4
  for (int kk = 0; kk < LAT / 16; ++kk) {
    const int k0 = kk * 16;
    const __nv_bfloat16* ar = Us + (mt * 16 + gq) * LDU + k0 + 2 * t;
    const uint32_t a[4] = {lds32(ar), lds32(ar + 8 * LDU), lds32(ar + 8), lds32(ar + 8 * LDU + 8)};
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      uint32_t b0, b1;
      ldsm_x2_trans(b0, b1, Wv + (k0 + (lane & 15)) * LDWV + c0 + nt * 8);
      mma16816(acc[nt], a, b0, b1);
    }
  }
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int i = i0 + mt * 16 + gq + 8 * hr;
      if (i >= n_seq) continue;
      const int col = c0 + nt * 8 + 2 * t;
      const size_t idx = ((size_t)i * HEADS + h) * 128 + col;
      float o0 = acc[nt][2 * hr], o1 = acc[nt][2 * hr + 1];
      if (g) {
        const float2 gv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(g + idx));
        o0 *= 1.f / (1.f + __expf(-gv.x));
        o1 *= 1.f / (1.f + __expf(-gv.y));
      }
      *reinterpret_cast<__nv_bfloat162*>(O + idx) = __floats2bfloat162_rn(o0, o1);
    }
}


inline size_t workspace_bytes(int n) {
  auto al = [](size_t x) { return (x + 1023) & ~(size_t)1023; };
  const size_t np = (size_t)G_CAP + n;
  return al((size_t)n * HEADS * WID * 2) + al(((size_t)n + 1 + G_CAP) * 4) + al(np * HEADS * 2 * 4) +
         al(np * HEADS * LAT * 4);
}

}  // namespace tc_dec
}  // namespace gmla
