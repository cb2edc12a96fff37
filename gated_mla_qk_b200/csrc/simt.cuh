// CUDA-core kernels: the fp32 path (tiny geometries, where tensor cores
// cannot give fp32 accuracy) and the general-shape path for geometries the
// tcgen05 kernels are not specialised for.  All arithmetic is fp32.
#pragma once

#include "common.cuh"

namespace gmla {
namespace simt {

// ---------------------------------------------------------------------------
// GEMM  C[M][N] = A[M][K] B[K][N]  (row-major), fp32 accumulation.
// 64x64 tile, 256 threads, 4x4 outputs per thread.  The epilogue functor
// decides where column n of row m is stored (plain, or split per head into
// K^C / V for the key/value up-projection).
// ---------------------------------------------------------------------------
template <typename T>
struct EpiPlain {
  T* C; int ldc;
  __device__ void operator()(int m, int n, float v) const { C[(size_t)m * ldc + n] = cvt<T>(v); }
};

// Column n of the [K^C_h | V_h]_h product goes to KC[m][h][j] or V[m][h][j-d_c].
template <typename T>
struct EpiSplitKV {
  T* KC; T* V; int H, d_c, d_v;
  __device__ void operator()(int m, int n, float v) const {
    const int w = d_c + d_v;
    const int h = n / w, j = n - h * w;
    if (j < d_c) KC[((size_t)m * H + h) * d_c + j] = cvt<T>(v);
    else         V[((size_t)m * H + h) * d_v + (j - d_c)] = cvt<T>(v);
  }
};

template <typename T, typename Epi>
__global__ void __launch_bounds__(256) gemm_kernel(int M, int N, int K, const T* __restrict__ A,
                                                   const T* __restrict__ B, Epi epi) {
  __shared__ float sA[16][64 + 4];
  __shared__ float sB[16][64 + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 64 * 16; i += 256) {
      const int r = i >> 4, c = i & 15;          // A tile: 64 rows x 16 k
      const int gm = m0 + r, gk = k0 + c;
      sA[c][r] = (gm < M && gk < K) ? ld(A + (size_t)gm * K + gk) : 0.f;
      const int kr = i >> 6, nc = i & 63;        // B tile: 16 k x 64 cols
      const int gk2 = k0 + kr, gn = n0 + nc;
      sB[kr][nc] = (gk2 < K && gn < N) ? ld(B + (size_t)gk2 * N + gn) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = sA[kk][ty + 16 * i]; b[i] = sB[kk][tx + 16 * i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty + 16 * i, n = n0 + tx + 16 * j;
      if (m < M && n < N) epi(m, n, acc[i][j]);
    }
}

template <typename T, typename Epi>
inline int gemm(int M, int N, int K, const T* A, const T* B, Epi epi, cudaStream_t st) {
  dim3 grid((N + 63) / 64, (M + 63) / 64);
  gemm_kernel<T, Epi><<<grid, 256, 0, st>>>(M, N, K, A, B, epi);
  note_launches(1);
  return check_launch();
}

// ---------------------------------------------------------------------------
// RMSNorm of each row: out = in / sqrt(mean(in^2) + eps) * w  (fp32 math).
// norm_rows: whole row.  norm_kv_rows: the joint [c^KV | k^S] row — the first
// kv_lora columns are normalised, the last d_s (k^S) are copied unchanged; the
// results also go to the optional latent cache row [RMSNorm(c^KV) | k^S].
// ---------------------------------------------------------------------------
template <typename T>
__device__ float block_sum_sq(const T* row, int n) {
  __shared__ float red[32];
  float s = 0.f;
  for (int j = threadIdx.x; j < n; j += blockDim.x) { const float v = ld(row + j); s = fmaf(v, v, s); }
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.f;
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) red[0] = s;
  }
  __syncthreads();
  const float r = red[0];
  __syncthreads();
  return r;
}

template <typename T>
__global__ void norm_rows_kernel(const T* __restrict__ in, int n, const T* __restrict__ w, float eps,
                                 T* __restrict__ out) {
  const T* row = in + (size_t)blockIdx.x * n;
  const float ss = block_sum_sq(row, n);
  const float inv = 1.f / sqrtf(ss / (float)n + eps);
  for (int j = threadIdx.x; j < n; j += blockDim.x)
    out[(size_t)blockIdx.x * n + j] = cvt<T>(ld(row + j) * inv * ld(w + j));
}

template <typename T>
__global__ void norm_kv_rows_kernel(const T* __restrict__ ckv_ks, int kv_lora, int d_s,
                                    const T* __restrict__ w, float eps, T* __restrict__ ckv_hat,
                                    T* __restrict__ kS, T* __restrict__ cache) {
  const int wid = kv_lora + d_s;
  const size_t m = blockIdx.x;
  const T* row = ckv_ks + m * wid;
  const float ss = block_sum_sq(row, kv_lora);
  const float inv = 1.f / sqrtf(ss / (float)kv_lora + eps);
  for (int j = threadIdx.x; j < kv_lora; j += blockDim.x) {
    const T v = cvt<T>(ld(row + j) * inv * ld(w + j));
    ckv_hat[m * kv_lora + j] = v;
    if (cache) cache[m * wid + j] = v;
  }
  for (int j = threadIdx.x; j < d_s; j += blockDim.x) {
    const T v = row[kv_lora + j];
    kS[m * d_s + j] = v;
    if (cache) cache[m * wid + kv_lora + j] = v;
  }
}

// bf16 forms of the two norms for row widths that are whole multiples of 256:
// one warp per row, the row held in registers (NV 16-byte vectors per lane),
// read once and written once with 16-byte accesses.
__device__ __forceinline__ void unpack_bf16x8(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 t = __bfloat1622float2(h[e]);
    f[2 * e] = t.x;
    f[2 * e + 1] = t.y;
  }
}
__device__ __forceinline__ uint4 pack_bf16x8(const float (&f)[8]) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
  return u;
}

// out[m] = in[m] / sqrt(mean(in[m]^2) + eps) * w for n = 256 NV columns.
template <int NV>
__global__ void __launch_bounds__(256) norm_rows_bf16_kernel(const __nv_bfloat16* __restrict__ in, int M,
                                                             const __nv_bfloat16* __restrict__ w, float eps,
                                                             __nv_bfloat16* __restrict__ out) {
  constexpr int n = 256 * NV;
  const int m = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (m >= M) return;
  const uint4* src = reinterpret_cast<const uint4*>(in + (size_t)m * n);
  float v[NV][8];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    unpack_bf16x8(src[lane + 32 * k], v[k]);
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(v[k][e], v[k][e], ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.f / sqrtf(ss / (float)n + eps);
  uint4* dst = reinterpret_cast<uint4*>(out + (size_t)m * n);
  const uint4* wv = reinterpret_cast<const uint4*>(w);
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    float wf[8], y[8];
    unpack_bf16x8(wv[lane + 32 * k], wf);
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] = v[k][e] * inv * wf[e];
    dst[lane + 32 * k] = pack_bf16x8(y);
  }
}

// The key/value latent: a row of [c^KV (256 NV) | k^S (64)]; writes c^KV's
// norm, k^S unchanged, and (if cache) the row [norm(c^KV) | k^S].
template <int NV>
__global__ void __launch_bounds__(256) norm_kv_rows_bf16_kernel(const __nv_bfloat16* __restrict__ ckv_ks, int M,
                                                                const __nv_bfloat16* __restrict__ w, float eps,
                                                                __nv_bfloat16* __restrict__ ckv_hat,
                                                                __nv_bfloat16* __restrict__ kS,
                                                                __nv_bfloat16* __restrict__ cache) {
  constexpr int kv = 256 * NV, wid = kv + 64;
  const int m = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (m >= M) return;
  const uint4* src = reinterpret_cast<const uint4*>(ckv_ks + (size_t)m * wid);
  float v[NV][8];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    unpack_bf16x8(src[lane + 32 * k], v[k]);
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(v[k][e], v[k][e], ss);
  }
  const uint4 ks = lane < 8 ? src[32 * NV + lane] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.f / sqrtf(ss / (float)kv + eps);
  const uint4* wv = reinterpret_cast<const uint4*>(w);
  uint4* hat = reinterpret_cast<uint4*>(ckv_hat + (size_t)m * kv);
  uint4* crow = cache ? reinterpret_cast<uint4*>(cache + (size_t)m * wid) : nullptr;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    float wf[8], y[8];
    unpack_bf16x8(wv[lane + 32 * k], wf);
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] = v[k][e] * inv * wf[e];
    const uint4 u = pack_bf16x8(y);
    hat[lane + 32 * k] = u;
    if (crow) crow[lane + 32 * k] = u;
  }
  if (lane < 8) {
    reinterpret_cast<uint4*>(kS + (size_t)m * 64)[lane] = ks;
    if (crow) crow[32 * NV + lane] = ks;
  }
}

// ---------------------------------------------------------------------------
// Causal gated attention with the fused per-head max logit.
// Block = (16 query rows, head h, batch b), 128 threads; key tiles of 32.
// Thread t serves query row r = t/8 and, inside a tile, keys j = t%8 + 8i.
// Online softmax over key tiles (exact running max), output columns
// c = t%8 + 8k accumulated in registers.  Supports d_qk <= 256, d_v <= 256.
// ---------------------------------------------------------------------------
constexpr int kAttnBQ = 16, kAttnBK = 32, kAttnMaxDV = 256;

template <typename T, typename TO = T>
__global__ void __launch_bounds__(128) attn_fwd_kernel(
    int T_, int H, int d_c, int d_s, int d_v, const T* __restrict__ Q, const T* __restrict__ KC,
    const T* __restrict__ kS, const T* __restrict__ V, const T* __restrict__ g, TO* __restrict__ O,
    float* __restrict__ maxlogit, float* __restrict__ lse, float scale) {
  extern __shared__ float smem[];
  const int d_qk = d_c + d_s;
  float* sQ = smem;                               // [BQ][d_qk]
  float* sK = sQ + kAttnBQ * d_qk;                // [BK][d_qk + 1]
  float* sV = sK + kAttnBK * (d_qk + 1);          // [BK][d_v]
  float* sP = sV + kAttnBK * d_v;                 // [BQ][BK + 1]
  __shared__ float sMax[kAttnBQ];

  const int q0 = blockIdx.x * kAttnBQ, h = blockIdx.y, b = blockIdx.z;
  const int r = threadIdx.x >> 3, lane8 = threadIdx.x & 7;
  const int t_row = q0 + r;

  for (int i = threadIdx.x; i < kAttnBQ * d_qk; i += 128) {
    const int rr = i / d_qk, k = i - rr * d_qk, t = q0 + rr;
    sQ[i] = (t < T_) ? ld(Q + (((size_t)b * T_ + t) * H + h) * d_qk + k) : 0.f;
  }
  float m_run = -INFINITY, l_run = 0.f;
  float acc[kAttnMaxDV / 8];
  const int n_cols = (d_v + 7 - lane8) / 8;   // columns lane8 + 8k < d_v
#pragma unroll
  for (int k = 0; k < kAttnMaxDV / 8; ++k) acc[k] = 0.f;

  const int k_end = min(T_, q0 + kAttnBQ);
  for (int k0 = 0; k0 < k_end; k0 += kAttnBK) {
    __syncthreads();
    for (int i = threadIdx.x; i < kAttnBK * d_qk; i += 128) {
      const int j = i / d_qk, k = i - j * d_qk, s = k0 + j;
      float v = 0.f;
      if (s < T_) v = (k < d_c) ? ld(KC + (((size_t)b * T_ + s) * H + h) * d_c + k)
                                : ld(kS + ((size_t)b * T_ + s) * d_s + (k - d_c));
      sK[j * (d_qk + 1) + k] = v;
    }
    for (int i = threadIdx.x; i < kAttnBK * d_v; i += 128) {
      const int j = i / d_v, c = i - j * d_v, s = k0 + j;
      sV[i] = (s < T_) ? ld(V + (((size_t)b * T_ + s) * H + h) * d_v + c) : 0.f;
    }
    __syncthreads();
    float sc[kAttnBK / 8];
    float tmax = -INFINITY;
#pragma unroll
    for (int i = 0; i < kAttnBK / 8; ++i) {
      const int j = lane8 + 8 * i, s = k0 + j;
      float dot = 0.f;
      for (int k = 0; k < d_qk; ++k) dot = fmaf(sQ[r * d_qk + k], sK[j * (d_qk + 1) + k], dot);
      sc[i] = (s <= t_row && s < T_) ? dot * scale : -INFINITY;
      tmax = fmaxf(tmax, sc[i]);
    }
    for (int o = 4; o > 0; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
    const float m_new = fmaxf(m_run, tmax);
    const float corr = expf(m_run - m_new);   // m_run = -inf on the first tile -> 0
    float psum = 0.f;
#pragma unroll
    for (int i = 0; i < kAttnBK / 8; ++i) {
      const float p = expf(sc[i] - m_new);
      sP[r * (kAttnBK + 1) + lane8 + 8 * i] = p;
      psum += p;
    }
    for (int o = 4; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
    l_run = l_run * corr + psum;
    m_run = m_new;
    __syncwarp();
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kAttnMaxDV / 8; ++k) {
      if (k < n_cols) {
        const int c = lane8 + 8 * k;
        float a = acc[k] * corr;
        for (int j = 0; j < kAttnBK; ++j) a = fmaf(sP[r * (kAttnBK + 1) + j], sV[j * d_v + c], a);
        acc[k] = a;
      }
    }
  }
  // Output row and the head's max logit (m_run is the exact row max here).
  if (t_row < T_) {
    if (lse && lane8 == 0) lse[((size_t)b * T_ + t_row) * H + h] = m_run + logf(l_run);
    const float inv_l = 1.f / l_run;
    for (int k = 0; k < n_cols; ++k) {
      const int c = lane8 + 8 * k;
      float o = acc[k] * inv_l;
      const size_t idx = ((size_t)b * T_ + t_row) * H * d_v + (size_t)h * d_v + c;
      if (g) o *= 1.f / (1.f + expf(-ld(g + idx)));
      O[idx] = cvt<TO>(o);
    }
  }
  if (lane8 == 0) sMax[r] = (t_row < T_) ? m_run : -INFINITY;
  __syncthreads();
  if (threadIdx.x == 0) {
    float mx = -INFINITY;
    for (int i = 0; i < kAttnBQ; ++i) mx = fmaxf(mx, sMax[i]);
    atomic_max_float(maxlogit + h, mx);
  }
}

__global__ void fill_kernel(float* p, int n, float v) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = v;
}

inline size_t attn_smem_bytes(int d_qk, int d_v) {
  return sizeof(float) * (size_t)(kAttnBQ * d_qk + kAttnBK * (d_qk + 1) + kAttnBK * d_v + kAttnBQ * (kAttnBK + 1));
}

template <typename T, typename TO = T>
inline int attn_fwd(int B, int T_, int H, int d_c, int d_s, int d_v, const T* Q, const T* KC, const T* kS,
                    const T* V, const T* g, TO* O, float* maxlogit, cudaStream_t st, float* lse = nullptr) {
  const size_t smem = attn_smem_bytes(d_c + d_s, d_v);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<T, TO>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_status(e);
  }
  fill_kernel<<<(H + 127) / 128, 128, 0, st>>>(maxlogit, H, -INFINITY);
  dim3 grid((T_ + kAttnBQ - 1) / kAttnBQ, H, B);
  attn_fwd_kernel<T, TO><<<grid, 128, smem, st>>>(T_, H, d_c, d_s, d_v, Q, KC, kS, V, g, O, maxlogit, lse,
                                              1.f / sqrtf((float)(d_c + d_s)));
  note_launches(2);
  return check_launch();
}

// ---------------------------------------------------------------------------
// Absorbed decode, CUDA-core form: absorb -> split-KV partials -> combine.
// ---------------------------------------------------------------------------
// q~[i][h] = [q^C_h W_UK,h^T | q^S_h] in fp32.  Block (h, i), 256 threads.
template <typename T>
__global__ void absorb_kernel(int H, int d_c, int d_s, int d_v, int kv_lora, const T* __restrict__ q,
                              const T* __restrict__ W_UKV, float* __restrict__ q_abs) {
  extern __shared__ float sq[];
  const int h = blockIdx.x, i = blockIdx.y, d_qk = d_c + d_s, w = kv_lora + d_s;
  const T* qh = q + ((size_t)i * H + h) * d_qk;
  for (int c = threadIdx.x; c < d_qk; c += blockDim.x) sq[c] = ld(qh + c);
  __syncthreads();
  float* out = q_abs + ((size_t)i * H + h) * w;
  const size_t ldw = (size_t)H * (d_c + d_v);
  for (int l = threadIdx.x; l < kv_lora; l += blockDim.x) {
    const T* wrow = W_UKV + l * ldw + (size_t)h * (d_c + d_v);
    float s = 0.f;
    for (int c = 0; c < d_c; ++c) s = fmaf(sq[c], ld(wrow + c), s);
    out[l] = s;
  }
  for (int j = threadIdx.x; j < d_s; j += blockDim.x) out[kv_lora + j] = sq[d_c + j];
}

// Partial softmax over one split of one sequence for one head.
// Block (h, split, i), 128 threads; thread t owns latent columns t + 128k.
constexpr int kDecMaxLatentPerThread = 8;   // kv_lora <= 1024

template <typename T>
__global__ void __launch_bounds__(128) decode_split_kernel(
    int H, int kv_lora, int d_s, int chunk, int n_split, const int* __restrict__ offs,
    const T* __restrict__ cache, const float* __restrict__ q_abs, float scale, float* __restrict__ part_ml,
    float* __restrict__ part_u) {
  extern __shared__ float sm[];
  const int w = kv_lora + d_s;
  float* sq = sm;               // [w]
  float* sp = sq + w;           // [32] scores of the current token tile
  const int h = blockIdx.x, sp_i = blockIdx.y, i = blockIdx.z;
  const int beg = offs[i], L = offs[i + 1] - beg;
  const int t0 = sp_i * chunk, t1 = min(L, t0 + chunk);
  const size_t pidx = ((size_t)i * H + h) * n_split + sp_i;
  for (int c = threadIdx.x; c < w; c += 128) sq[c] = q_abs[((size_t)i * H + h) * w + c];
  float acc[kDecMaxLatentPerThread];
#pragma unroll
  for (int k = 0; k < kDecMaxLatentPerThread; ++k) acc[k] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  for (int tt = t0; tt < t1; tt += 32) {
    // 4 warps x 8 tokens: lanes split the w-wide dot product.
    for (int jj = 0; jj < 8; ++jj) {
      const int j = warp * 8 + jj, tok = tt + j;
      float s = 0.f;
      if (tok < t1) {
        const T* row = cache + (size_t)(beg + tok) * w;
        for (int c = lane; c < w; c += 32) s = fmaf(sq[c], ld(row + c), s);
      }
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) sp[j] = (tok < t1) ? s * scale : -INFINITY;
    }
    __syncthreads();
    float tmax = -INFINITY;
    for (int j = 0; j < 32; ++j) tmax = fmaxf(tmax, sp[j]);
    const float m_new = fmaxf(m_run, tmax);
    const float corr = expf(m_run - m_new);
    float psum = 0.f;
    float p[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) { p[j] = expf(sp[j] - m_new); psum += p[j]; }
    l_run = l_run * corr + psum;
    m_run = m_new;
#pragma unroll
    for (int k = 0; k < kDecMaxLatentPerThread; ++k) {
      const int c = threadIdx.x + 128 * k;
      if (c < kv_lora) {
        float a = acc[k] * corr;
        for (int j = 0; j < 32; ++j) {
          const int tok = tt + j;
          if (tok < t1) a = fmaf(p[j], ld(cache + (size_t)(beg + tok) * w + c), a);
        }
        acc[k] = a;
      }
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) { part_ml[2 * pidx] = m_run; part_ml[2 * pidx + 1] = l_run; }
#pragma unroll
  for (int k = 0; k < kDecMaxLatentPerThread; ++k) {
    const int c = threadIdx.x + 128 * k;
    if (c < kv_lora) part_u[pidx * kv_lora + c] = acc[k];
  }
}

// Merge the splits of (sequence i, head h) and apply W_UV,h (and the gate).
template <typename T>
__global__ void decode_combine_kernel(int H, int d_c, int d_v, int kv_lora, int n_split, int chunk,
                                      const int* __restrict__ offs, const float* __restrict__ part_ml,
                                      const float* __restrict__ part_u, const T* __restrict__ W_UKV,
                                      const T* __restrict__ g, T* __restrict__ O) {
  extern __shared__ float su[];  // [kv_lora]
  const int h = blockIdx.x, i = blockIdx.y;
  const int L = offs[i + 1] - offs[i];
  const int ns = min(n_split, (L + chunk - 1) / chunk);
  const size_t base = ((size_t)i * H + h) * n_split;
  float M = -INFINITY;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, part_ml[2 * (base + s)]);
  float Lsum = 0.f;
  for (int s = 0; s < ns; ++s) Lsum += part_ml[2 * (base + s) + 1] * expf(part_ml[2 * (base + s)] - M);
  const float invL = Lsum > 0.f ? 1.f / Lsum : 0.f;   // an empty cache (no splits) decodes to 0
  for (int c = threadIdx.x; c < kv_lora; c += blockDim.x) {
    float u = 0.f;
    for (int s = 0; s < ns; ++s) u += part_u[(base + s) * kv_lora + c] * expf(part_ml[2 * (base + s)] - M);
    su[c] = u * invL;
  }
  __syncthreads();
  const size_t ldw = (size_t)H * (d_c + d_v);
  for (int c = threadIdx.x; c < d_v; c += blockDim.x) {
    const T* col = W_UKV + (size_t)h * (d_c + d_v) + d_c + c;
    float o = 0.f;
    for (int l = 0; l < kv_lora; ++l) o = fmaf(su[l], ld(col + l * ldw), o);
    const size_t idx = ((size_t)i * H + h) * d_v + c;
    if (g) o *= 1.f / (1.f + expf(-ld(g + idx)));
    O[idx] = cvt<T>(o);
  }
}

constexpr int kDecChunk = 1024;

inline int decode_splits(int max_len) { return (max_len + kDecChunk - 1) / kDecChunk; }

inline size_t decode_workspace(int H, int kv_lora, int d_s, int n, int max_len) {
  const size_t ns = decode_splits(max_len);
  size_t b = sizeof(float) * (size_t)n * H * (kv_lora + d_s);      // absorbed queries
  b = (b + 255) & ~(size_t)255;
  b += sizeof(float) * (size_t)n * H * ns * 2;                      // (m, l) per split
  b = (b + 255) & ~(size_t)255;
  b += sizeof(float) * (size_t)n * H * ns * kv_lora;                // latent partial sums
  return b;
}

template <typename T>
inline int decode(int n, int H, int d_c, int d_s, int d_v, int kv_lora, const T* q, const T* W_UKV,
                  const T* cache, const int* offs, int max_len, const T* g, T* O, void* ws, cudaStream_t st) {
  const int ns = decode_splits(max_len);
  char* p = static_cast<char*>(ws);
  float* q_abs = reinterpret_cast<float*>(p);
  size_t off = ((sizeof(float) * (size_t)n * H * (kv_lora + d_s)) + 255) & ~(size_t)255;
  float* part_ml = reinterpret_cast<float*>(p + off);
  off = (off + sizeof(float) * (size_t)n * H * ns * 2 + 255) & ~(size_t)255;
  float* part_u = reinterpret_cast<float*>(p + off);
  absorb_kernel<T><<<dim3(H, n), 256, sizeof(float) * (d_c + d_s), st>>>(H, d_c, d_s, d_v, kv_lora, q, W_UKV, q_abs);
  decode_split_kernel<T><<<dim3(H, ns, n), 128, sizeof(float) * (kv_lora + d_s + 32), st>>>(
      H, kv_lora, d_s, kDecChunk, ns, offs, cache, q_abs, 1.f / sqrtf((float)(d_c + d_s)), part_ml, part_u);
  decode_combine_kernel<T><<<dim3(H, n), 128, sizeof(float) * kv_lora, st>>>(
      H, d_c, d_v, kv_lora, ns, kDecChunk, offs, part_ml, part_u, W_UKV, g, O);
  note_launches(3);
  return check_launch();
}

}  // namespace simt
}  // namespace gmla
