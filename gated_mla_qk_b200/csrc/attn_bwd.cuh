// Backward of the causal gated MLA attention, CUDA-core form (fp32 arithmetic,
// fp32 gradients; Q/K^C/k^S/V/g in the layer's dtype, o and dL/do in fp32 as
// the training forward leaves them), for head widths other than Kimi K3's and
// for fp32 layers.  The row pass below also serves the tcgen05 kernels.
//
// Forward ("Kimi K3 · Gated MLA · OpenModelAtlas", "All 20 steps"):
//   S = Q_h K_h^T / sqrt(d_qk), K_h = [K^C_h | k^S];  A = causal softmax(S);
//   O~ = A V_h;  o = sigmoid(g) * O~.
// Gradients (chain rule through each step):
//   dO~ = dO * sigmoid(g);  dg = dO * o * (1 - sigmoid(g))   (o = sigmoid(g) O~)
//   D_t = sum_c dO~ O~ = sum_c dO * o                        (the gate cancels)
//   A_ts = exp(S_ts - lse_t);  dA = dO~ V_h^T;  dS = A * (dA - D)
//   dV_h = A^T dO~;  dQ_h = dS K_h / sqrt(d_qk);  dK_h = dS^T Q_h / sqrt(d_qk)
// and k^S, one key part shared by every head, gets the sum over heads of the
// last d_s columns of dK_h.
//
// Three kernels: a row pass (D, dO~, dg), a key-tile pass that owns dK_h and
// dV_h for 32 keys and walks the query tiles at or after them, and a
// query-tile pass that owns dQ_h for 32 rows and walks the key tiles at or
// before them (S and A are recomputed from lse in both, so neither needs
// atomics except the cross-head sum of dk^S).
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace gmla {
namespace bwd {

constexpr int BQ = 32, BK = 32, NT = 256;
constexpr int kMaxD = 256;                       // d_qk and d_v limits

// One warp per (b, t, h): D, dO~ and dg.
// TO = float for the CUDA-core passes, bf16 for the tcgen05 kernels (tc_bwd.cuh).
template <typename T, typename TO>
__global__ void __launch_bounds__(256) row_kernel(int rows, int H, int d_v, const float* __restrict__ O,
                                                  const float* __restrict__ dO, const T* __restrict__ g,
                                                  TO* __restrict__ dOt, float* __restrict__ D,
                                                  float* __restrict__ dg) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows) return;                       // row = (b*T + t)*H + h
  const size_t base = (size_t)row * d_v;
  float acc = 0.f;
  for (int c = lane; c < d_v; c += 32) {
    const float d = dO[base + c], o = O[base + c];
    acc = fmaf(d, o, acc);
    if (g) {
      const float sg = 1.f / (1.f + __expf(-ld(g + base + c)));
      dOt[base + c] = cvt<TO>(d * sg);
      dg[base + c] = d * o * (1.f - sg);
    } else {
      dOt[base + c] = cvt<TO>(d);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) D[row] = acc;
}

// The same row pass for d_v = 128 with a bf16 gate and bf16 dO~ (the tcgen05
// backward's form): one warp per row, lane l takes columns 4l .. 4l+3 through
// 16-byte fp32 and 8-byte bf16 accesses (4-byte accesses left the pass
// latency-bound).  D sums each lane's four products first, then across lanes.
__global__ void __launch_bounds__(256) row128_kernel(int rows, const float* __restrict__ O, const float* __restrict__ dO,
                                                     const __nv_bfloat16* __restrict__ g, __nv_bfloat16* __restrict__ dOt,
                                                     float* __restrict__ D, float* __restrict__ dg) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows) return;                       // row = (b*T + t)*H + h
  const size_t base = (size_t)row * 128 + 4 * lane;
  const float4 d = *reinterpret_cast<const float4*>(dO + base);
  const float4 o = *reinterpret_cast<const float4*>(O + base);
  float acc = fmaf(d.w, o.w, fmaf(d.z, o.z, fmaf(d.y, o.y, d.x * o.x)));
  float t[4] = {d.x, d.y, d.z, d.w};
  if (g) {
    const uint2 gv = *reinterpret_cast<const uint2*>(g + base);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
    const float2 ga = __bfloat1622float2(g2[0]), gb = __bfloat1622float2(g2[1]);
    const float sg[4] = {1.f / (1.f + __expf(-ga.x)), 1.f / (1.f + __expf(-ga.y)), 1.f / (1.f + __expf(-gb.x)),
                         1.f / (1.f + __expf(-gb.y))};
    const float dv[4] = {d.x, d.y, d.z, d.w}, ov[4] = {o.x, o.y, o.z, o.w};
    float q[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      t[e] = dv[e] * sg[e];
      q[e] = dv[e] * ov[e] * (1.f - sg[e]);
    }
    *reinterpret_cast<float4*>(dg + base) = make_float4(q[0], q[1], q[2], q[3]);
  }
  __nv_bfloat162 p0 = __floats2bfloat162_rn(t[0], t[1]), p1 = __floats2bfloat162_rn(t[2], t[3]);
  uint2 out;
  out.x = *reinterpret_cast<uint32_t*>(&p0);
  out.y = *reinterpret_cast<uint32_t*>(&p1);
  *reinterpret_cast<uint2*>(dOt + base) = out;
#pragma unroll
  for (int k = 16; k > 0; k >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, k);
  if (lane == 0) D[row] = acc;
}

struct Dims {
  int B, T, H, d_c, d_s, d_v;
  float scale;
};

// Loads columns [off, off + w) of rows [r0, r0 + 32) of a [B][T][row_stride]
// tensor into columns [col0, col0 + w) of s[32][ld_s] as fp32, zero past T.
template <typename T>
__device__ __forceinline__ void load_rows(float* s, int ld_s, const T* src, int b, int r0, int T_, size_t row_stride,
                                          size_t off, int w, int col0) {
  for (int i = threadIdx.x; i < 32 * w; i += NT) {
    const int r = i / w, k = i - r * w, t = r0 + r;
    s[r * ld_s + col0 + k] = (t < T_) ? ld(src + ((size_t)b * T_ + t) * row_stride + off + k) : 0.f;
  }
}

// A and dS of one (query tile, key tile) pair into sA / sdS [32][33]; thread
// (q = tid / 8, k = tid % 8 + 8m) computes four entries.
__device__ __forceinline__ void pair_scores(const float* sQ, const float* sK, const float* sdO, const float* sV,
                                            const float* slse, const float* sD, float* sA, float* sdS, int q0, int k0,
                                            int T_, int d_qk, int d_v, float scale) {
  const int q = threadIdx.x >> 3, kk = threadIdx.x & 7;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int k = kk + 8 * m;
    const int tq = q0 + q, tk = k0 + k;
    float s = 0.f, dp = 0.f;
    for (int d = 0; d < d_qk; ++d) s = fmaf(sQ[q * (d_qk + 1) + d], sK[k * (d_qk + 1) + d], s);
    for (int c = 0; c < d_v; ++c) dp = fmaf(sdO[q * (d_v + 1) + c], sV[k * (d_v + 1) + c], dp);
    const bool live = tq < T_ && tk <= tq;
    const float a = live ? __expf(s * scale - slse[q]) : 0.f;
    sA[q * (BK + 1) + k] = a;
    sdS[q * (BK + 1) + k] = a * (dp - sD[q]);
  }
}

inline size_t dkdv_smem(int d_qk, int d_v) {
  return sizeof(float) * (size_t)(2 * 32 * (d_qk + 1) + 2 * 32 * (d_v + 1) + 2 * 32 * (BK + 1) + 2 * 32);
}

// Block = (key tile, head, batch): dK_h and dV_h of 32 keys.
template <typename T>
__global__ void __launch_bounds__(NT) dkdv_kernel(Dims p, const T* __restrict__ Q, const T* __restrict__ KC,
                                                  const T* __restrict__ kS, const T* __restrict__ V,
                                                  const float* __restrict__ lse, const float* __restrict__ dOt,
                                                  const float* __restrict__ D, float* __restrict__ dKC,
                                                  float* __restrict__ dkS, float* __restrict__ dV) {
  extern __shared__ float sm[];
  const int d_qk = p.d_c + p.d_s, H = p.H;
  float* sK = sm;                                // [32][d_qk + 1]
  float* sV = sK + 32 * (d_qk + 1);              // [32][d_v + 1]
  float* sQ = sV + 32 * (p.d_v + 1);             // [32][d_qk + 1]
  float* sdO = sQ + 32 * (d_qk + 1);             // [32][d_v + 1]
  float* sA = sdO + 32 * (p.d_v + 1);            // [32][33]
  float* sdS = sA + 32 * (BK + 1);               // [32][33]
  float* slse = sdS + 32 * (BK + 1);             // [32]
  float* sD = slse + 32;                         // [32]
  const int kt = blockIdx.x, h = blockIdx.y, b = blockIdx.z, k0 = kt * BK;
  load_rows(sK, d_qk + 1, KC, b, k0, p.T, (size_t)H * p.d_c, (size_t)h * p.d_c, p.d_c, 0);
  if (p.d_s) load_rows(sK, d_qk + 1, kS, b, k0, p.T, (size_t)p.d_s, 0, p.d_s, p.d_c);
  load_rows(sV, p.d_v + 1, V, b, k0, p.T, (size_t)H * p.d_v, (size_t)h * p.d_v, p.d_v, 0);
  const int k = threadIdx.x >> 3, cc = threadIdx.x & 7;
  float accK[kMaxD / 8], accV[kMaxD / 8];
#pragma unroll
  for (int m = 0; m < kMaxD / 8; ++m) { accK[m] = 0.f; accV[m] = 0.f; }
  const int n_qt = (p.T + BQ - 1) / BQ;
  for (int qt = kt; qt < n_qt; ++qt) {
    const int q0 = qt * BQ;
    __syncthreads();
    load_rows(sQ, d_qk + 1, Q, b, q0, p.T, (size_t)H * d_qk, (size_t)h * d_qk, d_qk, 0);
    load_rows(sdO, p.d_v + 1, dOt, b, q0, p.T, (size_t)H * p.d_v, (size_t)h * p.d_v, p.d_v, 0);
    if (threadIdx.x < 32) {
      const int t = q0 + threadIdx.x;
      slse[threadIdx.x] = t < p.T ? lse[((size_t)b * p.T + t) * H + h] : 0.f;
      sD[threadIdx.x] = t < p.T ? D[((size_t)b * p.T + t) * H + h] : 0.f;
    }
    __syncthreads();
    pair_scores(sQ, sK, sdO, sV, slse, sD, sA, sdS, q0, k0, p.T, d_qk, p.d_v, p.scale);
    __syncthreads();
    // dV[k][c] += sum_q A[q][k] dO~[q][c];  dK[k][d] += sum_q dS[q][k] Q[q][d]
    for (int q = 0; q < BQ; ++q) {
      const float a = sA[q * (BK + 1) + k], ds = sdS[q * (BK + 1) + k];
#pragma unroll
      for (int m = 0; m < kMaxD / 8; ++m) {
        const int c = cc + 8 * m;
        if (c < p.d_v) accV[m] = fmaf(a, sdO[q * (p.d_v + 1) + c], accV[m]);
        if (c < d_qk) accK[m] = fmaf(ds, sQ[q * (d_qk + 1) + c], accK[m]);
      }
    }
  }
  const int tk = k0 + k;
  if (tk < p.T) {
    const size_t rk = (size_t)b * p.T + tk;
#pragma unroll
    for (int m = 0; m < kMaxD / 8; ++m) {
      const int c = cc + 8 * m;
      if (c < p.d_v) dV[(rk * H + h) * p.d_v + c] = accV[m];
      if (c < p.d_c) dKC[(rk * H + h) * p.d_c + c] = accK[m] * p.scale;
      else if (c < d_qk) atomicAdd(dkS + rk * p.d_s + (c - p.d_c), accK[m] * p.scale);
    }
  }
}

inline size_t dq_smem(int d_qk, int d_v) { return dkdv_smem(d_qk, d_v); }

// Block = (query tile, head, batch): dQ_h of 32 rows.
template <typename T>
__global__ void __launch_bounds__(NT) dq_kernel(Dims p, const T* __restrict__ Q, const T* __restrict__ KC,
                                                const T* __restrict__ kS, const T* __restrict__ V,
                                                const float* __restrict__ lse, const float* __restrict__ dOt,
                                                const float* __restrict__ D, float* __restrict__ dQ) {
  extern __shared__ float sm[];
  const int d_qk = p.d_c + p.d_s, H = p.H;
  float* sK = sm;
  float* sV = sK + 32 * (d_qk + 1);
  float* sQ = sV + 32 * (p.d_v + 1);
  float* sdO = sQ + 32 * (d_qk + 1);
  float* sA = sdO + 32 * (p.d_v + 1);
  float* sdS = sA + 32 * (BK + 1);
  float* slse = sdS + 32 * (BK + 1);
  float* sD = slse + 32;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z, q0 = qt * BQ;
  load_rows(sQ, d_qk + 1, Q, b, q0, p.T, (size_t)H * d_qk, (size_t)h * d_qk, d_qk, 0);
  load_rows(sdO, p.d_v + 1, dOt, b, q0, p.T, (size_t)H * p.d_v, (size_t)h * p.d_v, p.d_v, 0);
  if (threadIdx.x < 32) {
    const int t = q0 + threadIdx.x;
    slse[threadIdx.x] = t < p.T ? lse[((size_t)b * p.T + t) * H + h] : 0.f;
    sD[threadIdx.x] = t < p.T ? D[((size_t)b * p.T + t) * H + h] : 0.f;
  }
  const int q = threadIdx.x >> 3, cc = threadIdx.x & 7;
  float acc[kMaxD / 8];
#pragma unroll
  for (int m = 0; m < kMaxD / 8; ++m) acc[m] = 0.f;
  for (int kt = 0; kt <= qt; ++kt) {
    const int k0 = kt * BK;
    __syncthreads();
    load_rows(sK, d_qk + 1, KC, b, k0, p.T, (size_t)H * p.d_c, (size_t)h * p.d_c, p.d_c, 0);
    if (p.d_s) load_rows(sK, d_qk + 1, kS, b, k0, p.T, (size_t)p.d_s, 0, p.d_s, p.d_c);
    load_rows(sV, p.d_v + 1, V, b, k0, p.T, (size_t)H * p.d_v, (size_t)h * p.d_v, p.d_v, 0);
    __syncthreads();
    pair_scores(sQ, sK, sdO, sV, slse, sD, sA, sdS, q0, k0, p.T, d_qk, p.d_v, p.scale);
    __syncthreads();
    // dQ[q][d] += sum_k dS[q][k] K[k][d]
    for (int kk = 0; kk < BK; ++kk) {
      const float ds = sdS[q * (BK + 1) + kk];
#pragma unroll
      for (int m = 0; m < kMaxD / 8; ++m) {
        const int c = cc + 8 * m;
        if (c < d_qk) acc[m] = fmaf(ds, sK[kk * (d_qk + 1) + c], acc[m]);
      }
    }
  }
  const int t = q0 + q;
  if (t < p.T) {
#pragma unroll
    for (int m = 0; m < kMaxD / 8; ++m) {
      const int c = cc + 8 * m;
      if (c < d_qk) dQ[(((size_t)b * p.T + t) * H + h) * d_qk + c] = acc[m] * p.scale;
    }
  }
}


inline size_t workspace_bytes(int B, int T, int H, int d_v) {
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return al((size_t)B * T * H * d_v * 4) + al((size_t)B * T * H * 4);
}

template <typename T>
int run(const Dims& p, const T* Q, const T* KC, const T* kS, const T* V, const T* g, const float* O,
        const float* lse, const float* dO, float* dQ, float* dKC, float* dkS, float* dV, float* dg, void* ws,
        cudaStream_t st) {
  const int d_qk = p.d_c + p.d_s;
  const size_t smem = dkdv_smem(d_qk, p.d_v);
  cudaError_t e = cudaFuncSetAttribute(dkdv_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(dq_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return cuda_status(e);
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  float* dOt = static_cast<float*>(ws);
  float* D = reinterpret_cast<float*>(static_cast<char*>(ws) + al((size_t)p.B * p.T * p.H * p.d_v * 4));
  const int rows = p.B * p.T * p.H;
  if (p.d_s) {
    e = cudaMemsetAsync(dkS, 0, (size_t)p.B * p.T * p.d_s * sizeof(float), st);
    if (e != cudaSuccess) return cuda_status(e);
  }
  row_kernel<T, float><<<(rows + 7) / 8, 256, 0, st>>>(rows, p.H, p.d_v, O, dO, g, dOt, D, dg);
  const int nt = (p.T + 31) / 32;
  dkdv_kernel<T><<<dim3(nt, p.H, p.B), NT, smem, st>>>(p, Q, KC, kS, V, lse, dOt, D, dKC, dkS, dV);
  dq_kernel<T><<<dim3(nt, p.H, p.B), NT, smem, st>>>(p, Q, KC, kS, V, lse, dOt, D, dQ);
  note_launches(3);
  return check_launch();
}

}  // namespace bwd
}  // namespace gmla
