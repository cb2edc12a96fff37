// QK-Clip weight rescale ("Anthology of the SOTA", record SOTA-131, "Source":
// heads whose max logit exceeds the threshold get their query and key
// projection weights rescaled).  Bandwidth kernel: only the clipped heads'
// column blocks are read and written, 16 bytes per thread access.
#pragma once

#include "common.cuh"

namespace gmla {
namespace clip {

// gamma_h = tau / maxlogit_h with IEEE round-to-nearest division; the
// square root is the correctly rounded one.  No fast-math approximation:
// the rescaled weights must match a float32 reference bit for bit.
__device__ __forceinline__ bool head_gamma(const float* maxlogit, int h, float tau, float* gam, float* root) {
  const float ml = maxlogit[h];
  if (!(ml > tau)) return false;
  *gam = __fdiv_rn(tau, ml);
  *root = __fsqrt_rn(*gam);
  return true;
}

template <typename T> struct Vec;   // 16-byte vector of T
template <> struct Vec<__nv_bfloat16> { static constexpr int n = 8; };
template <> struct Vec<float> { static constexpr int n = 4; };

__device__ __forceinline__ void scale_vec(uint4& v, float f, __nv_bfloat16*) {
  __nv_bfloat162* p = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __bfloat1622float2(p[i]);
    p[i] = __floats2bfloat162_rn(__fmul_rn(x.x, f), __fmul_rn(x.y, f));
  }
}
__device__ __forceinline__ void scale_vec(uint4& v, float f, float*) {
  float* p = reinterpret_cast<float*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) p[i] = __fmul_rn(p[i], f);
}

// Grid: x = blocks over (rows x vectors of the head's scaled columns),
//       y = head, z = 0 for W_UQ, 1 for W_UKV.
// W_UQ : head block of d_c + d_s columns at h*(d_c+d_s): sqrt(gamma) then gamma.
// W_UKV: head block at h*(d_c+d_v): the first d_c columns get sqrt(gamma).
template <typename T>
__global__ void __launch_bounds__(256) qkclip_kernel(
    T* __restrict__ W_UQ, T* __restrict__ W_UKV, int q_lora, int kv_lora, int H, int d_c, int d_s,
    int d_v, const float* __restrict__ maxlogit, float tau, unsigned char* __restrict__ clipped,
    float* __restrict__ gamma_out) {
  const int h = blockIdx.y;
  float gam = 1.f, root = 1.f;
  const bool clip = head_gamma(maxlogit, h, tau, &gam, &root);
  if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0) {
    if (clipped) clipped[h] = clip ? 1 : 0;
    if (gamma_out) gamma_out[h] = gam;
  }
  if (!clip) return;
  constexpr int VN = Vec<T>::n;
  const bool is_q = blockIdx.z == 0;
  const int cols = is_q ? (d_c + d_s) : d_c;              // scaled columns per row
  const int rows = is_q ? q_lora : kv_lora;
  const size_t ldw = is_q ? (size_t)H * (d_c + d_s) : (size_t)H * (d_c + d_v);
  T* base = (is_q ? W_UQ : W_UKV) + (size_t)h * (is_q ? (d_c + d_s) : (d_c + d_v));
  const int vpr = cols / VN;                               // vectors per row
  const int total = rows * vpr;
  for (int v = blockIdx.x * blockDim.x + threadIdx.x; v < total; v += gridDim.x * blockDim.x) {
    const int r = v / vpr, c = (v - r * vpr) * VN;
    uint4* p = reinterpret_cast<uint4*>(base + r * ldw + c);
    uint4 x = *p;
    scale_vec(x, c < d_c ? root : gam, (T*)nullptr);
    *p = x;
  }
}

// Element-wise form for column counts that are not a multiple of the vector.
template <typename T>
__global__ void qkclip_scalar_kernel(T* W_UQ, T* W_UKV, int q_lora, int kv_lora, int H, int d_c, int d_s,
                                     int d_v, const float* maxlogit, float tau, unsigned char* clipped,
                                     float* gamma_out) {
  const int h = blockIdx.y;
  float gam = 1.f, root = 1.f;
  const bool clip = head_gamma(maxlogit, h, tau, &gam, &root);
  if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0) {
    if (clipped) clipped[h] = clip ? 1 : 0;
    if (gamma_out) gamma_out[h] = gam;
  }
  if (!clip) return;
  const bool is_q = blockIdx.z == 0;
  const int cols = is_q ? (d_c + d_s) : d_c;
  const int rows = is_q ? q_lora : kv_lora;
  const size_t ldw = is_q ? (size_t)H * (d_c + d_s) : (size_t)H * (d_c + d_v);
  T* base = (is_q ? W_UQ : W_UKV) + (size_t)h * (is_q ? (d_c + d_s) : (d_c + d_v));
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < rows * cols; e += gridDim.x * blockDim.x) {
    const int r = e / cols, c = e - r * cols;
    T* p = base + r * ldw + c;
    *p = cvt<T>(__fmul_rn(ld(p), c < d_c ? root : gam));
  }
}

template <typename T>
inline int rescale(T* W_UQ, T* W_UKV, int q_lora, int kv_lora, int H, int d_c, int d_s, int d_v,
                   const float* maxlogit, float tau, unsigned char* clipped, float* gamma, cudaStream_t st) {
  constexpr int VN = Vec<T>::n;
  const bool vec = (d_c % VN == 0) && (d_s % VN == 0) && (d_v % VN == 0);
  const int per_head = max(q_lora * (d_c + d_s), kv_lora * d_c) / (vec ? VN : 1);
  const int bx = min(64, max(1, (per_head + 255) / 256));
  dim3 grid(bx, H, 2);
  if (vec)
    qkclip_kernel<T><<<grid, 256, 0, st>>>(W_UQ, W_UKV, q_lora, kv_lora, H, d_c, d_s, d_v, maxlogit, tau, clipped, gamma);
  else
    qkclip_scalar_kernel<T><<<grid, 256, 0, st>>>(W_UQ, W_UKV, q_lora, kv_lora, H, d_c, d_s, d_v, maxlogit, tau, clipped, gamma);
  note_launches(1);
  return check_launch();
}

}  // namespace clip
}  // namespace gmla
