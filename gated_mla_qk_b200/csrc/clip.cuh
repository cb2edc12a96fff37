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

// Work items: (head h, matrix, chunk of kChunk 16-byte vectors of the head's
// scaled columns), walked by a grid-stride loop, so the blocks of unclipped
// heads cost one cached read of maxlogit[h] instead of a block launch each.
// W_UQ : head block of d_c + d_s columns at h*(d_c+d_s): sqrt(gamma) then gamma.
// W_UKV: head block at h*(d_c+d_v): the first d_c columns get sqrt(gamma).
// Each thread loads its four vectors before scaling and storing them.
constexpr int kPerThread = 4, kThreads = 256, kChunk = kPerThread * kThreads;

template <typename T>
__global__ void __launch_bounds__(kThreads) qkclip_kernel(
    T* __restrict__ W_UQ, T* __restrict__ W_UKV, int q_lora, int kv_lora, int H, int d_c, int d_s,
    int d_v, const float* __restrict__ maxlogit, float tau, unsigned char* __restrict__ clipped,
    float* __restrict__ gamma_out) {
  constexpr int VN = Vec<T>::n;
  if (blockIdx.x == 0)
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
      float gam = 1.f, root = 1.f;
      const bool clip = head_gamma(maxlogit, h, tau, &gam, &root);
      if (clipped) clipped[h] = clip ? 1 : 0;
      if (gamma_out) gamma_out[h] = gam;
    }
  const int vq = q_lora * (d_c + d_s) / VN, vk = kv_lora * d_c / VN;   // vectors per head and matrix
  const int nq = (vq + kChunk - 1) / kChunk, nk = (vk + kChunk - 1) / kChunk;
  const int per_head = nq + nk;
  for (int w = blockIdx.x; w < H * per_head; w += gridDim.x) {
    const int h = w / per_head, k = w - h * per_head;
    float gam = 1.f, root = 1.f;
    if (!head_gamma(maxlogit, h, tau, &gam, &root)) continue;
    const bool is_q = k < nq;
    const int chunk = is_q ? k : k - nq;
    const int cols = is_q ? (d_c + d_s) : d_c;              // scaled columns per row
    const int total = is_q ? vq : vk;
    const size_t ldw = is_q ? (size_t)H * (d_c + d_s) : (size_t)H * (d_c + d_v);
    T* base = (is_q ? W_UQ : W_UKV) + (size_t)h * (is_q ? (d_c + d_s) : (d_c + d_v));
    const int vpr = cols / VN;                               // vectors per row
    uint4 x[kPerThread];
    uint4* ptr[kPerThread];
    float f[kPerThread];
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
      const int v = chunk * kChunk + u * kThreads + (int)threadIdx.x;
      ptr[u] = nullptr;
      if (v < total) {
        const int r = v / vpr, c = (v - r * vpr) * VN;
        ptr[u] = reinterpret_cast<uint4*>(base + r * ldw + c);
        f[u] = c < d_c ? root : gam;
        x[u] = *ptr[u];
      }
    }
#pragma unroll
    for (int u = 0; u < kPerThread; ++u)
      if (ptr[u]) {
        scale_vec(x[u], f[u], (T*)nullptr);
        *ptr[u] = x[u];
      }
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
  if (vec) {
    const int items = H * ((q_lora * (d_c + d_s) / VN + kChunk - 1) / kChunk + (kv_lora * d_c / VN + kChunk - 1) / kChunk);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = max(1, min(items, 8 * sms));
    qkclip_kernel<T><<<grid, kThreads, 0, st>>>(W_UQ, W_UKV, q_lora, kv_lora, H, d_c, d_s, d_v, maxlogit, tau,
                                                clipped, gamma);
  } else {
    const int per_head = max(q_lora * (d_c + d_s), kv_lora * d_c);
    const int bx = min(64, max(1, (per_head + 255) / 256));
    qkclip_scalar_kernel<T><<<dim3(bx, H, 2), 256, 0, st>>>(W_UQ, W_UKV, q_lora, kv_lora, H, d_c, d_s, d_v, maxlogit,
                                                            tau, clipped, gamma);
  }
  note_launches(1);
  return check_launch();
}

}  // namespace clip
}  // namespace gmla
