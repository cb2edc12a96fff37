// libgmla: the C ABI declared in include/gmla.h.  One translation unit: the
// kernel headers are included here so the device error flag and the kernels
// live in one module.  Host code validates every argument before launching.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "simt.cuh"
#include "clip.cuh"
#include "sm100.cuh"
#include "tc_attn.cuh"
#include "tc_decode.cuh"
#include "tc_bwd.cuh"
#include "tc_gemm.cuh"
#include "attn_bwd.cuh"
#include "selftest.cuh"

namespace gmla {

static std::atomic<unsigned long long> g_launches{0};
static thread_local int g_last_cuda_error = 0;

void note_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return GMLA_OK;
  g_last_cuda_error = (int)e;
  return GMLA_ECUDA;
}

// ---------------------------------------------------------------------------
// Validation helpers
// ---------------------------------------------------------------------------
static int check_geom(const gmla_geom* g) {
  if (!g) return GMLA_EINVAL;
  if (g->H <= 0 || g->d_model <= 0 || g->q_lora <= 0 || g->kv_lora <= 0 || g->d_c <= 0 || g->d_s < 0 ||
      g->d_v <= 0 || !(g->rms_eps >= 0.f))
    return GMLA_EINVAL;
  return GMLA_OK;
}
static int check_dtype(gmla_dtype t) { return (t == GMLA_BF16 || t == GMLA_F32) ? GMLA_OK : GMLA_EINVAL; }

#define GMLA_REQUIRE(ptr)                      \
  do {                                         \
    if (!(ptr)) return GMLA_EINVAL;            \
    if (!aligned16(ptr)) return GMLA_EALIGN;   \
  } while (0)
#define GMLA_OPTIONAL(ptr)                           \
  do {                                               \
    if ((ptr) && !aligned16(ptr)) return GMLA_EALIGN; \
  } while (0)
#define GMLA_TRY(expr)              \
  do {                              \
    int _s = (expr);                \
    if (_s != GMLA_OK) return _s;   \
  } while (0)

static inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// A kernel's dynamic shared-memory opt-in is an attribute of the kernel in
// the current device's context, so it is set once per device the library is
// called on (devices past the table are set on every call).
constexpr int kMaxDevices = 64;
template <typename F>
static cudaError_t set_attributes_once(std::once_flag (&flags)[kMaxDevices], cudaError_t (&errs)[kMaxDevices], F set) {
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return set();
  std::call_once(flags[dev], [&] { errs[dev] = set(); });
  return errs[dev];
}

// ---------------------------------------------------------------------------
// TMA descriptors (driver entry point fetched once through the runtime)
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D bf16 tensor [d2][d1][d0] (d0 innermost, contiguous), box {64, box1, 1},
// 128-byte swizzle, out-of-range elements read as zero.
static int make_map_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box1 = 128) {
  auto enc = get_encode();
  if (!enc) return GMLA_EUNSUPPORTED;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {64, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GMLA_OK : GMLA_EUNSUPPORTED;
}

// 2-D bf16 tensor [d1][d0] (d0 innermost), box {64, box1}, 128-byte swizzle.
static int make_map_2d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint32_t box1) {
  auto enc = get_encode();
  if (!enc) return GMLA_EUNSUPPORTED;
  cuuint64_t dims[2] = {d0, d1};
  cuuint64_t strides[1] = {d0 * 2};
  cuuint32_t box[2] = {64, box1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GMLA_OK : GMLA_EUNSUPPORTED;
}

// Launch `k` on `st` with programmatic stream serialisation: the grid may be
// scheduled before the previous kernel on the stream has finished, and must
// call griddep_wait() before it reads anything that kernel writes.
template <typename... KArgs, typename... Args>
static cudaError_t launch_after_prev(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                     Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, args...);
}

static bool is_k3_head_geometry(const gmla_geom* g) { return g->d_c == 128 && g->d_s == 64 && g->d_v == 128; }

// The tensor-core decode is specialised for Kimi K3's heads and latent.
static bool is_k3_decode_geometry(const gmla_geom* g) {
  return is_k3_head_geometry(g) && g->H == tc_dec::HEADS && g->kv_lora == tc_dec::LAT;
}

static size_t decode_ws_bytes(const gmla_geom* g, gmla_dtype dtype, int n, int max_len) {
  size_t b = simt::decode_workspace(g->H, g->kv_lora, g->d_s, n, max_len);
  if (dtype == GMLA_BF16 && is_k3_decode_geometry(g)) b = std::max(b, tc_dec::workspace_bytes(n));
  return b;
}

// Absorbed attention of n queries over windows of the latent cache (decode:
// one window per sequence; prefill: each query's causal prefix).  cache_rows
// bounds the cache rows any window reaches, max_tiles the 96-token tiles of
// all windows; maxlogit (nullable) gets the per-head max of the scaled logits.
static int decode_tc(int n, const void* q, const void* W_UKV, const void* cache, tc_dec::Windows win,
                     uint64_t cache_rows, long long max_tiles, const void* gate, void* O, float* maxlogit, void* ws,
                     cudaStream_t st) {
  static std::once_flag once[kMaxDevices];
  static cudaError_t attr_err[kMaxDevices];
  const cudaError_t ae = set_attributes_once(once, attr_err, [] {
    cudaError_t e = cudaFuncSetAttribute(tc_dec::decode_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tc_dec::SMEM_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(tc_dec::merge_project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)tc_dec::MP_SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(tc_dec::absorb_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)tc_dec::ABS_SMEM);
    return e;
  });
  if (ae != cudaSuccess) return cuda_status(ae);
  // One split CTA per SM (at most G_CAP), never more CTAs than tiles can exist.
  int dev = 0, sms = 0;
  GMLA_TRY(cuda_status(cudaGetDevice(&dev)));
  GMLA_TRY(cuda_status(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)));
  const int G = (int)std::max<long long>(1, std::min<long long>(std::min(sms, tc_dec::G_CAP), max_tiles));
  using bf = __nv_bfloat16;
  auto al = [](size_t x) { return (x + 1023) & ~(size_t)1023; };
  const size_t np = (size_t)tc_dec::G_CAP + n;
  char* p = static_cast<char*>(ws);
  bf* q_abs = reinterpret_cast<bf*>(p);
  p += al((size_t)n * tc_dec::HEADS * tc_dec::WID * 2);
  int* plan = reinterpret_cast<int*>(p);
  p += al(((size_t)n + 1 + tc_dec::G_CAP) * 4);
  float* part_ml = reinterpret_cast<float*>(p);
  p += al(np * tc_dec::HEADS * 2 * 4);
  float* part_u = reinterpret_cast<float*>(p);
  CUtensorMap mC, mQ;
  // Rows of the cache map: every row a tile reads lies inside some window
  // (the last tile of a window is shifted back to end at its end), so
  // cache_rows bounds the coordinates that occur; rows before 0 read as zero.
  const uint64_t rows = std::min<uint64_t>(cache_rows, 0x7fffffffull);
  GMLA_TRY(make_map_2d(&mC, cache, tc_dec::WID, rows, tc_dec::BT));
  GMLA_TRY(make_map_2d(&mQ, q_abs, tc_dec::WID, (uint64_t)n * tc_dec::HEADS, tc_dec::HEADS));
  tc_dec::absorb_kernel<<<dim3(tc_dec::HEADS + 1, tc_dec::LAT / tc_dec::ABS_Q, (n + tc_dec::ABS_SEQ - 1) / tc_dec::ABS_SEQ), 256,
                          tc_dec::ABS_SMEM, st>>>(
      n, static_cast<const bf*>(q), static_cast<const bf*>(W_UKV), q_abs, win, G, plan);
  tc_dec::SplitParams sp;
  sp.n_seq = n; sp.G = G; sp.win = win; sp.plan = plan; sp.cache = static_cast<const bf*>(cache);
  sp.scale_log2 = (float)(1.4426950408889634 / std::sqrt(192.0));
  sp.part_ml = part_ml; sp.part_u = part_u;
  sp.maxlogit = maxlogit;
  sp.scale = 1.f / std::sqrt(192.f);
  // The split and merge kernels are launched behind their predecessor
  // (programmatic dependent launch): each waits for it with griddepcontrol.wait
  // before touching its results, so only their set-up overlaps its tail.
  GMLA_TRY(check_launch());
  GMLA_TRY(cuda_status(launch_after_prev(tc_dec::decode_split_kernel, dim3(G), dim3(192), tc_dec::SMEM_BYTES, st,
                                         mC, mQ, sp)));
  GMLA_TRY(cuda_status(launch_after_prev(tc_dec::merge_project_kernel,
                                         dim3(tc_dec::HEADS, (n + tc_dec::MP_SEQ - 1) / tc_dec::MP_SEQ),
                                         dim3(tc_dec::MP_THREADS), tc_dec::MP_SMEM, st, n, G, (const int*)plan,
                                         sp.scale_log2, (const float*)part_ml, (const float*)part_u,
                                         static_cast<const bf*>(W_UKV), static_cast<const bf*>(gate),
                                         static_cast<bf*>(O))));
  note_launches(3);
  return check_launch();
}

// ---------------------------------------------------------------------------
// Attention forward dispatch
// ---------------------------------------------------------------------------
static int attn_fwd_tc(const gmla_geom* g, int B, int T, const void* Q, const void* KC, const void* kS,
                       const void* V, const void* gate, void* O, bool out_f32, float* maxlogit, float* lse,
                       cudaStream_t st) {
  static std::once_flag once[kMaxDevices];
  static cudaError_t attr_err[kMaxDevices];
  const cudaError_t ae = set_attributes_once(once, attr_err, [] {
    cudaError_t e = cudaFuncSetAttribute(tc_attn::attn_fwd_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tc_attn::SMEM_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(tc_attn::attn_fwd_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)tc_attn::SMEM_BYTES);
    return e;
  });
  if (ae != cudaSuccess) return cuda_status(ae);
  CUtensorMap mQ, mKC, mKS, mV;
  const int H = g->H;
  GMLA_TRY(make_map_3d(&mQ, Q, (uint64_t)H * 192, T, B));
  GMLA_TRY(make_map_3d(&mKC, KC, (uint64_t)H * 128, T, B));
  GMLA_TRY(make_map_3d(&mKS, kS, 64, T, B));
  GMLA_TRY(make_map_3d(&mV, V, (uint64_t)H * 128, T, B));
  tc_attn::Params p;
  p.B = B; p.T = T; p.H = H; p.n_qtiles = (T + tc_attn::BM - 1) / tc_attn::BM;
  p.g = static_cast<const __nv_bfloat16*>(gate);
  p.O = O;
  p.maxlogit = maxlogit;
  p.lse = lse;
  p.scale = 1.f / std::sqrt(192.f);
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt(192.0));
  simt::fill_kernel<<<(H + 127) / 128, 128, 0, st>>>(maxlogit, H, -INFINITY);
  // bf16 output: maps of the gate and of O for the epilogue's tile copies.
  CUtensorMap mG = mQ, mO = mQ;
  if (!out_f32) {
    if (gate) GMLA_TRY(make_map_3d(&mG, gate, (uint64_t)H * 128, T, B));
    GMLA_TRY(make_map_3d(&mO, O, (uint64_t)H * 128, T, B));
  }
  const unsigned grid = (unsigned)p.n_qtiles * (unsigned)H * (unsigned)B;
  if (out_f32) tc_attn::attn_fwd_kernel<true><<<grid, 192, tc_attn::SMEM_BYTES, st>>>(mQ, mKC, mKS, mV, mG, mO, p);
  else tc_attn::attn_fwd_kernel<false><<<grid, 192, tc_attn::SMEM_BYTES, st>>>(mQ, mKC, mKS, mV, mG, mO, p);
  note_launches(2);
  return check_launch();
}

// bf16 GEMM on the tensor cores when the shapes suit TMA (row strides of
// whole 16-byte units), else the CUDA-core GEMM.  mode 1 writes the per-head
// [K^C_h | V_h] split of an N = H * 256 product.
// N2 > 0 (plain mode, from 256 rows on, N2 % 8 == 0): a second product
// C2 = A B2 [M][N2] runs in the same pair launch (see gemm_bf16_two).
static int gemm_bf16(int M, int N, int K, const __nv_bfloat16* A, const __nv_bfloat16* B, __nv_bfloat16* C,
                     __nv_bfloat16* KC, __nv_bfloat16* V, int H, int d_c, int d_v, int mode, cudaStream_t st,
                     int N2 = 0, const __nv_bfloat16* B2 = nullptr, __nv_bfloat16* C2 = nullptr) {
  const bool tc = (K % 8 == 0) && (N % 8 == 0) && (mode == 0 || (d_c == 128 && d_v == 128));
  if (!tc) {
    if (mode == 1) return simt::gemm<__nv_bfloat16>(M, N, K, A, B, simt::EpiSplitKV<__nv_bfloat16>{KC, V, H, d_c, d_v}, st);
    return simt::gemm<__nv_bfloat16>(M, N, K, A, B, simt::EpiPlain<__nv_bfloat16>{C, N}, st);
  }
  static std::once_flag once[kMaxDevices];
  static cudaError_t attr_err[kMaxDevices];
  const cudaError_t ae = set_attributes_once(once, attr_err, [] {
    cudaError_t e = cudaFuncSetAttribute(tc_gemm::gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tc_gemm::SMEM_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(tc_gemm::gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)tc_gemm::PAIR_SMEM_BYTES);
    return e;
  });
  if (ae != cudaSuccess) return cuda_status(ae);
  CUtensorMap mA, mB, mB2;
  GMLA_TRY(make_map_2d(&mA, A, (uint64_t)K, (uint64_t)M, tc_gemm::BM));
  GMLA_TRY(make_map_2d(&mB, B, (uint64_t)N, (uint64_t)K, tc_gemm::BK));
  mB2 = mB;
  if (N2 > 0) GMLA_TRY(make_map_2d(&mB2, B2, (uint64_t)N2, (uint64_t)K, tc_gemm::BK));
  tc_gemm::Params p;
  p.M = M; p.N = N; p.K = K; p.C = C; p.KC = KC; p.V = V; p.H = H; p.mode = mode; p.N2 = N2;
  // Persistent: one CTA per SM (never more CTAs than output tiles); from 256
  // rows on, CTA pairs on 256 x 256 tiles.
  int dev = 0, sms = 0;
  GMLA_TRY(cuda_status(cudaGetDevice(&dev)));
  GMLA_TRY(cuda_status(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)));
  const long long tiles_n = (N + tc_gemm::BN - 1) / tc_gemm::BN + (N2 + tc_gemm::BN - 1) / tc_gemm::BN;
  if (M >= tc_gemm::PAIR_BM) {
    const long long tiles = tiles_n * ((M + tc_gemm::PAIR_BM - 1) / tc_gemm::PAIR_BM);
    const unsigned pairs = (unsigned)std::max<long long>(1, std::min<long long>(tiles, sms / 2));
    // Output maps for the epilogue's tile stores: C (and C2), or K^C and V as [M][H * 128].
    CUtensorMap mC0, mC1;
    if (mode == 1) {
      GMLA_TRY(make_map_2d(&mC0, KC, (uint64_t)H * 128, (uint64_t)M, 32));
      GMLA_TRY(make_map_2d(&mC1, V, (uint64_t)H * 128, (uint64_t)M, 32));
    } else {
      GMLA_TRY(make_map_2d(&mC0, C, (uint64_t)N, (uint64_t)M, 32));
      mC1 = mC0;
      if (N2 > 0) GMLA_TRY(make_map_2d(&mC1, C2, (uint64_t)N2, (uint64_t)M, 32));
    }
    tc_gemm::gemm_pair_kernel<<<2 * pairs, 192, tc_gemm::PAIR_SMEM_BYTES, st>>>(mA, mB, mB2, mC0, mC1, p);
  } else {
    if (N2 > 0) return GMLA_EINVAL;              // the caller runs the two products separately here
    const long long tiles = tiles_n * ((M + tc_gemm::BM - 1) / tc_gemm::BM);
    const unsigned grid = (unsigned)std::max<long long>(1, std::min<long long>(tiles, sms));
    tc_gemm::gemm_kernel<<<grid, 192, tc_gemm::SMEM_BYTES, st>>>(mA, mB, p);
  }
  note_launches(1);
  return check_launch();
}

// C1 = A B1 [M][N1] and C2 = A B2 [M][N2], both plain: one pair launch over
// the column tiles of both products when it applies (A read once, one last
// wave for both), else two launches.
static int gemm_bf16_two(int M, int N1, int N2, int K, const __nv_bfloat16* A, const __nv_bfloat16* B1,
                         __nv_bfloat16* C1, const __nv_bfloat16* B2, __nv_bfloat16* C2, cudaStream_t st) {
  if (M >= tc_gemm::PAIR_BM && K % 8 == 0 && N1 % 8 == 0 && N2 % 8 == 0)
    return gemm_bf16(M, N1, K, A, B1, C1, nullptr, nullptr, 0, 0, 0, 0, st, N2, B2, C2);
  GMLA_TRY(gemm_bf16(M, N1, K, A, B1, C1, nullptr, nullptr, 0, 0, 0, 0, st));
  return gemm_bf16(M, N2, K, A, B2, C2, nullptr, nullptr, 0, 0, 0, 0, st);
}

template <typename T>
int up_proj_impl(const gmla_geom* g, int B, int Tn, const T* x, const T* W_DQ, const T* w_q,
                        const T* W_UQ, const T* W_DKV, const T* w_kv, const T* W_UKV, T* Q, T* KC, T* kS,
                        T* V, T* cache, void* ws, cudaStream_t st) {
  const int M = B * Tn;
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  char* p = static_cast<char*>(ws);
  T* cQ = reinterpret_cast<T*>(p);           p += al((size_t)M * g->q_lora * sizeof(T));
  T* cQh = reinterpret_cast<T*>(p);          p += al((size_t)M * g->q_lora * sizeof(T));
  T* ckv = reinterpret_cast<T*>(p);          p += al((size_t)M * (g->kv_lora + g->d_s) * sizeof(T));
  T* ckvh = reinterpret_cast<T*>(p);
  const int d_qk = g->d_c + g->d_s;
  auto plain = [&](int Mm, int N, int K, const T* A, const T* B, T* C) -> int {
    if constexpr (std::is_same<T, __nv_bfloat16>::value)
      return gemm_bf16(Mm, N, K, A, B, C, nullptr, nullptr, 0, 0, 0, 0, st);
    else
      return simt::gemm<T>(Mm, N, K, A, B, simt::EpiPlain<T>{C, N}, st);
  };
  // The two products of x: c^Q = x W_DQ and [c^KV k^S] = x W_DKV.
  constexpr bool bf = std::is_same<T, __nv_bfloat16>::value;
  if constexpr (bf) {
    GMLA_TRY(gemm_bf16_two(M, g->q_lora, g->kv_lora + g->d_s, g->d_model, x, W_DQ, cQ, W_DKV, ckv, st));
  } else {
    GMLA_TRY(plain(M, g->q_lora, g->d_model, x, W_DQ, cQ));
    GMLA_TRY(plain(M, g->kv_lora + g->d_s, g->d_model, x, W_DKV, ckv));
  }
  // bf16 K3 widths: one warp per row (simt.cuh); otherwise one block per row.
  if constexpr (bf) {
    if (g->q_lora == 1536)
      simt::norm_rows_bf16_kernel<6><<<(M + 7) / 8, 256, 0, st>>>(cQ, M, w_q, g->rms_eps, cQh);
    else
      simt::norm_rows_kernel<T><<<M, 256, 0, st>>>(cQ, g->q_lora, w_q, g->rms_eps, cQh);
  } else {
    simt::norm_rows_kernel<T><<<M, 256, 0, st>>>(cQ, g->q_lora, w_q, g->rms_eps, cQh);
  }
  note_launches(1);
  GMLA_TRY(plain(M, g->H * d_qk, g->q_lora, cQh, W_UQ, Q));
  if constexpr (bf) {
    if (g->kv_lora == 512 && g->d_s == 64)
      simt::norm_kv_rows_bf16_kernel<2><<<(M + 7) / 8, 256, 0, st>>>(ckv, M, w_kv, g->rms_eps, ckvh, kS, cache);
    else
      simt::norm_kv_rows_kernel<T><<<M, 256, 0, st>>>(ckv, g->kv_lora, g->d_s, w_kv, g->rms_eps, ckvh, kS, cache);
  } else {
    simt::norm_kv_rows_kernel<T><<<M, 256, 0, st>>>(ckv, g->kv_lora, g->d_s, w_kv, g->rms_eps, ckvh, kS, cache);
  }
  note_launches(1);
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    GMLA_TRY(gemm_bf16(M, g->H * (g->d_c + g->d_v), g->kv_lora, ckvh, W_UKV, nullptr, KC, V, g->H, g->d_c, g->d_v, 1, st));
  } else {
    GMLA_TRY(simt::gemm<T>(M, g->H * (g->d_c + g->d_v), g->kv_lora, ckvh, W_UKV,
                           simt::EpiSplitKV<T>{KC, V, g->H, g->d_c, g->d_v}, st));
  }
  return check_launch();
}

// ---------------------------------------------------------------------------
// Fixed scratch of the non-allocating decode entry point.  The array is part
// of the library's device image: every GPU that loads the library holds these
// bytes until the process exits.  In host code the symbol is only a handle;
// its device address is fetched with cudaGetSymbolAddress once per device,
// with that device current, and cached here.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;   // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
static std::mutex g_noalloc_mu;
static void* g_noalloc_ptr[kMaxDevices] = {};

static int noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (dev < 0 || dev >= kMaxDevices) return GMLA_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_status(e);
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return GMLA_OK;
}

}  // namespace gmla

using namespace gmla;

// ===========================================================================
// extern "C" entry points
// ===========================================================================
extern "C" {

int gmla_version(void) { return 100; }

unsigned long long gmla_launch_count(void) { return g_launches.load(); }

int gmla_last_cuda_error(void) { return g_last_cuda_error; }

const char* gmla_strerror(int s) {
  switch (s) {
    case GMLA_OK: return "ok";
    case GMLA_EINVAL: return "invalid argument";
    case GMLA_EALIGN: return "tensor pointer not 16-byte aligned";
    case GMLA_EUNSUPPORTED: return "unsupported shape or dtype for this build";
    case GMLA_ECUDA: return "CUDA error";
    case GMLA_ETIMEOUT: return "device-side wait timed out";
    case GMLA_EWORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int gmla_set_wait_limit_ns(unsigned long long ns) {
  const uint64_t v = ns == 0 ? kWaitLimitNs : (uint64_t)ns;
  return cuda_status(cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)));
}

int gmla_selftest_wait(unsigned long long* elapsed, void* stream) {
  if (!elapsed) return GMLA_EINVAL;
  selftest::wait_kernel<<<1, 64, 0, as_stream(stream)>>>(elapsed);
  note_launches(1);
  return check_launch();
}

int gmla_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return cuda_status(e);
  int flag = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&flag, g_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_status(e);
  if (flag != 0) {
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_status(e);
    return flag;
  }
  return GMLA_OK;
}

// ---------------------------------------------------------------------------
size_t mla_up_proj_workspace(const gmla_geom* g, gmla_dtype dtype, int B, int T) {
  if (check_geom(g) != GMLA_OK || check_dtype(dtype) != GMLA_OK || B <= 0 || T <= 0) return 0;
  const size_t M = (size_t)B * T, es = dsize(dtype);
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return al(M * g->q_lora * es) * 2 + al(M * (g->kv_lora + g->d_s) * es) + al(M * g->kv_lora * es);
}

int mla_up_proj(const gmla_geom* g, gmla_dtype dtype, int B, int T, const void* x, const void* W_DQ,
                const void* w_q, const void* W_UQ, const void* W_DKV, const void* w_kv, const void* W_UKV,
                void* Q, void* KC, void* kS, void* V, void* cache, void* workspace, size_t workspace_bytes,
                void* stream) {
  GMLA_TRY(check_geom(g));
  GMLA_TRY(check_dtype(dtype));
  if (B <= 0 || T <= 0) return GMLA_EINVAL;
  GMLA_REQUIRE(x); GMLA_REQUIRE(W_DQ); GMLA_REQUIRE(w_q); GMLA_REQUIRE(W_UQ); GMLA_REQUIRE(W_DKV);
  GMLA_REQUIRE(w_kv); GMLA_REQUIRE(W_UKV); GMLA_REQUIRE(Q); GMLA_REQUIRE(KC); GMLA_REQUIRE(kS); GMLA_REQUIRE(V);
  GMLA_OPTIONAL(cache);
  if (!workspace || workspace_bytes < mla_up_proj_workspace(g, dtype, B, T)) return GMLA_EWORKSPACE;
  if (!aligned16(workspace)) return GMLA_EALIGN;
  cudaStream_t st = as_stream(stream);
  if (dtype == GMLA_F32)
    return up_proj_impl<float>(g, B, T, (const float*)x, (const float*)W_DQ, (const float*)w_q,
                               (const float*)W_UQ, (const float*)W_DKV, (const float*)w_kv, (const float*)W_UKV,
                               (float*)Q, (float*)KC, (float*)kS, (float*)V, (float*)cache, workspace, st);
  using bf = __nv_bfloat16;
  return up_proj_impl<bf>(g, B, T, (const bf*)x, (const bf*)W_DQ, (const bf*)w_q, (const bf*)W_UQ,
                          (const bf*)W_DKV, (const bf*)w_kv, (const bf*)W_UKV, (bf*)Q, (bf*)KC, (bf*)kS, (bf*)V,
                          (bf*)cache, workspace, st);
}

// ---------------------------------------------------------------------------
int mla_attn_fwd(const gmla_geom* g, gmla_dtype dtype, int B, int T, const void* Q, const void* KC,
                 const void* kS, const void* V, const void* gate, void* O, float* maxlogit, void* stream) {
  GMLA_TRY(check_geom(g));
  GMLA_TRY(check_dtype(dtype));
  if (B <= 0 || T <= 0) return GMLA_EINVAL;
  GMLA_REQUIRE(Q); GMLA_REQUIRE(KC); GMLA_REQUIRE(V); GMLA_REQUIRE(O); GMLA_REQUIRE(maxlogit);
  if (g->d_s > 0) GMLA_REQUIRE(kS);
  GMLA_OPTIONAL(gate);
  cudaStream_t st = as_stream(stream);
  if (dtype == GMLA_BF16 && is_k3_head_geometry(g)) {
    if ((long long)B * T * g->H * 192 >= (1LL << 40)) return GMLA_EUNSUPPORTED;
    return attn_fwd_tc(g, B, T, Q, KC, kS, V, gate, O, false, maxlogit, nullptr, st);
  }
  if (g->d_c + g->d_s > 256 || g->d_v > simt::kAttnMaxDV) return GMLA_EUNSUPPORTED;
  if (dtype == GMLA_F32)
    return simt::attn_fwd<float>(B, T, g->H, g->d_c, g->d_s, g->d_v, (const float*)Q, (const float*)KC,
                                 (const float*)kS, (const float*)V, (const float*)gate, (float*)O, maxlogit, st);
  using bf = __nv_bfloat16;
  return simt::attn_fwd<bf>(B, T, g->H, g->d_c, g->d_s, g->d_v, (const bf*)Q, (const bf*)KC, (const bf*)kS,
                            (const bf*)V, (const bf*)gate, (bf*)O, maxlogit, st);
}

// ---------------------------------------------------------------------------
// Training variant: the same forward with o kept in fp32.
int mla_attn_fwd_train(const gmla_geom* g, gmla_dtype dtype, int B, int T, const void* Q, const void* KC,
                       const void* kS, const void* V, const void* gate, float* O, float* lse, float* maxlogit,
                       void* stream) {
  GMLA_TRY(check_geom(g));
  GMLA_TRY(check_dtype(dtype));
  if (B <= 0 || T <= 0) return GMLA_EINVAL;
  GMLA_REQUIRE(Q); GMLA_REQUIRE(KC); GMLA_REQUIRE(V); GMLA_REQUIRE(O); GMLA_REQUIRE(maxlogit);
  if (g->d_s > 0) GMLA_REQUIRE(kS);
  GMLA_OPTIONAL(gate);
  GMLA_OPTIONAL(lse);
  cudaStream_t st = as_stream(stream);
  if (dtype == GMLA_BF16 && is_k3_head_geometry(g)) {
    if ((long long)B * T * g->H * 192 >= (1LL << 40)) return GMLA_EUNSUPPORTED;
    return attn_fwd_tc(g, B, T, Q, KC, kS, V, gate, O, true, maxlogit, lse, st);
  }
  if (g->d_c + g->d_s > 256 || g->d_v > simt::kAttnMaxDV) return GMLA_EUNSUPPORTED;
  if (dtype == GMLA_F32)
    return simt::attn_fwd<float>(B, T, g->H, g->d_c, g->d_s, g->d_v, (const float*)Q, (const float*)KC,
                                 (const float*)kS, (const float*)V, (const float*)gate, O, maxlogit, st, lse);
  using bf = __nv_bfloat16;
  return simt::attn_fwd<bf, float>(B, T, g->H, g->d_c, g->d_s, g->d_v, (const bf*)Q, (const bf*)KC, (const bf*)kS,
                                   (const bf*)V, (const bf*)gate, O, maxlogit, st, lse);
}

// ---------------------------------------------------------------------------
// Backward of the training forward.
size_t mla_attn_bwd_workspace(const gmla_geom* g, int B, int T) {
  if (check_geom(g) != GMLA_OK || B <= 0 || T <= 0) return 0;
  return bwd::workspace_bytes(B, T, g->H, g->d_v);
}

// Backward on the tcgen05 tensor cores (K3 head widths, bf16): the row pass
// (dO~ in bf16 and D into the workspace), then the dK/dV and dQ kernels.
static int attn_bwd_tc(const bwd::Dims& d, const __nv_bfloat16* Q, const __nv_bfloat16* KC,
                       const __nv_bfloat16* kS, const __nv_bfloat16* V, const __nv_bfloat16* gate, const float* O,
                       const float* lse, const float* dO, float* dQ, float* dKC, float* dkS, float* dV, float* dg,
                       void* ws, cudaStream_t st) {
  static std::once_flag once[kMaxDevices];
  static cudaError_t attr_err[kMaxDevices];
  const cudaError_t ae = set_attributes_once(once, attr_err, [] {
    cudaError_t e = cudaFuncSetAttribute(tc_bwd::dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tc_bwd::kv::SMEM_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(tc_bwd::dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)tc_bwd::q::SMEM_BYTES);
    return e;
  });
  if (ae != cudaSuccess) return cuda_status(ae);
  using bf = __nv_bfloat16;
  const int B = d.B, T = d.T, H = d.H;
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  bf* dOt = static_cast<bf*>(ws);
  float* D = reinterpret_cast<float*>(static_cast<char*>(ws) + al((size_t)B * T * H * 128 * 4));
  // 64-row boxes for the tiles a CTA walks, 128-row boxes for its resident tile.
  CUtensorMap mQ64, mDO64, mKC128, mKS128, mV128, mQ128, mDO128, mKC64, mKS64, mV64;
  GMLA_TRY(make_map_3d(&mQ64, Q, (uint64_t)H * 192, T, B, 64));
  GMLA_TRY(make_map_3d(&mDO64, dOt, (uint64_t)H * 128, T, B, 64));
  GMLA_TRY(make_map_3d(&mKC128, KC, (uint64_t)H * 128, T, B, 128));
  GMLA_TRY(make_map_3d(&mKS128, kS, 64, T, B, 128));
  GMLA_TRY(make_map_3d(&mV128, V, (uint64_t)H * 128, T, B, 128));
  GMLA_TRY(make_map_3d(&mQ128, Q, (uint64_t)H * 192, T, B, 128));
  GMLA_TRY(make_map_3d(&mDO128, dOt, (uint64_t)H * 128, T, B, 128));
  GMLA_TRY(make_map_3d(&mKC64, KC, (uint64_t)H * 128, T, B, 64));
  GMLA_TRY(make_map_3d(&mKS64, kS, 64, T, B, 64));
  GMLA_TRY(make_map_3d(&mV64, V, (uint64_t)H * 128, T, B, 64));
  GMLA_TRY(cuda_status(cudaMemsetAsync(dkS, 0, (size_t)B * T * 64 * sizeof(float), st)));
  const int rows = B * T * H;
  bwd::row128_kernel<<<(rows + 7) / 8, 256, 0, st>>>(rows, O, dO, static_cast<const bf*>(gate), dOt, D, dg);
  tc_bwd::Params p;
  p.B = B; p.T = T; p.H = H; p.lse = lse; p.D = D; p.dQ = dQ; p.dKC = dKC; p.dkS = dkS; p.dV = dV;
  p.scale = d.scale;
  p.scale_log2 = (float)(1.4426950408889634 * (double)d.scale);
  const int nt = (T + 127) / 128;
  tc_bwd::dkdv_kernel<<<dim3(nt, H, B), 192, tc_bwd::kv::SMEM_BYTES, st>>>(mQ64, mDO64, mKC128, mKS128, mV128, p);
  tc_bwd::dq_kernel<<<dim3(nt, H, B), 192, tc_bwd::q::SMEM_BYTES, st>>>(mQ128, mDO128, mKC64, mKS64, mV64, p);
  note_launches(3);
  return check_launch();
}

int mla_attn_bwd(const gmla_geom* g, gmla_dtype dtype, int B, int T, const void* Q, const void* KC, const void* kS,
                 const void* V, const void* gate, const float* O, const float* lse, const float* dO, float* dQ,
                 float* dKC, float* dkS, float* dV, float* dg, void* workspace, size_t workspace_bytes,
                 void* stream) {
  GMLA_TRY(check_geom(g));
  GMLA_TRY(check_dtype(dtype));
  if (B <= 0 || T <= 0) return GMLA_EINVAL;
  GMLA_REQUIRE(Q); GMLA_REQUIRE(KC); GMLA_REQUIRE(V); GMLA_REQUIRE(O); GMLA_REQUIRE(lse); GMLA_REQUIRE(dO);
  GMLA_REQUIRE(dQ); GMLA_REQUIRE(dKC); GMLA_REQUIRE(dV);
  if (g->d_s > 0) { GMLA_REQUIRE(kS); GMLA_REQUIRE(dkS); }
  GMLA_OPTIONAL(gate);
  if (gate) GMLA_REQUIRE(dg);
  if (g->d_c + g->d_s > bwd::kMaxD || g->d_v > bwd::kMaxD) return GMLA_EUNSUPPORTED;
  if (!workspace || workspace_bytes < bwd::workspace_bytes(B, T, g->H, g->d_v)) return GMLA_EWORKSPACE;
  if (!aligned16(workspace)) return GMLA_EALIGN;
  cudaStream_t st = as_stream(stream);
  bwd::Dims p{B, T, g->H, g->d_c, g->d_s, g->d_v, 1.f / std::sqrt((float)(g->d_c + g->d_s))};
  if (dtype == GMLA_F32)
    return bwd::run<float>(p, (const float*)Q, (const float*)KC, (const float*)kS, (const float*)V,
                           (const float*)gate, O, lse, dO, dQ, dKC, dkS, dV, dg, workspace, st);
  using bf = __nv_bfloat16;
  if (is_k3_head_geometry(g))
    return attn_bwd_tc(p, (const bf*)Q, (const bf*)KC, (const bf*)kS, (const bf*)V, (const bf*)gate, O, lse, dO, dQ,
                       dKC, dkS, dV, dg, workspace, st);
  return bwd::run<bf>(p, (const bf*)Q, (const bf*)KC, (const bf*)kS, (const bf*)V, (const bf*)gate, O, lse, dO, dQ,
                      dKC, dkS, dV, dg, workspace, st);
}

// ---------------------------------------------------------------------------
int qkclip_rescale(const gmla_geom* g, gmla_dtype dtype, void* W_UQ, void* W_UKV, const float* maxlogit,
                   float tau, unsigned char* clipped, float* gamma, void* stream) {
  GMLA_TRY(check_geom(g));
  GMLA_TRY(check_dtype(dtype));
  GMLA_REQUIRE(W_UQ); GMLA_REQUIRE(W_UKV);
  if (!maxlogit) return GMLA_EINVAL;
  if (!(tau > 0.f) || !std::isfinite(tau)) return GMLA_EINVAL;
  cudaStream_t st = as_stream(stream);
  if (dtype == GMLA_F32)
    return clip::rescale<float>((float*)W_UQ, (float*)W_UKV, g->q_lora, g->kv_lora, g->H, g->d_c, g->d_s, g->d_v,
                                maxlogit, tau, clipped, gamma, st);
  using bf = __nv_bfloat16;
  return clip::rescale<bf>((bf*)W_UQ, (bf*)W_UKV, g->q_lora, g->kv_lora, g->H, g->d_c, g->d_s, g->d_v, maxlogit,
                           tau, clipped, gamma, st);
}

// ---------------------------------------------------------------------------
size_t mla_decode_workspace(const gmla_geom* g, gmla_dtype dtype, int n_seq, int max_len) {
  if (check_geom(g) != GMLA_OK || check_dtype(dtype) != GMLA_OK || n_seq <= 0 || max_len <= 0) return 0;
  return decode_ws_bytes(g, dtype, n_seq, max_len);
}

int mla_decode_absorbed(const gmla_geom* g, gmla_dtype dtype, int n_seq, const void* q, const void* W_UKV,
                        const void* cache, const int* seq_offsets, int max_len, const void* gate, void* O,
                        void* workspace, size_t workspace_bytes, void* stream) {
  GMLA_TRY(check_geom(g));
  GMLA_TRY(check_dtype(dtype));
  if (n_seq <= 0 || max_len <= 0) return GMLA_EINVAL;
  GMLA_REQUIRE(q); GMLA_REQUIRE(W_UKV); GMLA_REQUIRE(cache); GMLA_REQUIRE(O);
  if (!seq_offsets) return GMLA_EINVAL;
  GMLA_OPTIONAL(gate);
  if (g->kv_lora > 128 * simt::kDecMaxLatentPerThread) return GMLA_EUNSUPPORTED;
  if (!workspace || workspace_bytes < mla_decode_workspace(g, dtype, n_seq, max_len)) return GMLA_EWORKSPACE;
  if (!aligned16(workspace)) return GMLA_EALIGN;
  cudaStream_t st = as_stream(stream);
  if (dtype == GMLA_BF16 && is_k3_decode_geometry(g))
    return decode_tc(n_seq, q, W_UKV, cache, tc_dec::Windows{seq_offsets, 0}, (uint64_t)n_seq * (uint64_t)max_len,
                     (long long)n_seq * ((max_len + tc_dec::BT - 1) / tc_dec::BT), gate, O, nullptr, workspace, st);
  if (dtype == GMLA_F32)
    return simt::decode<float>(n_seq, g->H, g->d_c, g->d_s, g->d_v, g->kv_lora, (const float*)q,
                               (const float*)W_UKV, (const float*)cache, seq_offsets, max_len, (const float*)gate,
                               (float*)O, workspace, st);
  using bf = __nv_bfloat16;
  return simt::decode<bf>(n_seq, g->H, g->d_c, g->d_s, g->d_v, g->kv_lora, (const bf*)q, (const bf*)W_UKV,
                          (const bf*)cache, seq_offsets, max_len, (const bf*)gate, (bf*)O, workspace, st);
}

// ---------------------------------------------------------------------------
// Prefill on the latent cache: mla_attn_fwd's outputs computed the absorbed
// way, each query over its causal prefix of the cache.
size_t mla_attn_fwd_absorbed_workspace(const gmla_geom* g, int B, int T) {
  if (check_geom(g) != GMLA_OK || !is_k3_decode_geometry(g) || B <= 0 || T <= 0) return 0;
  if ((long long)B * T > (1LL << 24)) return 0;
  return tc_dec::workspace_bytes(B * T);
}

int mla_attn_fwd_absorbed(const gmla_geom* g, gmla_dtype dtype, int B, int T, const void* Q, const void* W_UKV,
                          const void* cache, const void* gate, void* O, float* maxlogit, void* workspace,
                          size_t workspace_bytes, void* stream) {
  GMLA_TRY(check_geom(g));
  GMLA_TRY(check_dtype(dtype));
  if (B <= 0 || T <= 0) return GMLA_EINVAL;
  GMLA_REQUIRE(Q); GMLA_REQUIRE(W_UKV); GMLA_REQUIRE(cache); GMLA_REQUIRE(O); GMLA_REQUIRE(maxlogit);
  GMLA_OPTIONAL(gate);
  if (dtype != GMLA_BF16 || !is_k3_decode_geometry(g)) return GMLA_EUNSUPPORTED;
  if ((long long)B * T > (1LL << 24)) return GMLA_EUNSUPPORTED;
  if (!workspace || workspace_bytes < mla_attn_fwd_absorbed_workspace(g, B, T)) return GMLA_EWORKSPACE;
  if (!aligned16(workspace)) return GMLA_EALIGN;
  cudaStream_t st = as_stream(stream);
  const int n = B * T;
  // Query b*T + t reads rows b*T .. b*T + t: ceil((t+1) / 96) tiles each.
  long long tiles = 0;
  for (int t = 0; t < T; ++t) tiles += (t + tc_dec::BT) / tc_dec::BT;
  simt::fill_kernel<<<(g->H + 127) / 128, 128, 0, st>>>(maxlogit, g->H, -INFINITY);
  note_launches(1);
  GMLA_TRY(check_launch());
  return decode_tc(n, Q, W_UKV, cache, tc_dec::Windows{nullptr, T}, (uint64_t)n, tiles * B, gate, O, maxlogit,
                   workspace, st);
}

// ---------------------------------------------------------------------------
int mla_gemm(gmla_dtype dtype, int M, int N, int K, const void* A, const void* B, void* C, void* stream) {
  GMLA_TRY(check_dtype(dtype));
  if (M <= 0 || N <= 0 || K <= 0) return GMLA_EINVAL;
  GMLA_REQUIRE(A); GMLA_REQUIRE(B); GMLA_REQUIRE(C);
  cudaStream_t st = as_stream(stream);
  if (dtype == GMLA_F32)
    return simt::gemm<float>(M, N, K, (const float*)A, (const float*)B, simt::EpiPlain<float>{(float*)C, N}, st);
  using bf = __nv_bfloat16;
  return gemm_bf16(M, N, K, (const bf*)A, (const bf*)B, (bf*)C, nullptr, nullptr, 0, 0, 0, 0, st);
}

// ---------------------------------------------------------------------------
// Decode without a caller workspace: the same kernels as the CUDA-core path of
// mla_decode_absorbed, run on the library's fixed device scratch.  No device
// memory is allocated; a request whose scratch need exceeds the fixed size is
// refused with GMLA_EWORKSPACE before anything is enqueued.  Every scratch
// byte the kernels read is written earlier in the same call, so nothing has
// to be cleared between calls.
int mla_decode_absorbed_noalloc(const gmla_geom* g, gmla_dtype dtype, int n_seq, const void* q,
                                const void* W_UKV, const void* cache, const int* seq_offsets, int max_len,
                                const void* gate, void* O, void* stream) {
  GMLA_TRY(check_geom(g));
  GMLA_TRY(check_dtype(dtype));
  if (n_seq <= 0 || max_len <= 0) return GMLA_EINVAL;
  GMLA_REQUIRE(q); GMLA_REQUIRE(W_UKV); GMLA_REQUIRE(cache); GMLA_REQUIRE(O);
  if (!seq_offsets) return GMLA_EINVAL;
  GMLA_OPTIONAL(gate);
  if (g->kv_lora > 128 * simt::kDecMaxLatentPerThread) return GMLA_EUNSUPPORTED;
  if (simt::decode_workspace(g->H, g->kv_lora, g->d_s, n_seq, max_len) > kNoAllocScratchBytes)
    return GMLA_EWORKSPACE;
  void* ws = nullptr;
  GMLA_TRY(noalloc_scratch(&ws));
  cudaStream_t st = as_stream(stream);
  if (dtype == GMLA_F32)
    return simt::decode<float>(n_seq, g->H, g->d_c, g->d_s, g->d_v, g->kv_lora, (const float*)q,
                               (const float*)W_UKV, (const float*)cache, seq_offsets, max_len, (const float*)gate,
                               (float*)O, ws, st);
  using bf = __nv_bfloat16;
  return simt::decode<bf>(n_seq, g->H, g->d_c, g->d_s, g->d_v, g->kv_lora, (const bf*)q, (const bf*)W_UKV,
                          (const bf*)cache, seq_offsets, max_len, (const bf*)gate, (bf*)O, ws, st);
}

}  // extern "C"
