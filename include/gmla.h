/*
 * gmla.h — C ABI of libgmla.so: gated multi-head latent attention (MLA) for
 * NVIDIA B200 (sm_100a), with the per-head max logit fused into the forward,
 * the QK-Clip weight rescale and the latent-absorbed decode.
 *
 * Notation and shapes follow "Kimi K3 · Gated MLA · OpenModelAtlas", section
 * "All 20 steps": y = x W with row-major weights W[in][out]; per head h the
 * query is [q^C_h (d_c) | q^S_h (d_s)], the key K_h = [K^C_h (d_c) | k^S (d_s)]
 * with k^S shared by every head, the value V_h (d_v); logits are
 * S = Q K^T / sqrt(d_c + d_s).  Kimi K3's geometry ("Gated MLA et NoPE",
 * "Récapitulatif des couches Gated MLA"): H = 96, d_model = 7168,
 * q_lora = 1536, kv_lora = 512, d_c = 128, d_s = 64, d_v = 128.
 *
 * Conventions shared by every entry point
 *   - Pointers named as tensors are DEVICE pointers, row-major and contiguous,
 *     owned by the caller; the library allocates nothing and keeps no pointer
 *     after the call returns.  `geom` is a host pointer read during the call.
 *   - Element type is chosen by `dtype`: GMLA_BF16 (bf16 storage, fp32
 *     accumulation) or GMLA_F32 (fp32 storage and arithmetic).  maxlogit and
 *     gamma are always float32, clipped is uint8, seq_offsets int32.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *     enqueued on it asynchronously; nothing synchronises the host.
 *   - Every tensor pointer must be 16-byte aligned (GMLA_EALIGN otherwise).
 *   - Arguments are validated on the host before anything is launched; on a
 *     negative return nothing was enqueued.  GMLA_ECUDA means a launch failed
 *     (gmla_last_cuda_error() gives the cudaError_t).  Device-side waits are
 *     bounded; a wait that gives up records GMLA_ETIMEOUT in a device flag
 *     read by gmla_device_status().  Nothing is printed and no C++ exception
 *     crosses this boundary.
 */
#ifndef GMLA_H
#define GMLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GMLA_OK = 0,
  GMLA_EINVAL = -1,        /* null pointer, non-positive size, bad geometry */
  GMLA_EALIGN = -2,        /* a tensor pointer is not 16-byte aligned */
  GMLA_EUNSUPPORTED = -3,  /* valid arguments this build has no kernel for */
  GMLA_ECUDA = -4,         /* a CUDA launch or runtime call failed */
  GMLA_ETIMEOUT = -5,      /* a bounded device-side wait gave up */
  GMLA_EWORKSPACE = -6     /* workspace pointer NULL or smaller than required */
} gmla_status;

typedef enum { GMLA_BF16 = 0, GMLA_F32 = 1 } gmla_dtype;

typedef struct {
  int H;        /* attention heads */
  int d_model;  /* model width d */
  int q_lora;   /* query latent rank */
  int kv_lora;  /* key/value latent rank */
  int d_c;      /* per-head content query/key width (qk_nope_head_dim) */
  int d_s;      /* shared key width k^S (qk_rope_head_dim, unrotated) */
  int d_v;      /* per-head value width */
  float rms_eps;
} gmla_geom;

/* Bytes of scratch mla_up_proj needs for B*T tokens. */
size_t mla_up_proj_workspace(const gmla_geom* geom, gmla_dtype dtype, int B, int T);

/*
 * mla_up_proj — queries, content keys, shared key and values from x.
 * Defined by "Kimi K3 · Gated MLA · OpenModelAtlas", "All 20 steps" (query
 * heads; key and value heads):
 *   c^Q = x W_DQ;  q = RMSNorm_{w_q}(c^Q) W_UQ
 *   [c^KV | k^S] = x W_DKV;  [K^C_h | V_h]_h = RMSNorm_{w_kv}(c^KV) W_UKV
 * RMSNorm(c) = c / sqrt(mean(c^2) + rms_eps) * w, computed in fp32; k^S is not
 * normalised.  Each projection/norm output is rounded to `dtype`.
 *   x      [B*T][d_model]              W_DQ  [d_model][q_lora]    w_q  [q_lora]
 *   W_UQ   [q_lora][H*(d_c+d_s)]       W_DKV [d_model][kv_lora+d_s]
 *   w_kv   [kv_lora]                   W_UKV [kv_lora][H*(d_c+d_v)] (head h: K^C cols then V cols)
 * Outputs (written, not accumulated):
 *   Q  [B*T][H][d_c+d_s]   KC [B*T][H][d_c]   kS [B*T][d_s]   V [B*T][H][d_v]
 *   cache (nullable) [B*T][kv_lora+d_s] = [RMSNorm(c^KV) | k^S], the decode latent.
 * workspace: device scratch of at least mla_up_proj_workspace() bytes.
 */
int mla_up_proj(const gmla_geom* geom, gmla_dtype dtype, int B, int T,
                const void* x, const void* W_DQ, const void* w_q, const void* W_UQ,
                const void* W_DKV, const void* w_kv, const void* W_UKV,
                void* Q, void* KC, void* kS, void* V, void* cache,
                void* workspace, size_t workspace_bytes, void* stream);

/*
 * mla_attn_fwd — causal gated attention and the per-head max logit.
 * Defined by "Kimi K3 · Gated MLA · OpenModelAtlas", "All 20 steps" (causal
 * attention, output gate) and, for the statistic, "Anthology of the SOTA"
 * record SOTA-131 ("Source", "Conditions": the per-head max-logit check).
 *   S_h = [Q^C_h | Q^S_h] [K^C_h | k^S]^T / sqrt(d_c+d_s)
 *   A = softmax over s <= t (fp32);  O_h = A V_h;  o = sigmoid(g) * o (g nullable = no gate)
 *   maxlogit[h] = max over b, t and s <= t of S_h[t][s]   (scaled logit)
 *   Q [B][T][H][d_c+d_s]   KC [B][T][H][d_c]   kS [B][T][d_s]   V [B][T][H][d_v]
 *   g [B][T][H*d_v] or NULL;  O [B][T][H*d_v] (written)
 *   maxlogit: device float[H], overwritten (the call resets it first).
 * bf16 with d_c=128, d_s=64, d_v=128 runs the tcgen05/TMA kernel; other shapes
 * (d_c+d_s <= 256, d_v <= 256) and fp32 run the CUDA-core kernel.
 */
int mla_attn_fwd(const gmla_geom* geom, gmla_dtype dtype, int B, int T,
                 const void* Q, const void* KC, const void* kS, const void* V,
                 const void* g, void* O, float* maxlogit, void* stream);

/*
 * mla_attn_fwd_train — the same forward with the output kept in fp32, the
 * training form of "Gated MLA et NoPE", "Un détail de précision numérique"
 * (the attention output stays in FP32 during training, so no biased
 * rounding of o to bf16).  Arguments, layouts, ownership and errors are those
 * of mla_attn_fwd except:
 *   O [B][T][H*d_v] float32 (written) whatever `dtype` is;
 *   lse (nullable) [B][T][H] float32 (written): log sum_{s<=t} exp S_h[t][s]
 *     of the scaled logits, the row statistic mla_attn_bwd recomputes A from.
 * bf16 with d_c=128, d_s=64, d_v=128 runs the tcgen05/TMA kernel (its epilogue
 * stores from registers: no output tile is staged in shared memory); other
 * shapes and fp32 inputs run the CUDA-core kernel with fp32 output.
 */
int mla_attn_fwd_train(const gmla_geom* geom, gmla_dtype dtype, int B, int T,
                       const void* Q, const void* KC, const void* kS, const void* V,
                       const void* g, float* O, float* lse, float* maxlogit, void* stream);

/* Bytes of scratch mla_attn_bwd needs (0 for a bad geometry or size). */
size_t mla_attn_bwd_workspace(const gmla_geom* geom, int B, int T);

/*
 * mla_attn_bwd — gradients of a loss L through the forward above (the layer
 * is trained: "Anthology of the SOTA" SOTA-131 "Source" clips it during
 * training; "Gated MLA et NoPE", "Un détail de précision numérique").  With
 * the forward of mla_attn_fwd ("Kimi K3 · Gated MLA · OpenModelAtlas",
 * "All 20 steps") and A_ts = exp(S_ts - lse_t) for s <= t:
 *   dO~ = dO * sigmoid(g);  dg = dO * o * (1 - sigmoid(g));  D_t = sum_c dO * o
 *   dS = A * (dO~ V_h^T - D);  dQ_h = dS K_h / sqrt(d_qk);  dV_h = A^T dO~
 *   dK_h = dS^T Q_h / sqrt(d_qk) -> dKC (first d_c columns), and dkS = the
 *   sum over heads of the last d_s columns (k^S is shared by every head).
 * Inputs: Q, KC, kS, V, g as for mla_attn_fwd, in `dtype`; O (= o) and lse
 *   from mla_attn_fwd_train; dO = dL/do [B][T][H*d_v] float32.
 * Outputs (written, not accumulated), float32 in the layouts of the inputs:
 *   dQ [B][T][H][d_c+d_s], dKC [B][T][H][d_c], dkS [B][T][d_s],
 *   dV [B][T][H][d_v], dg [B][T][H*d_v] (required when g is given).
 * workspace: device scratch of at least mla_attn_bwd_workspace() bytes.
 * bf16 with d_c=128, d_s=64, d_v=128 runs the tcgen05/TMA kernels (A and dS
 * enter the tensor-core products in bf16, accumulation in fp32); other shapes
 * (d_c+d_s <= 256, d_v <= 256) and fp32 run CUDA-core kernels in fp32.
 * dkS is zeroed on `stream` before the heads' contributions are added.
 */
int mla_attn_bwd(const gmla_geom* geom, gmla_dtype dtype, int B, int T,
                 const void* Q, const void* KC, const void* kS, const void* V, const void* g,
                 const float* O, const float* lse, const float* dO,
                 float* dQ, float* dKC, float* dkS, float* dV, float* dg,
                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * qkclip_rescale — QK-Clip applied to the weights, in place.
 * "Anthology of the SOTA" record SOTA-131, "Source": after a step, for each
 * head whose max logit exceeds the threshold, rescale that head's query and
 * key projection weights so it no longer does.  For head h with
 * maxlogit[h] > tau (strict): gamma_h = tau / maxlogit[h] (IEEE fp32 divide),
 *   W_UQ  cols h*(d_c+d_s) + [0, d_c)        *= sqrt(gamma_h)   (q^C_h)
 *   W_UQ  cols h*(d_c+d_s) + [d_c, d_c+d_s)  *= gamma_h         (q^S_h, meets shared k^S)
 *   W_UKV cols h*(d_c+d_v) + [0, d_c)        *= sqrt(gamma_h)   (K^C_h)
 * so every logit of head h scales by gamma_h; k^S (W_DKV) and V are untouched.
 * Each new weight is one fp32 product rounded to `dtype` (RNE): bit-exact.
 *   W_UQ [q_lora][H*(d_c+d_s)], W_UKV [kv_lora][H*(d_c+d_v)]: modified in place
 *   maxlogit: device float[H];  tau > 0
 *   clipped (nullable): device uint8[H] <- 1 if head clipped else 0
 *   gamma   (nullable): device float[H] <- gamma_h, or 1 for unclipped heads
 * Only the clipped heads' columns are read and written.
 */
int qkclip_rescale(const gmla_geom* geom, gmla_dtype dtype, void* W_UQ, void* W_UKV,
                   const float* maxlogit, float tau, unsigned char* clipped, float* gamma,
                   void* stream);

/* Bytes of scratch mla_decode_absorbed needs for n_seq sequences of at most max_len tokens. */
size_t mla_decode_workspace(const gmla_geom* geom, gmla_dtype dtype, int n_seq, int max_len);

/*
 * mla_decode_absorbed — one new query token per sequence over its latent cache.
 * "Kimi Qkclip" (Fireworks blog), section 3 (training materialises per-head
 * keys; decoding works on the cached latent), and "Gated MLA et NoPE",
 * "Le principe" (cache of kv_lora + d_s values per token).  W_UK,h / W_UV,h are
 * head h's K^C / V column blocks of W_UKV.
 *   q~_h = [q^C_h W_UK,h^T | q^S_h]          (absorbed query, kv_lora + d_s)
 *   s_j  = q~_h . cache_j / sqrt(d_c+d_s);   p = softmax over all cached j
 *   o_h  = (sum_j p_j cache_j[0:kv_lora]) W_UV,h,  then * sigmoid(g) if g != NULL
 * Equal (up to rounding) to attention over materialised keys
 * [cache_j[0:kv_lora] W_UK,h | cache_j[kv_lora:]] and values cache_j[0:kv_lora] W_UV,h.
 *   q [n_seq][H][d_c+d_s];  W_UKV [kv_lora][H*(d_c+d_v)]
 *   cache [total][kv_lora+d_s], sequence i = rows seq_offsets[i] .. seq_offsets[i+1]-1
 *   seq_offsets: device int32[n_seq+1], non-decreasing, seq_offsets[0] = 0,
 *     every length in [0, max_len].  A sequence of length 0 (an empty cache,
 *     e.g. a free serving slot) gets an output row of zeros and does not
 *     change any other sequence's output.  The offsets are device memory, so
 *     the host does not check them; a length above max_len leaves every
 *     sequence's output undefined (reads stay inside the cache rows the
 *     offsets name).
 *   g [n_seq][H*d_v] or NULL;  O [n_seq][H][d_v] (written)
 *   workspace: at least mla_decode_workspace() bytes.
 */
int mla_decode_absorbed(const gmla_geom* geom, gmla_dtype dtype, int n_seq,
                        const void* q, const void* W_UKV, const void* cache,
                        const int* seq_offsets, int max_len, const void* g, void* O,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * mla_attn_fwd_absorbed — mla_attn_fwd's outputs (O and maxlogit[H]) computed
 * on the latent cache instead of the materialised keys and values: every
 * query is absorbed (q~_h = [q^C_h W_UK,h^T | q^S_h], 576 wide) and attends to
 * the cache rows of its causal prefix, and the latent-space output is
 * projected by W_UV,h.  This is the inference form of "Kimi Qkclip" (Fireworks
 * blog), section 3, "Training vs. Inference in Multi-Head Latent Attention",
 * applied to a prefill: K^C and V are never written to memory, at the price of
 * (576 + 512) instead of (192 + 128) multiply-adds per query, key and head.
 *   Q      [B][T][H][d_c + d_s]   W_UKV [kv_lora][H*(d_c+d_v)]
 *   cache  [B][T][kv_lora + d_s] = [RMSNorm(c^KV) | k^S]  (mla_up_proj's `cache`)
 *   g [B][T][H*d_v] or NULL;  O [B][T][H*d_v] (written)
 *   maxlogit: device float[H], overwritten with max over b, t, s <= t of the
 *     scaled logit, as mla_attn_fwd defines it.
 *   workspace: at least mla_attn_fwd_absorbed_workspace() bytes.
 * bf16 and Kimi K3's decode geometry only (H = 96, kv_lora = 512, d_c = 128,
 * d_s = 64, d_v = 128), B * T <= 2^24; otherwise GMLA_EUNSUPPORTED.
 */
size_t mla_attn_fwd_absorbed_workspace(const gmla_geom* geom, int B, int T);
int mla_attn_fwd_absorbed(const gmla_geom* geom, gmla_dtype dtype, int B, int T, const void* Q,
                          const void* W_UKV, const void* cache, const void* g, void* O, float* maxlogit,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * mla_decode_absorbed_noalloc — mla_decode_absorbed for callers that cannot
 * allocate device memory.  The paper has no counterpart: this is a deployment
 * variant.  Some callers cannot provide a workspace: a serving loop that must
 * not call cudaMalloc / cudaFree on the request path (they can synchronise the
 * whole device and stall other streams), or a plugin whose host framework owns
 * every byte of device memory and hands it no scratch.  This entry point takes
 * the same inputs and outputs as mla_decode_absorbed (minus the workspace) and
 * runs the same CUDA-core decode kernels on a scratch array that is part of
 * the library itself.
 *   Limit: the fixed array holds 16 MiB (16777216 bytes).  This entry point
 *     runs the CUDA-core decode kernels, whose scratch need is (with
 *     S = ceil(max_len / 1024) splits per sequence and each of the first two
 *     parts rounded up to a multiple of 256 bytes)
 *       4 n_seq H (kv_lora + d_s)        absorbed queries
 *     + 4 n_seq H S 2                    per-split (max, sum)
 *     + 4 n_seq H S kv_lora              per-split latent sums
 *     bytes (not mla_decode_workspace(), which sizes the tensor-core path).  A
 *     request that needs more returns GMLA_EWORKSPACE and enqueues nothing.
 *     Example: H = 96, kv_lora = 512, d_s = 64, max_len = 8192 needs
 *     1,800,192 bytes per sequence, so 9 sequences fit (16,201,728 bytes) and
 *     10 are refused.
 *   Memory: every GPU that loads the library holds the 16 MiB until the
 *     process exits.  No device memory is allocated by the call.
 *   Set-up: the first call on a device (the current device) looks up the
 *     array's device address with cudaGetSymbolAddress; make that first call
 *     before any stream capture on that device.
 *   Sharing: all calls on a device share the one array, which keeps the last
 *     call's contents (nothing in it needs clearing: every byte read is first
 *     written by the same call).  Calls that overlap on the GPU — on different
 *     streams, or from different host threads without ordering — race on the
 *     array and corrupt each other's results; serialise them.
 */
int mla_decode_absorbed_noalloc(const gmla_geom* geom, gmla_dtype dtype, int n_seq,
                                const void* q, const void* W_UKV, const void* cache,
                                const int* seq_offsets, int max_len, const void* g, void* O,
                                void* stream);

/*
 * mla_gemm — C[M][N] = A[M][K] B[K][N], fp32 accumulation, rounded to dtype.
 * The plain projections of the layer: the gate g = x W_g and the output
 * Delta_attn = o W_O ("Kimi K3 · Gated MLA · OpenModelAtlas", "All 20 steps").
 */
int mla_gemm(gmla_dtype dtype, int M, int N, int K, const void* A, const void* B, void* C,
             void* stream);

/* Synchronise `stream`, then return and clear the device error flag: GMLA_OK,
 * or GMLA_ETIMEOUT if a bounded device wait gave up since the last call.
 * GMLA_ECUDA if the synchronisation itself failed. */
int gmla_device_status(void* stream);

/* Wall-time limit, in nanoseconds, after which a device-side pipeline wait
 * of this library's kernels gives up (default 2 s; 0 restores the default).
 * The pages have no counterpart: this is the failure-detection hook.  A wait
 * that gives up records GMLA_ETIMEOUT (read and cleared by
 * gmla_device_status); its CTA stops issuing work, waits (with the fixed 2 s
 * bound) for its own copies and MMAs still in flight, frees its tensor memory
 * and returns, and CTAs that start afterwards return at once, so the context
 * stays usable.  A short limit lets a test make a wait run out.  Applies to
 * the current device, to kernels launched after the call; synchronous with
 * respect to the host.  Do not change it while this library's kernels run. */
int gmla_set_wait_limit_ns(unsigned long long ns);

/* Self-test of the bounded waits: one CTA that holds tensor memory waits, as
 * the pipeline kernels do, on an mbarrier that nothing ever arrives at.  The
 * wait gives up after the current wait limit (gmla_set_wait_limit_ns) and
 * records GMLA_ETIMEOUT; the CTA frees its tensor memory and returns.
 * `elapsed` is a DEVICE pointer to two uint64: the wait's duration in ns and
 * 1 if it gave up.  Asynchronous on `stream`; kernels of this library that
 * start after it on the device return at once until gmla_device_status()
 * has read the error.  The pages have no counterpart: this is the
 * failure-detection test hook. */
int gmla_selftest_wait(unsigned long long* elapsed, void* stream);

/* The cudaError_t behind the last GMLA_ECUDA on this host thread (0 if none). */
int gmla_last_cuda_error(void);

/* Static text for a status code. */
const char* gmla_strerror(int status);

/* Library version as an integer (major * 10000 + minor * 100 + patch). */
int gmla_version(void);

/* Number of kernels this library has enqueued in this process (all threads). */
unsigned long long gmla_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* GMLA_H */
