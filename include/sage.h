/*
 * sage.h -- C ABI of libsage, a B200 (sm_100a) implementation of the
 * SageAttention quantized attention forward pass.
 *
 * Method (cited by page title and section):
 *   - "SageAttention2: Efficient Attention with Thorough Outlier Smoothing and
 *     Per-thread INT4 Quantization" reading note
 *     (zhaifeiyue.github.io/papers/2411.10958/detail), Algorithm 1: smooth K,
 *     smooth Q with the delta_S GEMV compensation, per-block INT8 Q/K,
 *     per-channel FP8 V, online softmax, P~ * 448 -> E4M3, FP8 PV with
 *     two-level FP32 accumulation, final O / l / 448 * delta_V.
 *   - "FlashAttention vs SageAttention" source note (kenforever1.github.io),
 *     sections "执行流水线" and "后端矩阵": the API takes Q/K/V, layout,
 *     is_causal, sm_scale; fp16/bf16 inputs only; head_dim 64/128 (larger is
 *     rejected); GQA needs Hq % Hkv == 0; smooth_k subtracts the token mean
 *     of K, broadcast to the Q heads of a KV group.
 *
 * Conventions for every entry point:
 *   - Tensors are HND [B, H, N, d] (default) or NHD [B, N, H, d] (p->layout),
 *     contiguous, d fastest.  Quantised tensors in the workspace, qkm and lse
 *     are head-major in either case.
 *   - Every pointer argument is a DEVICE pointer owned by the caller unless
 *     stated otherwise; the library never allocates device memory.  Scratch
 *     lives in a caller-provided workspace of sage_workspace_bytes() bytes.
 *   - Device pointers must be 16-byte aligned; the workspace 256-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *     enqueued asynchronously; argument errors are returned synchronously and
 *     nothing is enqueued.  Device-side failures (a bounded wait inside a
 *     kernel that gave up) are reported by sage_last_device_error().
 *   - Only sm_100 devices are accepted (SAGE_ERR_UNSUPPORTED_ARCH otherwise).
 */
#ifndef SAGE_H
#define SAGE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SAGE_API __attribute__((visibility("default")))
#else
#define SAGE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SAGE_OK = 0,
    SAGE_ERR_INVALID_ARG = 1,          /* null pointer, bad sizes, Hq % Hkv != 0, N < 1 ... */
    SAGE_ERR_UNSUPPORTED_HEADDIM = 2,  /* d not in {64, 128} */
    SAGE_ERR_UNSUPPORTED_DTYPE = 3,    /* dtype not bf16/fp16 */
    SAGE_ERR_UNSUPPORTED_ARCH = 4,     /* current device is not sm_100 */
    SAGE_ERR_WORKSPACE_TOO_SMALL = 5,
    SAGE_ERR_CUDA = 6,                 /* a CUDA runtime/driver call failed */
    SAGE_ERR_TIMEOUT = 7,              /* a bounded in-kernel wait gave up */
    SAGE_ERR_MISALIGNED = 8            /* a pointer is not 16-byte aligned */
} sage_status;

typedef enum { SAGE_BF16 = 0, SAGE_FP16 = 1 } sage_dtype;

/* Problem description shared by all entry points. */
typedef struct {
    int32_t B, Hq, Hkv, N, d;  /* batch, query heads, key/value heads, tokens, head_dim */
    int32_t dtype;             /* sage_dtype of Q, K, V and O */
    int32_t causal;            /* 1: key j > query i is masked (top-left aligned) */
    float   sm_scale;          /* softmax scale; <= 0 selects 1/sqrt(d) */
    int32_t smooth_k;          /* 1: subtract the per-(b, kv-head, channel) token mean of K */
    int32_t smooth_q;          /* 1: subtract each Q block's mean and add delta_S back */
    int32_t bq;                /* Q quantisation block in rows: 32, 64 or 128 (32: one
                                  scale per 32-row TMEM lane group; INT8/FP8 path only) */
    int32_t bk;                /* K quantisation block in rows: 64 or 128 */
    int32_t pv_accum;          /* FP32 accumulation of P~V across key tiles:
                                  SAGE_PV_TWO_LEVEL (0): each tile's P^V lands in a
                                    fresh TMEM tile, then O = e^(m_old-m) O + O_t on
                                    CUDA cores (SageAttention2 Algorithm 1, level 2);
                                  SAGE_PV_TMEM_FP32 (1): P^V accumulates in one FP32
                                    TMEM accumulator, rescaled on CUDA cores only for
                                    rows whose max grew (tcgen05 keeps full FP32 in
                                    the accumulator: see sage_debug_f8_accum_probe) */
    int32_t return_lse;        /* 1: sage_quant_qkv also computes Q_i . km (view->qkm) so
                                  that sage_attn_fwd_quantized_lse can write the
                                  log-sum-exp; 0: view->qkm is NULL (INT8/FP8 path) */
    int32_t layout;            /* sage_layout of q, k, v and o: SAGE_HND [B, H, N, d] or
                                  SAGE_NHD [B, N, H, d] (the quantised tensors in the
                                  workspace and lse are always head-major) */
} sage_params;

typedef enum { SAGE_HND = 0, SAGE_NHD = 1 } sage_layout;

enum { SAGE_PV_TWO_LEVEL = 0, SAGE_PV_TMEM_FP32 = 1 };

/*
 * Device views of the quantised tensors produced by sage_quant_qkv (all
 * pointers point into the caller's workspace).  Np = N rounded up to 128
 * (the attention kernel's tile); padded rows/columns hold zeros.
 * Tm = ceil(N / bq), Tn = ceil(N / bk).
 */
typedef struct {
    int8_t  *q8;    /* [B, Hq,  Np, d]  INT8 codes of (Q - qbar) or Q            */
    int8_t  *k8;    /* [B, Hkv, Np, d]  INT8 codes of gamma(K) = K - km          */
    uint8_t *v8t;   /* [B, Hkv, d, Np]  E4M3 codes of V / s_v, transposed        */
    float   *s_q;   /* [B, Hq,  Tm]     delta_Q: amax/127 per Q block            */
    float   *s_k;   /* [B, Hkv, Tn]     delta_K: amax/127 per K block            */
    float   *s_v;   /* [B, Hkv, d]      delta_V: amax/448 per channel            */
    float   *km;    /* [B, Hkv, d]      mean(K) over tokens (zeros if !smooth_k) */
    float   *qbar;  /* [B, Hq,  Tm, d]  Q block means (NULL unless smooth_q)     */
    float   *dS;    /* [B, Hq,  Tm, Np] delta_S = qbar . gamma(K)^T (or NULL)     */
    int64_t  Np;
    float   *qkm;   /* [B, Hq,  Np]     Q_i . km (fp32; zeros without smooth_k): the
                                        constant by which smooth K shifts row i's
                                        scores, sm_scale-free (log-sum-exp correction);
                                        NULL unless p->return_lse */
} sage_quant_view;

/* Bytes of workspace the entry points below need for `p` (0 if p is invalid). */
SAGE_API size_t sage_workspace_bytes(const sage_params *p);

/*
 * Preprocessing of SageAttention2 Algorithm 1 ("Preprocessing" and the
 * per-block psi_Q / psi_K quantisers; Figure 3 stages 1-3):
 *   km      = mean_n K[b,g,n,:]              (fp64 sum, one rounding to fp32)
 *   gamma K = K - km                         (fp32)
 *   qbar_i  = mean of Q block i (smooth_q)   (fp64 sum over valid rows)
 *   s_q/s_k = amax_block |x| / 127,  code = clamp(rint(x / s), -127, 127)
 *   s_v[c]  = amax_n |V[n,c]| / 448, v8t   = E4M3_rn_satfinite(V / s_v)
 *   dS[i,j] = qbar_i . gamma(K_j)            (smooth_q only; fp32 accumulation)
 * q, k, v: device [B,H,N,d] (or [B,N,H,d], p->layout) in p->dtype.  Fills *view (host struct) with
 * pointers into `workspace`.  Quantised tensors and scales are bit-exact with
 * the plain definitions above.
 * For d = 128, K and V are read from HBM once when the ceil(N/128) tiles of
 * one head fit twice in the CTAs the GPU holds at once (tiles wait in shared
 * memory for their head's km / s_v); otherwise a statistics pass runs first.
 * Both give the same bytes.  A wait that runs out (a GPU shared with a stalled kernel)
 * records SAGE_ERR_TIMEOUT for sage_last_device_error.
 */
SAGE_API sage_status sage_quant_qkv(const void *q, const void *k, const void *v, const sage_params *p,
                           void *workspace, size_t workspace_bytes,
                           sage_quant_view *view, void *stream);

/*
 * The fused attention kernel of SageAttention2 Algorithm 1 (inner loop) on
 * already-quantised tensors: per 128-row Q tile and 128-key K tile,
 *   S   = (Q^ K^T)_int32 * s_q * s_k (+ dS) * sm_scale      (tcgen05 kind::i8)
 *   m   = max(m, rowmax S); P~ = exp(S - m); l = e^(m_old-m) l + rowsum P~
 *   O_t = E4M3(448 P~) @ V^                                (tcgen05 kind::f8f6f4,
 *                                                            fresh TMEM tile)
 *   O   = e^(m_old - m) O + O_t                             (FP32, CUDA cores)
 * and finally O / l / 448 * s_v written to `o` [B,Hq,N,d] in p->dtype.
 * `view` must come from sage_quant_qkv with the same p.
 */
SAGE_API sage_status sage_attn_fwd_quantized(const sage_quant_view *view, void *o, const sage_params *p,
                                    void *stream);

/* sage_quant_qkv followed by sage_attn_fwd_quantized (the whole forward).
 * Both attention kernels check the device error word first: while an error
 * recorded by an earlier launch (a quantiser wait that ran out and left codes
 * unwritten) has not been read by sage_last_device_error, they return without
 * touching `o`, so O is never computed from stale codes. */
SAGE_API sage_status sage_attn_fwd(const void *q, const void *k, const void *v, void *o, const sage_params *p,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * sage_attn_fwd_quantized that also writes each row's log-sum-exp of the
 * attention scores (the return_lse of the SageAttention API):
 *   lse[b, h, i] = ln sum_j exp(S_ij) + sm_scale (Q_i . km)
 * S are the scores the kernel uses (dequantised INT8 Q^K^T on the smoothed K,
 * + delta_S, times sm_scale; causal: keys j <= i); the second term undoes the
 * row-constant shift of smooth K (zero without it), so lse refers to the
 * original keys.  lse: device fp32 [B, Hq, N], 4-byte aligned, caller-owned.
 * SAGE_ERR_INVALID_ARG if lse is misaligned or the view lacks qkm (the view
 * must come from sage_quant_qkv with p->return_lse = 1).
 */
SAGE_API sage_status sage_attn_fwd_quantized_lse(const sage_quant_view *view, void *o, float *lse,
                                                 const sage_params *p, void *stream);

/* sage_quant_qkv followed by sage_attn_fwd_quantized_lse (return_lse is
 * taken as 1 whatever p says). */
SAGE_API sage_status sage_attn_fwd_lse(const void *q, const void *k, const void *v, void *o, float *lse,
                                       const sage_params *p, void *workspace, size_t workspace_bytes,
                                       void *stream);

/*
 * Bit-exactness probe of the INT8 tensor-core path: the raw INT32 tile
 * (Q^ K^T) for rows [128*qtile, +128) of head (b, h) and keys [128*ktile, +128),
 * computed with the same TMA staging, shared-memory descriptors and
 * tcgen05.mma kind::i8 instruction as the attention kernel, written
 * row-major to out_128x128 (device, 128*128 int32).
 */
SAGE_API sage_status sage_debug_qk_int32(const sage_quant_view *view, const sage_params *p,
                                int32_t b, int32_t h, int32_t qtile, int32_t ktile,
                                int32_t *out_128x128, void *stream);

/*
 * Returns the first device-side error recorded since the last call
 * (SAGE_OK or SAGE_ERR_TIMEOUT) and clears it.  Synchronises `stream`.
 */
SAGE_API sage_status sage_last_device_error(void *stream);

/*
 * Failure-detection check: launches one CTA that waits on an mbarrier nobody
 * arrives at, bounded by `timeout_us`.  The wait gives up, records
 * SAGE_ERR_TIMEOUT and the kernel returns normally (the context stays
 * usable).  Returns the status sage_last_device_error() then reports.
 */
SAGE_API sage_status sage_debug_bounded_wait(uint32_t timeout_us, void *stream);

/*
 * Size of the device scratch array that sage_attn_fwd_noalloc uses (32 MiB).
 * Every GPU that loads this library reserves it until the process exits.
 */
#define SAGE_STATIC_SCRATCH_BYTES (32u << 20)

/*
 * sage_attn_fwd without a workspace argument.  The method has no counterpart
 * for this: it exists for callers that cannot allocate device memory at all
 * (a plugin interface that only hands over input and output pointers, or a
 * process whose device memory is owned by another allocator), so cudaMalloc
 * is not open to them.  It computes exactly what sage_attn_fwd computes, with
 * its scratch in a fixed library-owned device array of
 * SAGE_STATIC_SCRATCH_BYTES bytes instead of a caller workspace.
 *   - q, k, v, o: device pointers as for sage_attn_fwd (caller-owned).
 *   - Allocates nothing: no cudaMalloc / cudaFree and no allocating library
 *     routine.
 *   - Parameters are checked first, with the statuses sage_attn_fwd gives
 *     (e.g. SAGE_ERR_UNSUPPORTED_HEADDIM); then SAGE_ERR_WORKSPACE_TOO_SMALL
 *     when sage_workspace_bytes(p) exceeds SAGE_STATIC_SCRATCH_BYTES; then
 *     SAGE_ERR_UNSUPPORTED_ARCH off sm_100.  Nothing is enqueued on an error.
 *   - The first call on a device looks up the array's device address on
 *     that device (the device must be current) and caches it with the id of
 *     the device's context; make that first call before any stream capture.
 *     A context re-created on that device (after cudaDeviceReset) is noticed
 *     by its new id and the address is looked up again, so again make that
 *     next call outside a capture.
 *   - All calls on a device share the one array, and it keeps whatever the
 *     last call left in it.  Calls whose work overlaps on the GPU (different
 *     streams, or host threads without ordering) race on it; order them.
 */
SAGE_API sage_status sage_attn_fwd_noalloc(const void *q, const void *k, const void *v, void *o,
                                           const sage_params *p, void *stream);

/*
 * Accumulator-precision probe of the FP8 tensor-core path (tcgen05.mma
 * kind::f8f6f4, FP32 accumulator).  The SageAttention2 note ("5. Numerical
 * Considerations") reports that Ada/Hopper FP8 MMAs keep only ~13 mantissa
 * bits in their accumulator, the reason for the two-level accumulation.
 * Writes 8 floats to out8 (device) whose exact values are
 *   1+2^-18, 1+2^-14, 1+2^-12, 256, 32, 4096+2^-10, 1+2^-18, 1+2^-13
 * (cases 5-7 accumulate across two MMAs).  Comparing them with these values
 * shows how many accumulator bits the hardware keeps.
 */
SAGE_API sage_status sage_debug_f8_accum_probe(float *out8, void *stream);

/*
 * ---------------------------------------------------------------- NVFP4 path
 * SageAttention3 reading note (zhaifeiyue.github.io/papers/2505.11594),
 * "Microscaling FP4 attention" and the two-level quantisation of P.  Same
 * sage_params (d must be 128; bq is the smooth-Q block, 64 or 128; bk and
 * pv_accum are not used).  E2M1 codes are packed two per byte, the even
 * element in the low nibble; every 16 consecutive elements share one E4M3
 * scale E4M3(amax16 / 6).  Scale blocks hold, per 128-row tile, two 512-byte
 * blocks (64-element K chunks kk = 0, 1); in block kk the scale of row m
 * (Q row, key, or V channel) for its 16-element group 4 kk + k is at byte
 * 16 (m % 32) + 4 (m / 32) + k.  Padded rows hold zero codes and scales.
 */
typedef struct {
    uint8_t *q4;   /* [B, Hq,  Np, d/2]        E2M1 of (Q - qbar) or Q, along d       */
    uint8_t *k4;   /* [B, Hkv, Np, d/2]        E2M1 of gamma(K) = K - km, along d     */
    uint8_t *v4t;  /* [B, Hkv, d, Np/2]        E2M1 of V along tokens, transposed     */
    uint8_t *sfq;  /* [B, Hq,  Np/128, 1024]   E4M3 scales of q4 (16 channels each)   */
    uint8_t *sfk;  /* [B, Hkv, Np/128, 1024]   E4M3 scales of k4                      */
    uint8_t *sfv;  /* [B, Hkv, Np/128, 1024]   E4M3 scales of v4t (16 tokens each)    */
    float   *km;   /* [B, Hkv, d]              mean(K) over tokens (zeros if !smooth_k) */
    float   *qbar; /* [B, Hq,  Tm, d]          Q block means (NULL unless smooth_q)   */
    float   *dS;   /* [B, Hq,  Tm, Np]         delta_S = qbar . gamma(K)^T (or NULL)  */
    int64_t  Np;
} sage_nvfp4_view;

/* Workspace bytes the NVFP4 entry points need for `p` (0 if p is invalid or d != 128). */
SAGE_API size_t sage_nvfp4_workspace_bytes(const sage_params *p);

/*
 * NVFP4 preprocessing: km, gamma(K) and (smooth_q) qbar / delta_S exactly as
 * sage_quant_qkv; then per 16-element group sb = E4M3_rn_satfinite(amax / 6)
 * (IEEE fp32 division) and codes E2M1_rn_satfinite(x / sb) (0 when sb == 0),
 * along d for Q and K and along tokens for V.  Bit-exact with these
 * definitions.  Fills *view with pointers into `workspace`.
 */
SAGE_API sage_status sage_quant_nvfp4(const void *q, const void *k, const void *v, const sage_params *p,
                                      void *workspace, size_t workspace_bytes, sage_nvfp4_view *view,
                                      void *stream);

/*
 * The fused NVFP4 attention kernel on a view from sage_quant_nvfp4 (same p):
 * S = (Q^ sq)(K^ sk)^T (+ dS), scaled by sm_scale (tcgen05 kind::mxf4nvf4);
 * online softmax in FP32; per row and key tile s_P1 = rowmax(P~) / 2688,
 * P2 = P~ / s_P1, s_P2 = E4M3(amax16(P2) / 6), P^ = E2M1(P2 / s_P2); the
 * block-scaled P^ V^ product is accumulated in FP32 with the s_P1 and
 * exp(m_old - m) factors; o = O / l in p->dtype, [B, Hq, N, d].
 */
SAGE_API sage_status sage_attn_fwd_nvfp4_quantized(const sage_nvfp4_view *view, void *o, const sage_params *p,
                                                   void *stream);

/* sage_quant_nvfp4 followed by sage_attn_fwd_nvfp4_quantized. */
SAGE_API sage_status sage_attn_fwd_nvfp4(const void *q, const void *k, const void *v, void *o,
                                         const sage_params *p, void *workspace, size_t workspace_bytes,
                                         void *stream);

/*
 * Probe of the block-scaled FP4 tensor-core path: the FP32 tile
 * (Q^ sq)(K^ sk)^T (no delta_S, no sm_scale) for rows [128 qtile, +128) of
 * head (b, h) and keys [128 ktile, +128), through the same TMA staging,
 * scale-block copies and MMA as the attention kernel; row-major to
 * out_128x128 (device, 128*128 floats).
 */
SAGE_API sage_status sage_debug_qk_nvfp4(const sage_nvfp4_view *view, const sage_params *p, int32_t b,
                                         int32_t h, int32_t qtile, int32_t ktile, float *out_128x128,
                                         void *stream);

/*
 * Accuracy probe of the FMA-pipe exponential (a Cody-Waite range reduction and
 * a degree-4 polynomial on the FMA and ALU pipes, so that an exp2 need not use
 * the MUFU): y[i] = 2^x[i] for n device floats, computed by the same device
 * function the attention kernels can use for a share of their exponentials
 * (a compile-time choice; the shipped kernels compute every exponential of P
 * on the MUFU, which measured faster).  Valid for -126 <= x <= 100; x < -126
 * gives 2^-126 or less (the kernel's masked scores).
 */
SAGE_API sage_status sage_debug_exp2_poly(const float *x, float *y, int32_t n, void *stream);

/*
 * Tensor-core rate probe (the measured peak that the attention kernels are
 * compared with; the pages give no counterpart for B200).  Launches `ctas`
 * CTAs (0: one per SM), each issuing `iters` back-to-back passes of
 * tcgen05.mma with M = 128 on operand tiles resident in shared memory,
 * accumulating in TMEM:
 *   kind 0: kind::i8 (s8, s32 accumulator), n = 64, 128 or 256, 4 x K = 32 per pass
 *   kind 1: kind::f8f6f4 (E4M3, f32 accumulator), n = 64, 128 or 256, 4 x K = 32
 *   kind 2: kind::mxf4nvf4 block16 (E2M1 with UE4M3 scales), n = 128, 2 x K = 64
 * *ops (host) receives the launch's operation count, 2 x 128 x n x 128 per
 * pass per CTA; dividing it by the launch's duration (CUDA events on
 * `stream`) gives the rate.  1 <= iters <= 2,000,000.  SAGE_ERR_INVALID_ARG
 * for an unsupported (kind, n).
 */
SAGE_API sage_status sage_debug_mma_rate(int32_t kind, int32_t n, int32_t iters, int32_t ctas, double *ops,
                                         void *stream);

/*
 * Number of kernels sage_quant_qkv enqueues for p on the current device (not
 * counting memsets): 2 with the one-read K/V kernel (K and V, then Q), 4 with
 * the two-pass path (K/V statistics, K, V, Q); +1 with smooth_q (delta_S).
 * *n is written on SAGE_OK.  Needs the device (the choice depends on how many
 * CTAs it holds at once).
 */
SAGE_API sage_status sage_quant_kernel_count(const sage_params *p, int32_t *n);

/*
 * Number of kernels sage_quant_nvfp4 enqueues for p on the current device
 * (not counting memsets): 3 with the one-read K kernel (K, V, Q), 4 with the
 * statistics pass (K statistics, K, V, Q); +1 with smooth_q (delta_S).
 * Argument checks as sage_quant_nvfp4 (head_dim 128 only).
 */
SAGE_API sage_status sage_quant_nvfp4_kernel_count(const sage_params *p, int32_t *n);

/*
 * Test hook: on = 1 makes sage_quant_qkv and sage_quant_nvfp4 (and the calls
 * built on them) take the two-pass K/V path (statistics kernel, then the code
 * kernels) in this process; on = 2 makes them take the one-read path even when
 * a (head, K|V) group's tiles may not all be resident at once, so that its
 * bounded waits can run out (a test of the timeout path: the waits give up,
 * SAGE_ERR_TIMEOUT is recorded, the tiles that gave up write no codes); on = 0
 * restores the default choice.  Not thread-safe with concurrent
 * sage_quant_qkv calls.  SAGE_ERR_INVALID_ARG for other values.
 */
SAGE_API sage_status sage_debug_kv_quant_two_pass(int32_t on);

/*
 * Test hook: the limit of every bounded in-kernel wait, in microseconds, for
 * the launches enqueued after this call on `stream` (0 restores the default of
 * 4 s).  Synchronises `stream`.  1 <= timeout_us <= 10 s, or 0.
 */
SAGE_API sage_status sage_debug_wait_limit(uint32_t timeout_us, void *stream);

/* Human-readable name of a status code (static storage). */
SAGE_API const char *sage_status_string(sage_status s);

#ifdef __cplusplus
}
#endif
#endif /* SAGE_H */
