// common.cuh -- argument blocks shared by the host entry points (api.cu) and
// the kernels (quant.cu, attn_i8f8.cu).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace sage {

constexpr int kTile = 128;  // attention tile: 128 Q rows x 128 keys

// Element offset of row n of head bh (= b H + h) in a caller tensor of H heads,
// N rows and D channels: [B, H, N, D] (HND) or [B, N, H, D] (NHD, nhd = 1).
__host__ __device__ inline int64_t row_offset(int64_t bh, int64_t n, int H, int64_t N, int D, int nhd) {
  return nhd ? (((bh / H) * N + n) * H + bh % H) * D : (bh * N + n) * D;
}
// elements between consecutive rows of one head
__host__ __device__ inline int64_t row_stride(int H, int D, int nhd) { return nhd ? (int64_t)H * D : (int64_t)D; }

struct QuantArgs {
  const void* q;  // [B,Hq,N,D] bf16/fp16
  const void* k;  // [B,Hkv,N,D]
  const void* v;  // [B,Hkv,N,D]
  int B, Hq, Hkv, N, D;
  int64_t Np;
  int Tm, Tn, bq, bk;
  int smooth_k, smooth_q;
  int nhd;  // q, k, v are [B, N, H, D] (else [B, H, N, D])
  // outputs / scratch (workspace)
  int8_t* q8;
  int8_t* k8;
  uint8_t* v8t;
  float* s_q;
  float* s_k;
  float* s_v;
  float* km;
  float* qbar;
  float* dS;
  float* qkm;  // [B,Hq,Np] Q_i . km in fp32 (written by the Q kernel; zeros without smooth K)
  double* ksum;     // [B,Hkv,D] fp64 column sums of K
  unsigned* vamax;  // [B,Hkv,D] bit pattern of max |V| (non-negative floats order as uints);
                    // nullptr: the statistics pass skips V (NVFP4 path)
  // one-read K/V quantisation (kv_fused_quant_kernel); kv_sync == nullptr
  // selects the two-pass path (statistics kernel, then the code kernels)
  int* kv_sync;          // ticket counter, then tiles published per group: [1 + 2 B Hkv]
                         // ints on the INT8 path ((head, K|V) groups), [1 + B Hkv] on the
                         // NVFP4 path (K only)
  size_t kv_zero_bytes;  // bytes from ksum through the end of kv_sync (consecutive in
                         // the workspace), zeroed before the one-read kernel
  int force_one_read;    // test hook: take the one-read path even when a group's tiles may
                         // not all be resident at once (its bounded waits then run out)
  // NVFP4 path (E2M1 codes two per byte, low nibble first; 1 KB scale blocks
  // per 128-row tile in the tcgen05 scale-factor order)
  uint8_t* q4;   // [B,Hq,Np,D/2]
  uint8_t* k4;   // [B,Hkv,Np,D/2]
  uint8_t* v4t;  // [B,Hkv,D,Np/2]
  uint8_t* sfq;  // [B,Hq,Np/128,1024]
  uint8_t* sfk;  // [B,Hkv,Np/128,1024]
  uint8_t* sfv;  // [B,Hkv,Np/128,1024]
};

struct AttnArgs {
  int B, Hq, Hkv, N, D;
  int64_t Np;
  int Tm, Tn, bq, bk;
  int causal;
  int n_qtiles;
  float scale_log2;  // sm_scale * log2(e)
  float sm_scale;
  const float* s_q;
  const float* s_k;
  const float* s_v;
  const float* dS;  // nullptr when smooth_q is off
  void* o;          // [B,Hq,N,D] bf16/fp16 ([B,N,Hq,D] when the caller's layout is NHD)
  int64_t o_bs, o_hs, o_rs;  // element strides of o between batches, heads and rows
  int nhd;                   // the caller's layout is NHD (NVFP4 kernel: a template choice)
  float* lse;        // [B,Hq,N] natural-log log-sum-exp of the rows' scores, or nullptr
  const float* qkm;  // [B,Hq,Np] Q_i . km (the smooth-K correction of lse / sm_scale)
  int out_fp16;
  int two_level;  // 1: fresh O_t per key tile + FP32 add on CUDA cores; 0: TMEM FP32 accumulator
  // NVFP4 scale blocks (1 KB per 128-row tile)
  const uint8_t* sfq;
  const uint8_t* sfk;
  const uint8_t* sfv;
  // probe mode (sage_debug_qk_int32)
  int probe_b, probe_h, probe_qtile, probe_ktile;
  int32_t* probe_out;
};

// TMA maps of the preprocessing: the bf16/fp16 inputs as 4D (D, N, H, B) tensors
// with the caller's layout in the strides (box D x 128 x 1 x 1), and the
// transposed E4M3 V output v8t (box D x 128 bytes).
struct QuantMaps {
  CUtensorMap q, k, v, vt;
};

// launchers (defined in the .cu files)
// kernels (not counting memsets) that launch_quant enqueues for a's sizes and
// flags (the one-read K/V path if allowed and it fits the current device,
// else the two-pass path)
int quant_kernel_count(const QuantArgs& a, int is_fp16, bool allow_one_read);
cudaError_t launch_quant(const QuantArgs& a, const QuantMaps& m, int is_fp16, cudaStream_t st);
// tmO: the caller's output as a 4D tensor (d, N, Hq, B), box 64 x 32, 128-byte
// swizzle (the one-warp-per-row kernel writes its output tiles through it)
cudaError_t launch_attn_i8f8(const AttnArgs& a, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                             const CUtensorMap& tmV, const CUtensorMap& tmO, cudaStream_t st);
cudaError_t launch_qk_probe(const AttnArgs& a, const CUtensorMap& tmQ, const CUtensorMap& tmK, cudaStream_t st);
cudaError_t launch_bounded_wait_probe(cudaStream_t st);
cudaError_t launch_exp2_poly_probe(const float* x, float* y, int n, cudaStream_t st);
cudaError_t launch_f8_accum_probe(float* out, cudaStream_t st);
// tensor-core rate probe (peak.cu): ops of one launch (0: unsupported kind / n) and its launcher
double mma_rate_ops(int kind, int n, int iters, int ctas);
cudaError_t launch_mma_rate(int kind, int n, int iters, int ctas, cudaStream_t st);
cudaError_t launch_quant_nvfp4(const QuantArgs& a, const QuantMaps& m, int is_fp16, cudaStream_t st);
// kernels (not counting memsets) that launch_quant_nvfp4 enqueues for a's sizes and flags
int quant_nvfp4_kernel_count(const QuantArgs& a, int is_fp16, bool allow_one_read);
cudaError_t launch_attn_nvfp4(const AttnArgs& a, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                              const CUtensorMap& tmV, cudaStream_t st);
cudaError_t launch_qk_probe_nvfp4(const AttnArgs& a, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                  float* out, cudaStream_t st);

}  // namespace sage
