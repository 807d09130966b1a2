// attn_i8f8.cu -- fused SageAttention forward on sm_100a: INT8 Q K^T and FP8 P V
// on the 5th-generation tensor core (tcgen05), accumulators in TMEM.
//
// Algorithm (SageAttention2 note, zhaifeiyue.github.io/papers/2411.10958/detail,
// Algorithm 1 inner loop; online softmax as on the "FlashAttention vs
// SageAttention" page, section "Online Softmax"), per 128-row Q tile i and
// 128-key tile j:
//   S_ij  = psi^-1(Q^_i K^_j^T) + delta_S        INT8 MMA (kind::i8) -> S32 in TMEM
//   m_ij  = max(m_i,j-1, rowmax S_ij)
//   P~_ij = exp(S_ij - m_ij),   l_ij = e^(m_i,j-1 - m_ij) l_i,j-1 + rowsum P~_ij
//   O_t   = E4M3(448 P~_ij) V^_j                  FP8 MMA (kind::f8f6f4) into a
//                                                 fresh TMEM tile (level 1)
//   O     = e^(m_i,j-1 - m_ij) O + O_t             FP32 in registers (level 2)
//   out   = O / l / 448 * delta_V
// The exponentials run in base 2 (scores pre-multiplied by log2 e); the 448
// is folded into the exponent (exp2(t - m + log2 448)), so l accumulates
// 448 P~ and the final division by l absorbs the /448.
//
// CTA = one (batch, head, Q tile); 192 threads in three roles:
//   warp 0      TMA producer: Q tile once, then K_j / V_j^T into a 2-stage ring
//   warp 1      MMA issuer (one thread) and TMEM owner (whole warp)
//   warps 2..5  softmax + correction + epilogue; thread = one Q row = one TMEM lane
// TMEM columns: [0, 128) S (int32), [128, 128 + D) O_t (fp32).
// P goes through shared memory in the 128-byte-swizzled K-major layout the
// MMA reads (the same layout TMA writes for K and V^T).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace sage {

namespace {

constexpr int kStages = 2;
constexpr int kThreadsAttn = 192;
constexpr float kLog2_448 = 8.807354922057604f;  // log2(448)

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int D>
struct Smem {
  static constexpr uint32_t kQ = 128 * D, kK = 128 * D, kV = D * 128, kP = 128 * 128;
  static constexpr uint32_t oQ = 0;
  static constexpr uint32_t oK = oQ + kQ;
  static constexpr uint32_t oV = oK + kStages * kK;
  static constexpr uint32_t oP = oV + kStages * kV;
  static constexpr uint32_t oBar = oP + kP;
  static constexpr uint32_t kNumBars = 1 + 3 * kStages + 4;
  static constexpr uint32_t oTmem = oBar + 8 * kNumBars;
  static constexpr uint32_t kBytes = oTmem + 16 + 1024;  // + alignment slack
};

template <typename TO>
__device__ __forceinline__ uint32_t pack2(float a, float b);
template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <>
__device__ __forceinline__ uint32_t pack2<__half>(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int D, bool CAUSAL, bool HAS_DS, typename TO>
__global__ void __launch_bounds__(kThreadsAttn, 1)
    attn_i8f8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
  using L = Smem<D>;
  constexpr uint32_t kSwzQK = (D == 128) ? kSwizzle128B : kSwizzle64B;
  constexpr uint32_t kSboQK = 8 * D;  // 8 rows x D bytes per swizzle atom
  constexpr uint32_t kIdescQK = make_idesc(/*S32*/ 2, /*s8*/ 1, /*s8*/ 1, 128, 128);
  constexpr uint32_t kIdescPV = make_idesc(/*F32*/ 1, /*E4M3*/ 0, /*E4M3*/ 0, 128, D);
  constexpr uint32_t kTmemCols = 256;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem + L::oQ;
  uint8_t* sK = smem + L::oK;
  uint8_t* sV = smem + L::oV;
  uint8_t* sP = smem + L::oP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::oBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + kStages;
  uint64_t* kv_empty = v_full + kStages;
  uint64_t* s_full = kv_empty + kStages;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_full = s_free + 1;
  uint64_t* pv_done = p_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::oTmem);

  // heavy (long causal) tiles first
  const int bhq = a.B * a.Hq;
  const int qtile = a.n_qtiles - 1 - (int)(blockIdx.x / bhq);
  const int bh = blockIdx.x % bhq;
  const int b = bh / a.Hq, h = bh % a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  const int nT = CAUSAL ? qtile + 1 : (int)(a.Np / kTile);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 128);
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + 128;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_map(&tmQ);
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      const int qrow = (int)((int64_t)(b * a.Hq + h) * a.Np + (int64_t)qtile * kTile);
      const int krow0 = (int)((int64_t)(b * a.Hkv + g) * a.Np);
      const int vrow = (b * a.Hkv + g) * D;
      mbar_expect_tx(q_full, L::kQ);
      tma_load_2d(sQ, &tmQ, q_full, 0, qrow);
      bool ok = true;
      int j = 0;
      for (; j < nT && ok; ++j) {
        const int s = j % kStages;
        if (j >= kStages) ok = mbar_wait(&kv_empty[s], ((j / kStages) + 1) & 1);
        if (!ok) break;
        mbar_expect_tx(&k_full[s], L::kK);
        tma_load_2d(sK + s * L::kK, &tmK, &k_full[s], 0, krow0 + j * kTile);
        mbar_expect_tx(&v_full[s], L::kV);
        tma_load_2d(sV + s * L::kV, &tmV, &v_full[s], j * kTile, vrow);
      }
      // never leave a copy in flight: wait for the last loads to land
      for (int jj = max(0, j - kStages); jj < j; ++jj) {
        mbar_wait(&k_full[jj % kStages], (jj / kStages) & 1);
        mbar_wait(&v_full[jj % kStages], (jj / kStages) & 1);
      }
      mbar_wait(q_full, 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t aQ = smem_u32(sQ), aP = smem_u32(sP);
      bool ok = mbar_wait(q_full, 0);
      int issued_pv = 0;
      auto issue_pv = [&](int jj) -> bool {
        const int s = jj % kStages;
        if (!mbar_wait(p_full, jj & 1)) return false;
        if (!mbar_wait(&v_full[s], (jj / kStages) & 1)) return false;
        tc_fence_after();
        const uint32_t aV = smem_u32(sV + s * L::kV);
#pragma unroll
        for (int kk = 0; kk < kTile / 32; ++kk)
          mma_f8f6f4(tO, make_sdesc(aP + kk * 32, 1024, kSwizzle128B), make_sdesc(aV + kk * 32, 1024, kSwizzle128B),
                     kIdescPV, kk > 0 ? 1u : 0u);
        mma_commit(pv_done);
        mma_commit(&kv_empty[s]);
        ++issued_pv;
        return true;
      };
      for (int j = 0; j < nT && ok; ++j) {
        const int s = j % kStages;
        ok = mbar_wait(&k_full[s], (j / kStages) & 1);
        if (ok && j > 0) ok = mbar_wait(s_free, (j - 1) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t aK = smem_u32(sK + s * L::kK);
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          mma_i8(tS, make_sdesc(aQ + kk * 32, kSboQK, kSwzQK), make_sdesc(aK + kk * 32, kSboQK, kSwzQK), kIdescQK,
                 kk > 0 ? 1u : 0u);
        mma_commit(s_full);
        if (j > 0) ok = issue_pv(j - 1);
      }
      if (ok) ok = issue_pv(nT - 1);
      // all tensor-core work retired before the CTA frees TMEM
      if (issued_pv > 0) mbar_wait(pv_done, (issued_pv - 1) & 1);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / correction
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int64_t qrow = (int64_t)qtile * kTile + row;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int qblk = min((int)(qrow / a.bq), a.Tm - 1);
    const float row_scale = a.s_q[(int64_t)(b * a.Hq + h) * a.Tm + qblk] * a.scale_log2;
    const float* sk = a.s_k + (int64_t)(b * a.Hkv + g) * a.Tn;
    const float* dsr = HAS_DS ? a.dS + ((int64_t)(b * a.Hq + h) * a.Tm + qblk) * a.Np : nullptr;

    float o[D];
#pragma unroll
    for (int c = 0; c < D; ++c) o[c] = 0.0f;
    float m = -INFINITY, l = 0.0f, alpha_prev = 0.0f;
    bool ok = true;
    uint32_t r[32];

    for (int j = 0; j < nT && ok; ++j) {
      if (!(ok = mbar_wait_warp(s_full, j & 1))) break;
      tc_fence_after();
      const int col0 = j * kTile;
      float ak[4];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) ak[c4] = row_scale * __ldg(sk + min((col0 + c4 * 32) / a.bk, a.Tn - 1));
      const bool need_mask = (col0 + kTile > a.N) || (CAUSAL && col0 + kTile - 1 > qtile * kTile);

      // pass 1: row max of this tile (log2 units)
      float mx = -INFINITY;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        tmem_ld32(tS + lane_off + c4 * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int col = col0 + c4 * 32 + e;
          float t = (float)(int)r[e] * ak[c4];
          if (HAS_DS) t = fmaf(__ldg(dsr + col), a.scale_log2, t);
          const bool masked = need_mask && (col >= a.N || (CAUSAL && col > qrow));
          if (!masked) mx = fmaxf(mx, t);
        }
      }
      const float m_new = fmaxf(m, mx);
      const float alpha = (m == -INFINITY) ? 0.0f : ex2_approx(m - m_new);
      const float mm = (m_new == -INFINITY) ? 0.0f : m_new - kLog2_448;

      // level-2 accumulation of the previous tile: O = alpha_{j-1} O + O_t
      if (j > 0) {
        if (!(ok = mbar_wait_warp(pv_done, (j - 1) & 1))) break;
        tc_fence_after();
#pragma unroll
        for (int c4 = 0; c4 < D / 32; ++c4) {
          tmem_ld32(tO + lane_off + c4 * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[c4 * 32 + e] = fmaf(o[c4 * 32 + e], alpha_prev, __uint_as_float(r[e]));
        }
      }

      // pass 2: P = exp2(t - m + log2 448) -> E4M3 -> shared memory (SW128 K-major)
      float rs = 0.0f;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        tmem_ld32(tS + lane_off + c4 * 32, r);
        tmem_ld_wait();
        float p[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int col = col0 + c4 * 32 + e;
          float t = (float)(int)r[e] * ak[c4];
          if (HAS_DS) t = fmaf(__ldg(dsr + col), a.scale_log2, t);
          const bool masked = need_mask && (col >= a.N || (CAUSAL && col > qrow));
          p[e] = masked ? 0.0f : ex2_approx(t - mm);
          rs += p[e];
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint4 w;
          w.x = cvt_e4m3x2(p[hh * 16 + 0], p[hh * 16 + 1]) | (cvt_e4m3x2(p[hh * 16 + 2], p[hh * 16 + 3]) << 16);
          w.y = cvt_e4m3x2(p[hh * 16 + 4], p[hh * 16 + 5]) | (cvt_e4m3x2(p[hh * 16 + 6], p[hh * 16 + 7]) << 16);
          w.z = cvt_e4m3x2(p[hh * 16 + 8], p[hh * 16 + 9]) | (cvt_e4m3x2(p[hh * 16 + 10], p[hh * 16 + 11]) << 16);
          w.w = cvt_e4m3x2(p[hh * 16 + 12], p[hh * 16 + 13]) | (cvt_e4m3x2(p[hh * 16 + 14], p[hh * 16 + 15]) << 16);
          const int chunk = c4 * 2 + hh;
          *reinterpret_cast<uint4*>(sP + row * 128 + ((chunk ^ (row & 7)) << 4)) = w;
        }
      }
      tc_fence_before();
      mbar_arrive(s_free);
      fence_proxy_async_smem();
      mbar_arrive(p_full);
      l = fmaf(l, alpha, rs);
      alpha_prev = alpha;
      m = m_new;
    }

    if (ok && nT > 0 && (ok = mbar_wait_warp(pv_done, (nT - 1) & 1))) {
      tc_fence_after();
#pragma unroll
      for (int c4 = 0; c4 < D / 32; ++c4) {
        tmem_ld32(tO + lane_off + c4 * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) o[c4 * 32 + e] = fmaf(o[c4 * 32 + e], alpha_prev, __uint_as_float(r[e]));
      }
      // epilogue: out = O / l * delta_V   (l carries the 448)
      if (qrow < a.N) {
        const float inv_l = 1.0f / l;
        const float* sv = a.s_v + (int64_t)(b * a.Hkv + g) * D;
        TO* out = reinterpret_cast<TO*>(a.o) + ((int64_t)(b * a.Hq + h) * a.N + qrow) * D;
#pragma unroll
        for (int c = 0; c < D; c += 8) {
          uint4 w;
          w.x = pack2<TO>(o[c + 0] * inv_l * __ldg(sv + c + 0), o[c + 1] * inv_l * __ldg(sv + c + 1));
          w.y = pack2<TO>(o[c + 2] * inv_l * __ldg(sv + c + 2), o[c + 3] * inv_l * __ldg(sv + c + 3));
          w.z = pack2<TO>(o[c + 4] * inv_l * __ldg(sv + c + 4), o[c + 5] * inv_l * __ldg(sv + c + 5));
          w.w = pack2<TO>(o[c + 6] * inv_l * __ldg(sv + c + 6), o[c + 7] * inv_l * __ldg(sv + c + 7));
          *reinterpret_cast<uint4*>(out + c) = w;
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Bit-exactness probe: one INT32 tile Q^_i K^_j^T through the same TMA layout,
// descriptors and kind::i8 instruction as the attention kernel.
template <int D>
__global__ void __launch_bounds__(128, 1)
    qk_probe_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const AttnArgs a) {
  constexpr uint32_t kSwzQK = (D == 128) ? kSwizzle128B : kSwizzle64B;
  constexpr uint32_t kSboQK = 8 * D;
  constexpr uint32_t kIdescQK = make_idesc(2, 1, 1, 128, 128);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem;
  uint8_t* sK = smem + 128 * D;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 256 * D);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int g = a.probe_h / (a.Hq / a.Hkv);
  bool ok = true;
  if (threadIdx.x == 0) {
    const int qrow = (int)((int64_t)(a.probe_b * a.Hq + a.probe_h) * a.Np + (int64_t)a.probe_qtile * kTile);
    const int krow = (int)((int64_t)(a.probe_b * a.Hkv + g) * a.Np + (int64_t)a.probe_ktile * kTile);
    mbar_expect_tx(&bars[0], 256 * D);
    tma_load_2d(sQ, &tmQ, &bars[0], 0, qrow);
    tma_load_2d(sK, &tmK, &bars[0], 0, krow);
    if (mbar_wait(&bars[0], 0)) {
      tc_fence_after();
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK);
#pragma unroll
      for (int kk = 0; kk < D / 32; ++kk)
        mma_i8(tmem, make_sdesc(aQ + kk * 32, kSboQK, kSwzQK), make_sdesc(aK + kk * 32, kSboQK, kSwzQK), kIdescQK,
               kk > 0 ? 1u : 0u);
      mma_commit(&bars[1]);
    }
  }
  __syncwarp();
  ok = mbar_wait_warp(&bars[1], 0);
  if (ok) {
    tc_fence_after();
    const int row = (warp & 3) * 32 + lane;
    uint32_t r[32];
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
      tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + c4 * 32, r);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) a.probe_out[row * 128 + c4 * 32 + e] = (int32_t)r[e];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// A wait nobody ends: the bounded wait gives up, records the timeout, returns.
__global__ void bounded_wait_probe_kernel() {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0);
  __syncthreads();
}

template <int D, bool CAUSAL, bool HAS_DS, typename TO>
cudaError_t launch_attn_t(const AttnArgs& a, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                          cudaStream_t st) {
  auto kern = attn_i8f8_kernel<D, CAUSAL, HAS_DS, TO>;
  const int smem = (int)Smem<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)a.n_qtiles * (unsigned)(a.B * a.Hq);
  kern<<<grid, kThreadsAttn, smem, st>>>(tmQ, tmK, tmV, a);
  return cudaGetLastError();
}

template <int D, bool CAUSAL>
cudaError_t launch_attn_d(const AttnArgs& a, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                          cudaStream_t st) {
  if (a.dS) {
    return a.out_fp16 ? launch_attn_t<D, CAUSAL, true, __half>(a, q, k, v, st)
                      : launch_attn_t<D, CAUSAL, true, __nv_bfloat16>(a, q, k, v, st);
  }
  return a.out_fp16 ? launch_attn_t<D, CAUSAL, false, __half>(a, q, k, v, st)
                    : launch_attn_t<D, CAUSAL, false, __nv_bfloat16>(a, q, k, v, st);
}

}  // namespace

cudaError_t launch_attn_i8f8(const AttnArgs& a, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                             const CUtensorMap& tmV, cudaStream_t st) {
  if (a.D == 128)
    return a.causal ? launch_attn_d<128, true>(a, tmQ, tmK, tmV, st) : launch_attn_d<128, false>(a, tmQ, tmK, tmV, st);
  return a.causal ? launch_attn_d<64, true>(a, tmQ, tmK, tmV, st) : launch_attn_d<64, false>(a, tmQ, tmK, tmV, st);
}

cudaError_t launch_qk_probe(const AttnArgs& a, const CUtensorMap& tmQ, const CUtensorMap& tmK, cudaStream_t st) {
  const int smem = 256 * a.D + 64 + 1024;
  cudaError_t e;
  if (a.D == 128) {
    e = cudaFuncSetAttribute(qk_probe_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    qk_probe_kernel<128><<<1, 128, smem, st>>>(tmQ, tmK, a);
  } else {
    e = cudaFuncSetAttribute(qk_probe_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    qk_probe_kernel<64><<<1, 128, smem, st>>>(tmQ, tmK, a);
  }
  return cudaGetLastError();
}

cudaError_t launch_bounded_wait_probe(cudaStream_t st) {
  bounded_wait_probe_kernel<<<1, 32, 0, st>>>();
  return cudaGetLastError();
}

}  // namespace sage
