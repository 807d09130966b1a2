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
//   O     = e^(m_i,j-1 - m_ij) O + O_t             FP32 on CUDA cores (level 2)
//   out   = O / l / 448 * delta_V
// The exponentials run in base 2 (scores pre-multiplied by log2 e); the 448
// is folded into the exponent (exp2(t - m + log2 448)), so l accumulates
// 448 P~ and the final division by l absorbs the /448.
//
// CTA = one (batch, head) and TWO consecutive 128-row Q tiles that share every
// K / V tile.  512 threads in four warpgroups:
//   WG0  warp 0: TMA producer (Q tiles once, K_j / V_j^T through a ring)
//        warp 1: MMA issuer (one thread) and TMEM owner; warps 2-3 idle
//   WG1  softmax of Q tile 0    (thread = one Q row = one TMEM lane); in two-level
//        mode also the level-2 sum O = alpha O + O_t of its tile
//   WG2  the same for Q tile 1
//   WG3  (TMEM accumulator mode) the rescale of O before each P V; the epilogue
//        of both tiles (output through TMA bulk stores)
// The two softmax warpgroups run concurrently (two softmax warps per SM
// sub-partition hide each other's latencies).  TMEM (512 columns): S_i at
// [128 i, 128 i + 128), holding the magic fill 0x4B400000 between uses (QK^T
// accumulates onto it, see below), and O_i at [256 + D i, 256 + D (i + 1)).
// P goes through shared memory, two buffers per tile, so the softmax of tile
// j + 1 never waits for P V(j).
// Two P~V accumulation modes (template TWO_LEVEL):
//   two-level: PV(i, j) writes a fresh O_t into S_i's columns (S is dead once
//     the softmax read it); the softmax warpgroup of tile i adds it into O_i on
//     CUDA cores: O_i = alpha O_i + O_t (SageAttention2 Algorithm 1, level 2).
//   TMEM accumulator: PV(i, j) accumulates into O_i itself (tcgen05 keeps the
//     FP8 products' sum in full FP32); before it, the correction warpgroup
//     rescales the rows of O_i whose max grew (alpha != 1; alpha == 1 is exact).
#include <cfloat>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace sage {

namespace {

constexpr int kStages = 3;
constexpr int kThreadsAttn = 512;
constexpr float kLog2_448 = 8.807354922057604f;  // log2(448)
// S starts from the magic fill and gets it back after every read.  (Measured:
// this beats fresh int32 accumulators converted in the softmax by 10-16%.  The
// exp argument keeps the exact (y - 12582912) a - m: folding the offset into
// one FMA, y a - (12582912 a + m), rounds y a at 2^23 magnitude and broke the
// 1e-2 output tolerance on the prefill recipe.)
// Of the 8 element pairs in each 16-key group of the exp loop, those whose bit
// is set here compute 2^u with exp2_poly2 (FMA/ALU pipes) instead of ex2 (MUFU).
// Measured on B200: every split tried (1/4, 3/8, 1/2 of the pairs) was slower
// than MUFU only -- the loop is bound by issue slots, not by the MUFU rate.
#ifndef SAGE_POLY_PAIRS
#define SAGE_POLY_PAIRS 0x00
#endif
constexpr unsigned kPolyPairs = SAGE_POLY_PAIRS;

// per-warpgroup register budgets after setmaxnreg (sum x 128 <= 65536).  In
// TMEM-accumulator mode 56 / 192 / 72 (with the correction's rescale loop not
// unrolled) leaves no warpgroup spilling; the two-level instances keep
// 40 / 192 / 88, which measured faster for them than any spill-free split.
template <bool TWO_LEVEL>
constexpr uint32_t kRegsProducer = TWO_LEVEL ? 40 : 56;
constexpr uint32_t kRegsSoftmax = 192;
template <bool TWO_LEVEL>
constexpr uint32_t kRegsCorrection = TWO_LEVEL ? 88 : 72;
static_assert(kRegsProducer<true> + 2 * kRegsSoftmax + kRegsCorrection<true> <= 512 &&
                  kRegsProducer<false> + 2 * kRegsSoftmax + kRegsCorrection<false> <= 512,
              "register split exceeds the launch");

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int D>
struct Smem {
  static constexpr uint32_t kQ = 128 * D, kK = 128 * D, kV = D * 128, kP = 128 * 128;  // kP: one P buffer
  static constexpr uint32_t oQ = 0;                      // 2 tiles
  static constexpr uint32_t oK = oQ + 2 * kQ;            // kStages
  static constexpr uint32_t oV = oK + kStages * kK;      // kStages
  static constexpr uint32_t oP = oV + kStages * kV;      // [tile][2 buffers]
  static constexpr uint32_t kDS = 2 * 4 * 128 * 4;      // delta_S rows of one key tile: [tile][Q block (<= 4)][128]
  static constexpr uint32_t oDS = oP + 4 * kP;           // kStages
  static constexpr uint32_t oAlpha = oDS + kStages * kDS;  // float[tile][buffer][128]
  static constexpr uint32_t oL = oAlpha + 4 * 128 * 4;   // float[2][128] l, then float[2][128] m
  static constexpr uint32_t oSV = oL + 2 * 2 * 128 * 4;  // float[D] delta_V of the KV head (epilogue)
  static constexpr uint32_t oBar = oSV + D * 4;
  static constexpr uint32_t kNumBars = 1 + 3 * kStages + 2 + 4 + 4 + 2 + 2 + 2 + 2 + 1;
  static constexpr uint32_t oTmem = oBar + 8 * kNumBars;
  static constexpr uint32_t kBytes = oTmem + 16 + 1024;  // + alignment slack
  static_assert(kBytes <= 227 * 1024, "attention tile buffers exceed the shared memory of one CTA");
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

struct Bars {
  uint64_t* q_full;
  uint64_t* k_full;    // [kStages]  K_j (+ delta_S rows) landed
  uint64_t* v_full;    // [kStages]
  uint64_t* kv_empty;  // [kStages]
  uint64_t* s_full;    // [2]  QK^T of tile i done            (tcgen05.commit)
  uint64_t* p_full;    // [tile][buffer j & 1]  P_i(j) and alpha_i(j) written (one arrival per softmax
                       //      warp); one barrier per buffer keeps every waiter at most one phase behind
  uint64_t* p_empty;   // [tile][buffer]  the P V that read that P buffer retired (tcgen05.commit)
  uint64_t* ot_full;   // [2]  P V of tile i retired              (tcgen05.commit)
  uint64_t* r_free;    // [2]  S_i columns hold the magic fill again and may take the next QK^T
                       //      (the softmax refilled them; in two-level mode after it read
                       //      O_t_i there); one arrival per warp
  uint64_t* l_ready;   // [2]  final l of tile i in shared memory (128 threads)
  uint64_t* o_ready;   // [2]  (TMEM accumulator mode) O_i rescaled for the next P V (one per warp)
  uint64_t* mma_done;  // all tensor-core work of the CTA retired (one commit at the end)
};

// LSE: also write each row's log-sum-exp (a separate instance, so that kernels
// without it carry none of its code)
template <int D, bool CAUSAL, bool HAS_DS, bool TWO_LEVEL, typename TO, bool LSE>
__global__ void __launch_bounds__(kThreadsAttn, 1)
    attn_i8f8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                     const AttnArgs a) {
  using L = Smem<D>;
  constexpr uint32_t kSwzQK = (D == 128) ? kSwizzle128B : kSwizzle64B;
  constexpr uint32_t kSboQK = 8 * D;  // 8 rows x D bytes per swizzle atom
  constexpr uint32_t kIdescQK = make_idesc(/*S32*/ 2, /*s8*/ 1, /*s8*/ 1, 128, 128);
  constexpr uint32_t kIdescPV = make_idesc(/*F32*/ 1, /*E4M3*/ 0, /*E4M3*/ 0, 128, D);
  constexpr uint32_t kTmemCols = 512;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem + L::oQ;
  uint8_t* sK = smem + L::oK;
  uint8_t* sV = smem + L::oV;
  uint8_t* sP = smem + L::oP;
  const float* sDS = reinterpret_cast<const float*>(smem + L::oDS);
  float* s_alpha = reinterpret_cast<float*>(smem + L::oAlpha);
  float* s_l = reinterpret_cast<float*>(smem + L::oL);
  uint64_t* bar0 = reinterpret_cast<uint64_t*>(smem + L::oBar);
  Bars bar;
  bar.q_full = bar0;
  bar.k_full = bar0 + 1;
  bar.v_full = bar.k_full + kStages;
  bar.kv_empty = bar.v_full + kStages;
  bar.s_full = bar.kv_empty + kStages;
  bar.p_full = bar.s_full + 2;
  bar.p_empty = bar.p_full + 4;
  bar.ot_full = bar.p_empty + 4;
  bar.r_free = bar.ot_full + 2;
  bar.l_ready = bar.r_free + 2;
  bar.o_ready = bar.l_ready + 2;
  bar.mma_done = bar.o_ready + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::oTmem);

  // ---- work: (b, h, pair of Q tiles), heavy causal pairs first
  const int bhq = a.B * a.Hq;
  const int n_pairs = (a.n_qtiles + 1) / 2;
  const int pr = n_pairs - 1 - (int)(blockIdx.x / bhq);
  const int bh = blockIdx.x % bhq;
  const int b = bh / a.Hq, h = bh % a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  const int n_kt = (int)(a.Np / kTile);
  int nTi[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int qt = 2 * pr + i;
    nTi[i] = qt >= a.n_qtiles ? 0 : (CAUSAL ? qt + 1 : n_kt);
  }
  const int nT = nTi[0] > nTi[1] ? nTi[0] : nTi[1];

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int wg = warp / 4;
  // TMA loads of K_j (with the delta_S rows of both Q tiles) and V_j^T into
  // ring stage j % kStages; krow0 / vrow: the KV head's first K row and V^T row
  auto issue_kv = [&](int j, int krow0, int vrow) {
    const int s = j % kStages;
    const int ds_rows = kTile / a.bq;  // Q blocks per tile (1, 2 or 4)
    const uint32_t ds_bytes = (uint32_t)((nTi[0] > 0) + (nTi[1] > 0)) * ds_rows * 512;
    mbar_expect_tx(&bar.k_full[s], L::kK + (HAS_DS ? ds_bytes : 0u));
    tma_load_2d(sK + s * L::kK, &tmK, &bar.k_full[s], 0, krow0 + j * kTile);
    if (HAS_DS) {
      // delta_S[b, h, Q block, keys of tile j] for the Q blocks of both tiles
      for (int i = 0; i < 2; ++i)
        for (int hb = 0; hb < ds_rows; ++hb)
          if (nTi[i] > 0) {
            const int blk = min((2 * pr + i) * ds_rows + hb, a.Tm - 1);
            bulk_load_1d(smem + L::oDS + s * L::kDS + (i * 4 + hb) * 512,
                         a.dS + ((int64_t)(b * a.Hq + h) * a.Tm + blk) * a.Np + (int64_t)j * kTile, 512,
                         &bar.k_full[s]);
          }
    }
    mbar_expect_tx(&bar.v_full[s], L::kV);
    tma_load_2d(sV + s * L::kV, &tmV, &bar.v_full[s], j * kTile, vrow);
  };
  // Thread 0 initialises the barriers and, before the CTA's first barrier,
  // starts the loads of both Q tiles and of the first kStages K / V tiles, so
  // that their latency overlaps the TMEM allocation and the magic fill.  An
  // unread device error (a quantiser wait that ran out leaves some codes
  // unwritten) stops the launch before anything is computed from the
  // quantised tensors: O is left as it was rather than computed from stale
  // codes.  The error word is read first but looked at only after the loads
  // are out, so its latency is off their path; with an error pending the CTA
  // lets those loads land and ends.
  __shared__ int s_skip;
  if (threadIdx.x == 0) {
    const int pending = device_error_pending() ? 1 : 0;
    const int j_pre = nT < kStages ? nT : kStages;  // K / V tiles loaded before the first barrier
    mbar_init(bar.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar.s_full[i], 1);
      mbar_init(&bar.ot_full[i], 1);
      mbar_init(&bar.r_free[i], 4);
      mbar_init(&bar.l_ready[i], 128);
      mbar_init(&bar.o_ready[i], 4);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&bar.p_full[i], 4);
      mbar_init(&bar.p_empty[i], 1);
    }
    mbar_init(bar.mma_done, 1);
    mbar_fence_init();
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
    const int64_t qhead = (int64_t)(b * a.Hq + h) * a.Np;
    mbar_expect_tx(bar.q_full, (nTi[0] > 0 ? L::kQ : 0u) + (nTi[1] > 0 ? L::kQ : 0u));
    for (int i = 0; i < 2; ++i)
      if (nTi[i] > 0) tma_load_2d(sQ + i * L::kQ, &tmQ, bar.q_full, 0, (int)(qhead + (int64_t)(2 * pr + i) * kTile));
    const int krow0 = (int)((int64_t)(b * a.Hkv + g) * a.Np), vrow = (b * a.Hkv + g) * D;
    for (int j = 0; j < j_pre; ++j) issue_kv(j, krow0, vrow);
    s_skip = pending;
    if (pending) {
      // never leave a copy in flight (bounded waits)
      mbar_wait(bar.q_full, 0);
      for (int j = 0; j < j_pre; ++j) {
        mbar_wait(&bar.k_full[j], 0);
        mbar_wait(&bar.v_full[j], 0);
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (s_skip) {
    if (warp == 1) tmem_dealloc(*tmem_slot, kTmemCols);
    return;
  }
  const uint32_t tmem = *tmem_slot;
  // S accumulators start at the int32 bit pattern of 1.5 * 2^23: QK^T accumulates
  // onto it, so TMEM returns 0x4B400000 + acc, which read as fp32 is exactly
  // 12582912 + acc (|acc| <= 127 * 127 * 128 < 2^22): no int -> float step.
  if (wg == 1 || wg == 2) {
    const uint32_t tS0 = tmem + 128 * (wg - 1) + ((uint32_t)((warp & 3) * 32) << 16);
#pragma unroll
    for (int c = 0; c < 128; c += 8) tmem_fill8(tS0 + c, kMagicBits);
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (wg == 0) {
    regs_dec<kRegsProducer<TWO_LEVEL>>();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------ TMA producer
      // (Q and K / V tiles 0 .. kStages - 1 went out before the first barrier)
      const int krow0 = (int)((int64_t)(b * a.Hkv + g) * a.Np), vrow = (b * a.Hkv + g) * D;
      bool ok = true;
      int j = nT < kStages ? nT : kStages;  // (tiles below went out before the first barrier)
      for (; j < nT && ok; ++j) {
        if (!(ok = mbar_wait(&bar.kv_empty[j % kStages], ((j / kStages) + 1) & 1))) break;
        issue_kv(j, krow0, vrow);
      }
      // never leave a copy in flight
      for (int jj = (j - kStages > 0 ? j - kStages : 0); jj < j; ++jj) {
        mbar_wait(&bar.k_full[jj % kStages], (jj / kStages) & 1);
        mbar_wait(&bar.v_full[jj % kStages], (jj / kStages) & 1);
      }
      mbar_wait(bar.q_full, 0);
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        const uint32_t aP0 = smem_u32(sP);
        bool ok = mbar_wait(bar.q_full, 0);
        auto issue_qk = [&](int i, int j) {
          const int s = j % kStages;
          const uint32_t aQ = smem_u32(sQ + i * L::kQ), aK = smem_u32(sK + s * L::kK);
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            mma_i8(tmem + 128 * i, make_sdesc(aQ + kk * 32, kSboQK, kSwzQK), make_sdesc(aK + kk * 32, kSboQK, kSwzQK),
                   kIdescQK, 1u);  // accumulate onto the magic fill
          mma_commit(&bar.s_full[i]);
        };
        auto issue_pv = [&](int i, int j) {
          const int s = j % kStages;
          const uint32_t aP = aP0 + (i * 2 + (j & 1)) * L::kP, aV = smem_u32(sV + s * L::kV);
          // two-level: a fresh O_t tile in S_i's columns; else accumulate into O_i
          const uint32_t dst = TWO_LEVEL ? tmem + 128 * i : tmem + 256 + D * i;
#pragma unroll
          for (int kk = 0; kk < kTile / 32; ++kk)
            mma_f8f6f4(dst, make_sdesc(aP + kk * 32, 1024, kSwizzle128B), make_sdesc(aV + kk * 32, 1024, kSwizzle128B),
                       kIdescPV, (kk > 0 || (!TWO_LEVEL && j > 0)) ? 1u : 0u);
          mma_commit(&bar.ot_full[i]);
          mma_commit(&bar.p_empty[i * 2 + (j & 1)]);
        };
        // Two independent per-tile chains, each op issued as soon as its inputs
        // are ready (non-blocking polls), so one tile never holds the other back.
        //   QK(i,j): K_j landed; j > 0: S_i columns refilled (r_free) and, two-level,
        //            PV(i,j-1) issued (its O_t shares those columns)
        //   PV(i,j): QK(i,j) issued; V_j landed; P_i(j) written; TMEM-accumulator
        //            mode, j > 0: O_i rescaled (o_ready)
        // Stage j of the K/V ring is released once every active tile issued PV(i,j).
        int next_qk[2] = {0, 0}, next_pv[2] = {0, 0};
        int released = 0;
        uint64_t t_idle = 0;
        while (ok) {
          bool progress = false;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int jq = next_qk[i], jp = next_pv[i];
            if (jq < nTi[i] && (!TWO_LEVEL || jp >= jq) &&
                mbar_test_wait(smem_u32(&bar.k_full[jq % kStages]), (jq / kStages) & 1) &&
                (jq == 0 || mbar_test_wait(smem_u32(&bar.r_free[i]), (jq - 1) & 1))) {
              tc_fence_after();
              issue_qk(i, jq);
              next_qk[i] = jq + 1;
              progress = true;
            }
            if (jp < nTi[i] && next_qk[i] > jp &&
                mbar_test_wait(smem_u32(&bar.p_full[i * 2 + (jp & 1)]), (jp >> 1) & 1) &&
                mbar_test_wait(smem_u32(&bar.v_full[jp % kStages]), (jp / kStages) & 1) &&
                (TWO_LEVEL || jp == 0 || mbar_test_wait(smem_u32(&bar.o_ready[i]), (jp - 1) & 1))) {
              tc_fence_after();
              issue_pv(i, jp);
              next_pv[i] = jp + 1;
              progress = true;
            }
          }
          while (released < nT && (next_pv[0] > released || released >= nTi[0]) &&
                 (next_pv[1] > released || released >= nTi[1])) {
            mma_commit(&bar.kv_empty[released % kStages]);
            ++released;
          }
          if (next_pv[0] >= nTi[0] && next_pv[1] >= nTi[1] && released >= nT) break;
          // spin (a sleep here delays the reaction to a ready operand), bounded by the idle time
          if (progress) {
            t_idle = 0;
          } else if (t_idle == 0) {
            t_idle = globaltimer_ns();
          } else if (globaltimer_ns() - t_idle > g_wait_limit_ns) {
            record_error(kDevErrTimeout);
            ok = false;
          }
        }
        // every tensor-core op retired before TMEM is released
        mma_commit(bar.mma_done);
        mbar_wait(bar.mma_done, 0);
      }
      __syncwarp();
    }
  } else if (wg == 1 || wg == 2) {
    // ------------------------------------------------------------ softmax
    regs_inc<kRegsSoftmax>();
    const int ti = wg - 1;  // Q tile of this warpgroup
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int qtile = 2 * pr + ti;
    const int64_t qrow = (int64_t)qtile * kTile + row;
    const uint32_t tS = tmem + 128 * ti + ((uint32_t)(quarter * 32) << 16);
    const int qblk = min((int)(qrow / a.bq), a.Tm - 1);
    const float row_scale = a.s_q[(int64_t)(b * a.Hq + h) * a.Tm + qblk] * a.scale_log2;
    const float* sk = a.s_k + (int64_t)(b * a.Hkv + g) * a.Tn;
    // this row's Q block within the tile (warp-uniform: bq >= 32); a shift, not a
    // division by the runtime bq (which the compiler would redo in the tile loop)
    const int ds_blk = row >> (a.bq == 32 ? 5 : (a.bq == 64 ? 6 : 7));
    float sk_lo = __ldg(sk + 0), sk_hi = __ldg(sk + min(64 / a.bk, a.Tn - 1));
    const float sl2 = a.scale_log2;
    const float2 neg_magic = make_float2(-kMagic, -kMagic);
    float m = -INFINITY, l = 0.0f;
    bool ok = true;

    for (int j = 0; j < nTi[ti] && ok; ++j) {
      if (!(ok = mbar_wait_warp(&bar.s_full[ti], j & 1))) break;
      tc_fence_after();
      uint32_t s[128];  // fp32 bits of y = 12582912 + acc (acc = the INT8 dot product)
      tmem_ld32p(tS + 0, s + 0);
      tmem_ld32p(tS + 32, s + 32);
      tmem_ld32p(tS + 64, s + 64);
      tmem_ld32p(tS + 96, s + 96);
      const int col0 = j * kTile;
      // a = s_q s_k sm_scale log2 e per 64-key half, kept > 0 so that a masked
      // -inf stays -inf (a zero scale only multiplies zero dot products)
      const float a_lo = fmaxf(row_scale * sk_lo, FLT_MIN), a_hi = fmaxf(row_scale * sk_hi, FLT_MIN);
      // next tile's key-block scales (their load latency hides behind this tile)
      sk_lo = __ldg(sk + min((col0 + kTile) / a.bk, a.Tn - 1));
      sk_hi = __ldg(sk + min((col0 + kTile + 64) / a.bk, a.Tn - 1));
      const float* dsr = sDS + (j % kStages) * (L::kDS / 4) + (ti * 4 + ds_blk) * 128;
      if (HAS_DS && !(ok = mbar_wait_warp(&bar.k_full[j % kStages], (j / kStages) & 1))) break;
      tmem_ld_wait();
      if (!TWO_LEVEL) {
        // S_i is in registers: restore the magic fill, then the next QK^T may run
#pragma unroll
        for (int c = 0; c < 128; c += 8) tmem_fill8(tS + c, kMagicBits);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.r_free[ti]);
      }
      const bool need_mask = (col0 + kTile > a.N) || (CAUSAL && j == qtile);
      float mx;
      // with delta_S: x = (y - 12582912) + delta_S sm_scale log2 e / a in place, so
      // that the score is t = x a (a >= 1e-30 here keeps the quotient finite; a
      // zero scale only multiplies zero dot products)
      const float ad_lo = fmaxf(a_lo, 1e-30f), ad_hi = fmaxf(a_hi, 1e-30f);
      if (HAS_DS) {
        const float k_lo = sl2 / ad_lo, k_hi = sl2 / ad_hi;
#pragma unroll
        for (int c = 0; c < 128; c += 4) {
          const float kc = c < 64 ? k_lo : k_hi;
          const float4 ds = *reinterpret_cast<const float4*>(dsr + c);
          const float2 x0 = ffma2(make_float2(ds.x, ds.y), make_float2(kc, kc),
                                  fadd2(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), neg_magic));
          const float2 x1 = ffma2(make_float2(ds.z, ds.w), make_float2(kc, kc),
                                  fadd2(make_float2(__uint_as_float(s[c + 2]), __uint_as_float(s[c + 3])), neg_magic));
          s[c] = __float_as_uint(x0.x);
          s[c + 1] = __float_as_uint(x0.y);
          s[c + 2] = __float_as_uint(x1.x);
          s[c + 3] = __float_as_uint(x1.y);
        }
      }
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const int col = col0 + c;
          // -inf as y (or, raw int32 without the fill, the value whose y is -inf)
          if (col >= a.N || (CAUSAL && col > qrow)) s[c] = __float_as_uint(-INFINITY);
        }
      }
      if (HAS_DS) {
        // row max of t = x a per 64-key half (a > 0 keeps the order of x)
        float mx8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 64; c += 8)
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            mx8[k] = fmax3(mx8[k], __uint_as_float(s[c + 2 * k]), __uint_as_float(s[c + 2 * k + 1]));
            mx8[4 + k] = fmax3(mx8[4 + k], __uint_as_float(s[64 + c + 2 * k]), __uint_as_float(s[64 + c + 2 * k + 1]));
          }
        mx = fmaxf(fmax3(mx8[0], mx8[1], fmaxf(mx8[2], mx8[3])) * ad_lo,
                   fmax3(mx8[4], mx8[5], fmaxf(mx8[6], mx8[7])) * ad_hi);
      } else {
        // y is monotonic in acc: take the max of each 64-key half on y and scale
        // only the two maxima
        float mx8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 64; c += 8)
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            mx8[k] = fmax3(mx8[k], __uint_as_float(s[c + 2 * k]), __uint_as_float(s[c + 2 * k + 1]));
            mx8[4 + k] = fmax3(mx8[4 + k], __uint_as_float(s[64 + c + 2 * k]), __uint_as_float(s[64 + c + 2 * k + 1]));
          }
        const float ylo = fmax3(mx8[0], mx8[1], fmaxf(mx8[2], mx8[3]));
        const float yhi = fmax3(mx8[4], mx8[5], fmaxf(mx8[6], mx8[7]));
        mx = fmaxf((ylo - kMagic) * a_lo, (yhi - kMagic) * a_hi);
      }
      const float m_new = fmaxf(m, mx);
      const float alpha = (m == -INFINITY) ? 0.0f : ex2_approx(m - m_new);
      const float mm = (m_new == -INFINITY) ? 0.0f : m_new - kLog2_448;
      // P buffer (j & 1) is free once P V(j - 2) retired
      if (j >= 2 && !(ok = mbar_wait_warp(&bar.p_empty[ti * 2 + (j & 1)], ((j >> 1) - 1) & 1))) break;
      uint8_t* myP = sP + (ti * 2 + (j & 1)) * L::kP + row * 128;
      // P = exp2(t - m + log2 448) -> E4M3 -> shared memory (128B-swizzled K-major)
      // row sum: 8 independent f32x2 partial sums (fp32 rounding order only)
      float2 rs[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) rs[k] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int grp = 0; grp < 8; ++grp) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          const int c = grp * 16 + e;
          float2 u0, u1;
          const float2 y0 = make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1]));
          const float2 y1 = make_float2(__uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
          if (HAS_DS) {
            const float sc = c < 64 ? ad_lo : ad_hi;
            u0 = ffma2(y0, make_float2(sc, sc), make_float2(-mm, -mm));
            u1 = ffma2(y1, make_float2(sc, sc), make_float2(-mm, -mm));
          } else {
            const float sc = c < 64 ? a_lo : a_hi;
            u0 = ffma2(fadd2(y0, neg_magic), make_float2(sc, sc), make_float2(-mm, -mm));
            u1 = ffma2(fadd2(y1, neg_magic), make_float2(sc, sc), make_float2(-mm, -mm));
          }
          // pairs selected by kPolyPairs take the FMA-pipe exponential, the rest MUFU
          const float2 p0 = ((kPolyPairs >> (e / 2)) & 1) ? exp2_poly2(u0)
                                                          : make_float2(ex2_approx(u0.x), ex2_approx(u0.y));
          const float2 p1 = ((kPolyPairs >> (e / 2 + 1)) & 1) ? exp2_poly2(u1)
                                                              : make_float2(ex2_approx(u1.x), ex2_approx(u1.y));
          rs[e / 2] = fadd2(rs[e / 2], p0);
          rs[e / 2 + 1] = fadd2(rs[e / 2 + 1], p1);
          w[e / 4] = cvt_e4m3x4(p0.x, p0.y, p1.x, p1.y);
        }
        *reinterpret_cast<uint4*>(myP + ((grp ^ (row & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      const float2 rs2 = fadd2(fadd2(fadd2(rs[0], rs[1]), fadd2(rs[2], rs[3])),
                               fadd2(fadd2(rs[4], rs[5]), fadd2(rs[6], rs[7])));
      s_alpha[(ti * 2 + (j & 1)) * 128 + row] = alpha;
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.p_full[ti * 2 + (j & 1)]);
      l = fmaf(l, alpha, rs2.x + rs2.y);
      m = m_new;
      if constexpr (TWO_LEVEL) {
        // Level 2 in this warpgroup, whose registers can hold a whole O_t row:
        // P V(j) put a fresh O_t into S_i's columns [0, D).  Read it (S is dead),
        // give S_i's columns their magic fill back and let the next Q K^T run,
        // then form O = alpha O + O_t while that MMA works.
        if (!(ok = mbar_wait_warp(&bar.ot_full[ti], j & 1))) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D; c += 32) tmem_ld32p(tS + c, s + c);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 128; c += 8) tmem_fill8(tS + c, kMagicBits);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.r_free[ti]);
        const uint32_t tO = tmem + 256 + D * ti + ((uint32_t)(quarter * 32) << 16);
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t x[32];
          if (j == 0) {
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = s[c + e];
          } else {
            tmem_ld32(tO + c, x);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 o = ffma2(make_float2(__uint_as_float(x[e]), __uint_as_float(x[e + 1])),
                                     make_float2(alpha, alpha),
                                     make_float2(__uint_as_float(s[c + e]), __uint_as_float(s[c + e + 1])));
              x[e] = __float_as_uint(o.x);
              x[e + 1] = __float_as_uint(o.y);
            }
          }
          tmem_st32(tO + c, x);
        }
        tmem_st_wait();  // O is final before l_ready (the epilogue reads it)
      }
    }
    s_l[ti * 128 + row] = l;
    if (LSE) s_l[256 + ti * 128 + row] = m;
    tc_fence_before();  // (two-level) this warp's O stores before the epilogue's reads
    mbar_arrive(&bar.l_ready[ti]);
  } else {
    // ------------------------------------------------------------ correction + epilogue
    regs_dec<kRegsCorrection<TWO_LEVEL>>();
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    uint32_t x[32];
    // delta_V of this KV head into shared memory now, while the tile loop
    // runs: read from global in the epilogue, its first touch of each line
    // would miss L1 once per 32-column chunk
    float* s_sv = reinterpret_cast<float*>(smem + L::oSV);
    if (row < D) s_sv[row] = __ldg(a.s_v + (int64_t)(b * a.Hkv + g) * D + row);
    named_bar_sync(1, 128);
    // every phase of p_full[tile][buffer] is waited in order, j = 0 included (a
    // parity wait on a phase two ahead of the barrier would pass at once).
    // Two-level mode: the softmax warpgroups form the level-2 sums themselves;
    // this warpgroup only writes the output.
    if constexpr (TWO_LEVEL) {
    } else {
      // O_i accumulates in TMEM; before PV(i, j) adds tile j, rows whose max grew
      // are rescaled by alpha = e^(m_old - m_new).  A warp whose 32 rows all have
      // alpha == 1 leaves O_i untouched (exact).
      for (int j = 0; j < nT && ok; ++j) {
        for (int i = 0; i < 2; ++i) {
          if (j >= nTi[i]) continue;
          if (!(ok = mbar_wait_warp(&bar.p_full[i * 2 + (j & 1)], (j >> 1) & 1))) break;
          if (j == 0) continue;
          if (!(ok = mbar_wait_warp(&bar.ot_full[i], (j - 1) & 1))) break;
          tc_fence_after();
          const float alpha = s_alpha[(i * 2 + (j & 1)) * 128 + row];
          if (__any_sync(0xffffffffu, alpha != 1.0f)) {
            const uint32_t tO = tmem + 256 + D * i + lane_off;
            // (not unrolled: it keeps this warpgroup within its 72 registers)
#pragma unroll 1
            for (int c = 0; c < D; c += 32) {
              tmem_ld32(tO + c, x);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                const float2 o = fmul2(make_float2(__uint_as_float(x[e]), __uint_as_float(x[e + 1])),
                                       make_float2(alpha, alpha));
                x[e] = __float_as_uint(o.x);
                x[e + 1] = __float_as_uint(o.y);
              }
              tmem_st32(tO + c, x);
            }
            tmem_st_wait();
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar.o_ready[i]);
        }
      }
    }
    // epilogue: out = O / l * delta_V   (l carries the 448)
    for (int i = 0; i < 2 && ok; ++i) {
      if (nTi[i] == 0) continue;
      if (!(ok = mbar_wait_warp(&bar.l_ready[i], 0))) break;
      if (!TWO_LEVEL && !(ok = mbar_wait_warp(&bar.ot_full[i], (nTi[i] - 1) & 1))) break;
      tc_fence_after();
      const float inv_l = 1.0f / s_l[i * 128 + row];
      const int64_t qrow = (int64_t)(2 * pr + i) * kTile + row;
      if (LSE && qrow < a.N) {
        // ln sum_j e^(S_ij) = (m + log2(l / 448)) ln 2 (m: running max of the
        // log2-domain scores, l: sum of 448 2^(t - m)), plus the smooth-K shift
        const float l = s_l[i * 128 + row], m = s_l[256 + i * 128 + row];
        const int64_t bhq = (int64_t)(b * a.Hq + h);
        a.lse[bhq * a.N + qrow] =
            l > 0.0f ? (m + log2f(l) - kLog2_448) * 0.69314718055994531f + a.sm_scale * a.qkm[bhq * a.Np + qrow]
                     : -INFINITY;
      }
      // The warp stages its 32 output rows in tile i's P buffers (free: the
      // tile's last P V retired) as boxes of 64 columns x 32 rows in the TMA
      // 128-byte swizzle (16-byte chunk q of row r at q ^ (r & 7)), and one lane
      // writes them out with bulk tensor stores (rows past N are clipped by the
      // tensor map): no per-thread global stores.
      constexpr int kBoxes = D * (int)sizeof(TO) / 128;  // 64-column boxes per row (1 or 2)
      uint8_t* stg = sP + i * 2 * L::kP + quarter * kBoxes * 4096;
      const uint32_t tO = tmem + 256 + D * i + lane_off;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        tmem_ld32(tO + c, x);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          float f[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) f[u] = __uint_as_float(x[e + u]) * inv_l * s_sv[c + e + u];
          const int col = c + e, q = (col % 64) / 8;
          *reinterpret_cast<uint4*>(stg + (col / 64) * 4096 + lane * 128 + ((q ^ (lane & 7)) << 4)) =
              make_uint4(pack2<TO>(f[0], f[1]), pack2<TO>(f[2], f[3]), pack2<TO>(f[4], f[5]), pack2<TO>(f[6], f[7]));
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      const int qrow0 = (2 * pr + i) * kTile + quarter * 32;
      if (lane == 0 && qrow0 < a.N) {
#pragma unroll
        for (int bx = 0; bx < kBoxes; ++bx) tma_store_4d(&tmO, stg + bx * 4096, bx * 64, qrow0, h, b);
        bulk_commit();
      }
    }
    // the bulk stores have read their shared-memory source before the CTA ends
    if (lane == 0) bulk_wait_read_all();
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
// Split-row variant, taken when delta_S is added (smooth Q).  Folding delta_S
// into the scores costs every score another FMA and a shared-memory read in
// the softmax, whose instruction stream bounds the kernel; here each 128-key
// tile of a Q row is split between two warps, so twice the warps share that
// work.  640 threads in five warpgroups:
//   WG0      warp 0: TMA producer; warp 1: MMA issuer and TMEM owner
//   WG1, 2   Q tile 0, key columns [0, 64) and [64, 128) of every K tile, and
//            O columns [0, D/2) and [D/2, D) (rescale / level-2 sum, epilogue)
//   WG3, 4   the same for Q tile 1
// The two warps on the same 32 TMEM lanes (one row each per thread) exchange
// their half-row maxima through shared memory, so both quantise P with the
// row's maximum; their row sums are added at the end.  The schedule, the
// TMEM layout and the shared-memory operands are those of the kernel above;
// without delta_S that kernel is faster (its exchange-free rows beat the
// halved work).
constexpr int kThreadsSplit = 640;

// per-warpgroup register budgets of the split-row kernel after setmaxnreg (640 threads launch with
// 96 registers each; the five warpgroups must not ask for more in total)
constexpr uint32_t kRegsSplitProducer = 32, kRegsSplitSoftmax = 112;
static_assert(kRegsSplitProducer + 4 * kRegsSplitSoftmax <= 5 * 96, "register split exceeds the launch");

template <int D>
struct SmemSplit {
  static constexpr uint32_t kQ = 128 * D, kK = 128 * D, kV = D * 128, kP = 128 * 128;  // kP: one P buffer
  static constexpr uint32_t oQ = 0;                      // 2 tiles
  static constexpr uint32_t oK = oQ + 2 * kQ;            // kStages
  static constexpr uint32_t oV = oK + kStages * kK;      // kStages
  static constexpr uint32_t oP = oV + kStages * kV;      // [tile][2 buffers]
  static constexpr uint32_t kDS = 2 * 4 * 128 * 4;      // delta_S rows of one key tile: [tile][Q block (<= 4)][128]
  static constexpr uint32_t oDS = oP + 4 * kP;           // kStages
  static constexpr uint32_t oMx = oDS + kStages * kDS;   // float[buffer j & 1][tile][half][128] half-row maxima
  static constexpr uint32_t oL = oMx + 2 * 2 * 2 * 128 * 4;  // float[tile][half][128] l, then [tile][128] m
  static constexpr uint32_t oBar = oL + (2 * 2 * 128 + 2 * 128) * 4;
  static constexpr uint32_t kNumBars = 1 + 3 * kStages + 2 + 4 + 4 + 2 + 2 + 2 + 1 + 16 + 8;
  static constexpr uint32_t oTmem = oBar + 8 * kNumBars;
  static constexpr uint32_t kBytes = oTmem + 16 + 1024;  // + alignment slack
  static_assert(kBytes <= 227 * 1024, "attention tile buffers exceed the shared memory of one CTA");
};

struct BarsSplit {
  uint64_t* q_full;
  uint64_t* k_full;    // [kStages]  K_j (+ delta_S rows) landed
  uint64_t* v_full;    // [kStages]
  uint64_t* kv_empty;  // [kStages]
  uint64_t* s_full;    // [2]  QK^T of tile i done            (tcgen05.commit)
  uint64_t* p_full;    // [tile][buffer j & 1]  P_i(j) written (one arrival per softmax warp of the
                       //      tile, 8); one barrier per buffer keeps every waiter at most one phase behind
  uint64_t* p_empty;   // [tile][buffer]  the P V that read that P buffer retired (tcgen05.commit)
  uint64_t* ot_full;   // [2]  P V of tile i retired              (tcgen05.commit)
  uint64_t* r_free;    // [2]  S_i columns hold the magic fill again and may take the next QK^T
                       //      (TMEM accumulator: S read; two-level: O_t read); one arrival per warp
  uint64_t* o_ready;   // [2]  (TMEM accumulator mode) O_i rescaled by alpha_i(j) for P V(i, j); one
                       //      arrival per softmax warp, every j
  uint64_t* mma_done;  // all tensor-core work of the CTA retired (one commit at the end)
  uint64_t* mx;        // [tile][lane quarter][buffer j & 1]  both halves of these rows posted their
                       //      maximum of tile j (one arrival per warp, 2)
  uint64_t* lx;        // [tile][lane quarter]  both halves posted their row sums (2)
};

// LSE: also write each row's log-sum-exp (a separate instance, so that kernels
// without it carry none of its code)
template <int D, bool CAUSAL, bool HAS_DS, bool TWO_LEVEL, typename TO, bool LSE>
__global__ void __launch_bounds__(kThreadsSplit, 1)
    attn_i8f8_split_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV,
                           const __grid_constant__ CUtensorMap /*tmO: unused*/, const AttnArgs a) {
  using L = SmemSplit<D>;
  constexpr uint32_t kSwzQK = (D == 128) ? kSwizzle128B : kSwizzle64B;
  constexpr uint32_t kSboQK = 8 * D;  // 8 rows x D bytes per swizzle atom
  constexpr uint32_t kIdescQK = make_idesc(/*S32*/ 2, /*s8*/ 1, /*s8*/ 1, 128, 128);
  constexpr uint32_t kIdescPV = make_idesc(/*F32*/ 1, /*E4M3*/ 0, /*E4M3*/ 0, 128, D);
  constexpr uint32_t kTmemCols = 512;
  constexpr int DH = D / 2;  // O columns per softmax half

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem + L::oQ;
  uint8_t* sK = smem + L::oK;
  uint8_t* sV = smem + L::oV;
  uint8_t* sP = smem + L::oP;
  const float* sDS = reinterpret_cast<const float*>(smem + L::oDS);
  float* s_mx = reinterpret_cast<float*>(smem + L::oMx);
  float* s_l = reinterpret_cast<float*>(smem + L::oL);
  uint64_t* bar0 = reinterpret_cast<uint64_t*>(smem + L::oBar);
  BarsSplit bar;
  bar.q_full = bar0;
  bar.k_full = bar0 + 1;
  bar.v_full = bar.k_full + kStages;
  bar.kv_empty = bar.v_full + kStages;
  bar.s_full = bar.kv_empty + kStages;
  bar.p_full = bar.s_full + 2;
  bar.p_empty = bar.p_full + 4;
  bar.ot_full = bar.p_empty + 4;
  bar.r_free = bar.ot_full + 2;
  bar.o_ready = bar.r_free + 2;
  bar.mma_done = bar.o_ready + 2;
  bar.mx = bar.mma_done + 1;
  bar.lx = bar.mx + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::oTmem);

  // An unread device error (a quantiser wait that ran out leaves some codes
  // unwritten) stops the launch before it reads the quantised tensors: O is
  // left as it was rather than computed from stale codes.
  __shared__ int s_skip;
  if (threadIdx.x == 0) s_skip = device_error_pending() ? 1 : 0;
  __syncthreads();
  if (s_skip) return;

  // ---- work: (b, h, pair of Q tiles), heavy causal pairs first
  const int bhq = a.B * a.Hq;
  const int n_pairs = (a.n_qtiles + 1) / 2;
  const int pr = n_pairs - 1 - (int)(blockIdx.x / bhq);
  const int bh = blockIdx.x % bhq;
  const int b = bh / a.Hq, h = bh % a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  const int n_kt = (int)(a.Np / kTile);
  int nTi[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int qt = 2 * pr + i;
    nTi[i] = qt >= a.n_qtiles ? 0 : (CAUSAL ? qt + 1 : n_kt);
  }
  const int nT = nTi[0] > nTi[1] ? nTi[0] : nTi[1];

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int wg = warp / 4;
  if (threadIdx.x == 0) {
    mbar_init(bar.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar.s_full[i], 1);
      mbar_init(&bar.ot_full[i], 1);
      mbar_init(&bar.r_free[i], 8);
      mbar_init(&bar.o_ready[i], 8);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&bar.p_full[i], 8);
      mbar_init(&bar.p_empty[i], 1);
    }
    mbar_init(bar.mma_done, 1);
    for (int i = 0; i < 16; ++i) mbar_init(&bar.mx[i], 2);
    for (int i = 0; i < 8; ++i) mbar_init(&bar.lx[i], 2);
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
  // S accumulators start at the int32 bit pattern of 1.5 * 2^23: QK^T accumulates
  // onto it, so TMEM returns 0x4B400000 + acc, which read as fp32 is exactly
  // 12582912 + acc (|acc| <= 127 * 127 * 128 < 2^22): no int -> float step.
  // Each softmax warp fills (and later refills) its half of its tile's columns.
  if (wg >= 1) {
    const int ti = (wg - 1) >> 1, hf = (wg - 1) & 1;
    const uint32_t tS0 = tmem + 128 * ti + 64 * hf + ((uint32_t)((warp & 3) * 32) << 16);
#pragma unroll
    for (int c = 0; c < 64; c += 8) tmem_fill8(tS0 + c, kMagicBits);
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (wg == 0) {
    regs_dec<kRegsSplitProducer>();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------ TMA producer
      tma_prefetch_map(&tmQ);
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      const int64_t qhead = (int64_t)(b * a.Hq + h) * a.Np;
      const int krow0 = (int)((int64_t)(b * a.Hkv + g) * a.Np);
      const int vrow = (b * a.Hkv + g) * D;
      const int ds_rows = kTile / a.bq;  // Q blocks per tile (1, 2 or 4)
      const uint32_t ds_bytes = (uint32_t)((nTi[0] > 0) + (nTi[1] > 0)) * ds_rows * 512;
      mbar_expect_tx(bar.q_full, (nTi[0] > 0 ? L::kQ : 0u) + (nTi[1] > 0 ? L::kQ : 0u));
      for (int i = 0; i < 2; ++i)
        if (nTi[i] > 0) tma_load_2d(sQ + i * L::kQ, &tmQ, bar.q_full, 0, (int)(qhead + (int64_t)(2 * pr + i) * kTile));
      bool ok = true;
      int j = 0;
      for (; j < nT && ok; ++j) {
        const int s = j % kStages;
        if (j >= kStages) ok = mbar_wait(&bar.kv_empty[s], ((j / kStages) + 1) & 1);
        if (!ok) break;
        mbar_expect_tx(&bar.k_full[s], L::kK + (HAS_DS ? ds_bytes : 0u));
        tma_load_2d(sK + s * L::kK, &tmK, &bar.k_full[s], 0, krow0 + j * kTile);
        if (HAS_DS) {
          // delta_S[b, h, Q block, keys of tile j] for the Q blocks of both tiles
          for (int i = 0; i < 2; ++i)
            for (int hb = 0; hb < ds_rows; ++hb)
              if (nTi[i] > 0) {
                const int blk = min((2 * pr + i) * ds_rows + hb, a.Tm - 1);
                bulk_load_1d(smem + L::oDS + s * L::kDS + (i * 4 + hb) * 512,
                             a.dS + ((int64_t)(b * a.Hq + h) * a.Tm + blk) * a.Np + (int64_t)j * kTile, 512,
                             &bar.k_full[s]);
              }
        }
        mbar_expect_tx(&bar.v_full[s], L::kV);
        tma_load_2d(sV + s * L::kV, &tmV, &bar.v_full[s], j * kTile, vrow);
      }
      // never leave a copy in flight
      for (int jj = (j - kStages > 0 ? j - kStages : 0); jj < j; ++jj) {
        mbar_wait(&bar.k_full[jj % kStages], (jj / kStages) & 1);
        mbar_wait(&bar.v_full[jj % kStages], (jj / kStages) & 1);
      }
      mbar_wait(bar.q_full, 0);
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        const uint32_t aP0 = smem_u32(sP);
        bool ok = mbar_wait(bar.q_full, 0);
        auto issue_qk = [&](int i, int j) {
          const int s = j % kStages;
          const uint32_t aQ = smem_u32(sQ + i * L::kQ), aK = smem_u32(sK + s * L::kK);
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            mma_i8(tmem + 128 * i, make_sdesc(aQ + kk * 32, kSboQK, kSwzQK), make_sdesc(aK + kk * 32, kSboQK, kSwzQK),
                   kIdescQK, 1u);  // accumulate onto the magic fill
          mma_commit(&bar.s_full[i]);
        };
        auto issue_pv = [&](int i, int j) {
          const int s = j % kStages;
          const uint32_t aP = aP0 + (i * 2 + (j & 1)) * L::kP, aV = smem_u32(sV + s * L::kV);
          // two-level: a fresh O_t tile in S_i's columns; else accumulate into O_i
          const uint32_t dst = TWO_LEVEL ? tmem + 128 * i : tmem + 256 + D * i;
#pragma unroll
          for (int kk = 0; kk < kTile / 32; ++kk)
            mma_f8f6f4(dst, make_sdesc(aP + kk * 32, 1024, kSwizzle128B), make_sdesc(aV + kk * 32, 1024, kSwizzle128B),
                       kIdescPV, (kk > 0 || (!TWO_LEVEL && j > 0)) ? 1u : 0u);
          mma_commit(&bar.ot_full[i]);
          mma_commit(&bar.p_empty[i * 2 + (j & 1)]);
        };
        // Two independent per-tile chains, each op issued as soon as its inputs
        // are ready (non-blocking polls), so one tile never holds the other back.
        //   QK(i,j): K_j landed; j > 0: S_i columns refilled (r_free) and, two-level,
        //            PV(i,j-1) issued (its O_t shares those columns)
        //   PV(i,j): QK(i,j) issued; V_j landed; P_i(j) written; TMEM-accumulator
        //            mode: O_i rescaled by alpha_i(j) (o_ready phase j)
        // Stage j of the K/V ring is released once every active tile issued PV(i,j).
        int next_qk[2] = {0, 0}, next_pv[2] = {0, 0};
        int released = 0;
        uint64_t t_idle = 0;
        while (ok) {
          bool progress = false;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int jq = next_qk[i], jp = next_pv[i];
            if (jq < nTi[i] && (!TWO_LEVEL || jp >= jq) &&
                mbar_test_wait(smem_u32(&bar.k_full[jq % kStages]), (jq / kStages) & 1) &&
                (jq == 0 || mbar_test_wait(smem_u32(&bar.r_free[i]), (jq - 1) & 1))) {
              tc_fence_after();
              issue_qk(i, jq);
              next_qk[i] = jq + 1;
              progress = true;
            }
            if (jp < nTi[i] && next_qk[i] > jp &&
                mbar_test_wait(smem_u32(&bar.p_full[i * 2 + (jp & 1)]), (jp >> 1) & 1) &&
                mbar_test_wait(smem_u32(&bar.v_full[jp % kStages]), (jp / kStages) & 1) &&
                (TWO_LEVEL || mbar_test_wait(smem_u32(&bar.o_ready[i]), jp & 1))) {
              tc_fence_after();
              issue_pv(i, jp);
              next_pv[i] = jp + 1;
              progress = true;
            }
          }
          while (released < nT && (next_pv[0] > released || released >= nTi[0]) &&
                 (next_pv[1] > released || released >= nTi[1])) {
            mma_commit(&bar.kv_empty[released % kStages]);
            ++released;
          }
          if (next_pv[0] >= nTi[0] && next_pv[1] >= nTi[1] && released >= nT) break;
          // spin (a sleep here delays the reaction to a ready operand), bounded by the idle time
          if (progress) {
            t_idle = 0;
          } else if (t_idle == 0) {
            t_idle = globaltimer_ns();
          } else if (globaltimer_ns() - t_idle > g_wait_limit_ns) {
            record_error(kDevErrTimeout);
            ok = false;
          }
        }
        // every tensor-core op retired before TMEM is released
        mma_commit(bar.mma_done);
        mbar_wait(bar.mma_done, 0);
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ softmax, accumulation, epilogue
    // Warpgroups 1, 2 take Q tile 0 and 3, 4 tile 1; within a tile warpgroup
    // hf = 0 owns key columns [0, 64) of every 128-key tile and O columns
    // [0, D/2), hf = 1 the other halves.  A thread owns one Q row (one TMEM
    // lane) in both; the two halves of a row exchange their maxima through
    // shared memory (an mbarrier of the two warps on the same 32 lanes), so
    // both quantise P with the same row max, and add their partial row sums
    // at the end.
    regs_inc<kRegsSplitSoftmax>();
    const int ti = (wg - 1) >> 1;  // Q tile
    const int hf = (wg - 1) & 1;   // column half
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int qtile = 2 * pr + ti;
    const int64_t qrow = (int64_t)qtile * kTile + row;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + 128 * ti + 64 * hf + lane_off;  // this half's 64 S columns
    const uint32_t tO = tmem + 256 + D * ti + DH * hf + lane_off;  // this half's D/2 O columns
    uint64_t* mxbar = bar.mx + (ti * 4 + quarter) * 2;  // the two warps on these lanes, per buffer
    const int qblk = min((int)(qrow / a.bq), a.Tm - 1);
    const float row_scale = a.s_q[(int64_t)(b * a.Hq + h) * a.Tm + qblk] * a.scale_log2;
    const float* sk = a.s_k + (int64_t)(b * a.Hkv + g) * a.Tn;
    // this row's Q block within the tile (warp-uniform: bq >= 32); a shift, not a
    // division by the runtime bq (which the compiler would redo in the tile loop)
    const int ds_blk = row >> (a.bq == 32 ? 5 : (a.bq == 64 ? 6 : 7));
    // key-block scale of this half's 64 keys (bk = 64: one block; bk = 128: the tile's)
    float sk_h = __ldg(sk + min((64 * hf) / a.bk, a.Tn - 1));
    const float sl2 = a.scale_log2;
    const float2 neg_magic = make_float2(-kMagic, -kMagic);
    float m = -INFINITY, l = 0.0f;
    bool ok = true;
    uint32_t x[32];

    for (int j = 0; j < nTi[ti] && ok; ++j) {
      if (!(ok = mbar_wait_warp(&bar.s_full[ti], j & 1))) break;
      tc_fence_after();
      uint32_t s[64];  // fp32 bits of y = 12582912 + acc (acc = the INT8 dot product)
      tmem_ld32p(tS + 0, s + 0);
      tmem_ld32p(tS + 32, s + 32);
      const int col0 = j * kTile + 64 * hf;
      // a = s_q s_k sm_scale log2 e of this half's keys, kept > 0 so that a masked
      // -inf stays -inf (a zero scale only multiplies zero dot products)
      const float a_h = fmaxf(row_scale * sk_h, FLT_MIN);
      // next tile's key-block scale (its load latency hides behind this tile)
      sk_h = __ldg(sk + min((j * kTile + kTile + 64 * hf) / a.bk, a.Tn - 1));
      const float* dsr = sDS + (j % kStages) * (L::kDS / 4) + (ti * 4 + ds_blk) * 128 + 64 * hf;
      if (HAS_DS && !(ok = mbar_wait_warp(&bar.k_full[j % kStages], (j / kStages) & 1))) break;
      tmem_ld_wait();
      if (!TWO_LEVEL) {
        // S_i is in registers: restore the magic fill, then the next QK^T may run
#pragma unroll
        for (int c = 0; c < 64; c += 8) tmem_fill8(tS + c, kMagicBits);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.r_free[ti]);
      }
      const bool need_mask = (j * kTile + kTile > a.N) || (CAUSAL && j == qtile);
      // with delta_S: x = (y - 12582912) + delta_S sm_scale log2 e / a in place, so
      // that the score is t = x a (a >= 1e-30 here keeps the quotient finite)
      const float ad = fmaxf(a_h, 1e-30f);
      if (HAS_DS) {
        const float kc = sl2 / ad;
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          const float4 ds = *reinterpret_cast<const float4*>(dsr + c);
          const float2 x0 = ffma2(make_float2(ds.x, ds.y), make_float2(kc, kc),
                                  fadd2(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), neg_magic));
          const float2 x1 = ffma2(make_float2(ds.z, ds.w), make_float2(kc, kc),
                                  fadd2(make_float2(__uint_as_float(s[c + 2]), __uint_as_float(s[c + 3])), neg_magic));
          s[c] = __float_as_uint(x0.x);
          s[c + 1] = __float_as_uint(x0.y);
          s[c + 2] = __float_as_uint(x1.x);
          s[c + 3] = __float_as_uint(x1.y);
        }
      }
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int col = col0 + c;
          if (col >= a.N || (CAUSAL && col > qrow)) s[c] = __float_as_uint(-INFINITY);
        }
      }
      // max of this half (on the raw values: x, or y, is monotonic in the score)
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; c += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = fmax3(mx8[k], __uint_as_float(s[c + 2 * k]), __uint_as_float(s[c + 2 * k + 1]));
      const float mraw = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
      const float mx_h = HAS_DS ? mraw * ad : (mraw - kMagic) * a_h;
      // the row max over both halves (the partner warp's value of this tile)
      float* mxb = s_mx + (j & 1) * 512 + ti * 256;
      mxb[hf * 128 + row] = mx_h;
      __syncwarp();
      if (lane == 0) mbar_arrive(&mxbar[j & 1]);
      if (!(ok = mbar_wait_warp(&mxbar[j & 1], (j >> 1) & 1))) break;
      const float m_new = fmaxf(m, fmaxf(mx_h, mxb[(1 - hf) * 128 + row]));
      const float alpha = (m == -INFINITY) ? 0.0f : ex2_approx(m - m_new);
      const float mm = (m_new == -INFINITY) ? 0.0f : m_new - kLog2_448;
      // P buffer (j & 1) is free once P V(j - 2) retired
      if (j >= 2 && !(ok = mbar_wait_warp(&bar.p_empty[ti * 2 + (j & 1)], ((j >> 1) - 1) & 1))) break;
      uint8_t* myP = sP + (ti * 2 + (j & 1)) * L::kP + row * 128;
      // P = exp2(t - m + log2 448) -> E4M3 -> shared memory (128B-swizzled K-major);
      // this half writes 16-byte chunks 4 hf .. 4 hf + 3 of its row
      float2 rs[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) rs[k] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int grp = 0; grp < 4; ++grp) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          const int c = grp * 16 + e;
          float2 u0, u1;
          const float2 y0 = make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1]));
          const float2 y1 = make_float2(__uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
          if (HAS_DS) {
            u0 = ffma2(y0, make_float2(ad, ad), make_float2(-mm, -mm));
            u1 = ffma2(y1, make_float2(ad, ad), make_float2(-mm, -mm));
          } else {
            u0 = ffma2(fadd2(y0, neg_magic), make_float2(a_h, a_h), make_float2(-mm, -mm));
            u1 = ffma2(fadd2(y1, neg_magic), make_float2(a_h, a_h), make_float2(-mm, -mm));
          }
          const float2 p0 = make_float2(ex2_approx(u0.x), ex2_approx(u0.y));
          const float2 p1 = make_float2(ex2_approx(u1.x), ex2_approx(u1.y));
          rs[e / 4] = fadd2(rs[e / 4], fadd2(p0, p1));
          w[e / 4] = cvt_e4m3x4(p0.x, p0.y, p1.x, p1.y);
        }
        *reinterpret_cast<uint4*>(myP + (((4 * hf + grp) ^ (row & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      const float2 rs2 = fadd2(fadd2(rs[0], rs[1]), fadd2(rs[2], rs[3]));
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.p_full[ti * 2 + (j & 1)]);
      l = fmaf(l, alpha, rs2.x + rs2.y);
      m = m_new;
      if constexpr (TWO_LEVEL) {
        // level 2 on this half of O_i: O = alpha O + O_t, where P V(j) put a fresh
        // O_t into S_i's columns [0, D).  O_t is read first, then S_i's columns of
        // this half get the magic fill back (this half's O_t columns and, for
        // D = 64, its share of the columns O_t does not cover) and the next QK^T
        // may run while the sum is formed.
        if (!(ok = mbar_wait_warp(&bar.ot_full[ti], j & 1))) break;
        tc_fence_after();
        const uint32_t tOt = tmem + 128 * ti + DH * hf + lane_off;
        uint32_t* ot = s;  // S is consumed: its registers take O_t
#pragma unroll
        for (int c = 0; c < DH; c += 32) tmem_ld32p(tOt + c, ot + c);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < DH; c += 8) tmem_fill8(tOt + c, kMagicBits);
        if (D < 128) {
#pragma unroll
          for (int c = 0; c < (128 - D) / 2; c += 8) tmem_fill8(tmem + 128 * ti + D + (128 - D) / 2 * hf + lane_off + c, kMagicBits);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.r_free[ti]);
#pragma unroll
        for (int c = 0; c < DH; c += 32) {
          if (j == 0) {
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = ot[c + e];
          } else {
            tmem_ld32(tO + c, x);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 o = ffma2(make_float2(__uint_as_float(x[e]), __uint_as_float(x[e + 1])),
                                     make_float2(alpha, alpha),
                                     make_float2(__uint_as_float(ot[c + e]), __uint_as_float(ot[c + e + 1])));
              x[e] = __float_as_uint(o.x);
              x[e + 1] = __float_as_uint(o.y);
            }
          }
          tmem_st32(tO + c, x);
        }
        tmem_st_wait();
      } else {
        // O_i accumulates in TMEM; before P V(i, j) adds tile j, this half's columns
        // of rows whose max grew are rescaled by alpha = e^(m_old - m_new) (a warp
        // whose 32 rows all have alpha == 1 leaves them untouched: exact).  P V(i, j - 1)
        // must have retired first, and is waited for even when nothing is rescaled:
        // o_ready(j + 1) then cannot complete before P V(i, j) was issued, so the
        // issuer's parity test of o_ready never sees it two phases ahead.  o_ready is
        // signalled for every j (P V(i, 0) waits for it too).
        if (j > 0) {
          if (!(ok = mbar_wait_warp(&bar.ot_full[ti], (j - 1) & 1))) break;
          tc_fence_after();
        }
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
          for (int c = 0; c < DH; c += 32) {
            tmem_ld32(tO + c, x);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 o = fmul2(make_float2(__uint_as_float(x[e]), __uint_as_float(x[e + 1])),
                                     make_float2(alpha, alpha));
              x[e] = __float_as_uint(o.x);
              x[e + 1] = __float_as_uint(o.y);
            }
            tmem_st32(tO + c, x);
          }
          tmem_st_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.o_ready[ti]);
      }
    }
    // ---- epilogue: out = O / l * delta_V on this half's columns (l carries the 448)
    if (nTi[ti] > 0) {
      float* lb = s_l + ti * 256;
      lb[hf * 128 + row] = l;
      __syncwarp();
      uint64_t* lxbar = bar.lx + ti * 4 + quarter;
      if (lane == 0) mbar_arrive(lxbar);
      if (ok) ok = mbar_wait_warp(lxbar, 0);
      l += lb[(1 - hf) * 128 + row];
      // TMEM accumulator: the last P V must have retired (two-level: this warp
      // already formed the final sum)
      if (ok && !TWO_LEVEL) ok = mbar_wait_warp(&bar.ot_full[ti], (nTi[ti] - 1) & 1);
      if (ok) {
        tc_fence_after();
        const float inv_l = 1.0f / l;
        if (LSE && hf == 0 && qrow < a.N) {
          // ln sum_j e^(S_ij) = (m + log2(l / 448)) ln 2 (m: running max of the
          // log2-domain scores, l: sum of 448 2^(t - m)), plus the smooth-K shift
          const int64_t bhq64 = (int64_t)(b * a.Hq + h);
          a.lse[bhq64 * a.N + qrow] =
              l > 0.0f ? (m + log2f(l) - kLog2_448) * 0.69314718055994531f + a.sm_scale * a.qkm[bhq64 * a.Np + qrow]
                       : -INFINITY;
        }
        const float* sv = a.s_v + (int64_t)(b * a.Hkv + g) * D + DH * hf;
        // row qrow of head (b, h): one formula for either layout (strides from the host)
        TO* out = reinterpret_cast<TO*>(a.o) + b * a.o_bs + h * a.o_hs + qrow * a.o_rs + DH * hf;
#pragma unroll
        for (int c = 0; c < DH; c += 32) {
          tmem_ld32(tO + c, x);
          tmem_ld_wait();
          if (qrow < a.N) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              float f[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) f[u] = __uint_as_float(x[e + u]) * inv_l * __ldg(sv + c + e + u);
              *reinterpret_cast<uint4*>(out + c + e) = make_uint4(pack2<TO>(f[0], f[1]), pack2<TO>(f[2], f[3]),
                                                                  pack2<TO>(f[4], f[5]), pack2<TO>(f[6], f[7]));
            }
          }
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

// Accumulator-precision probe of tcgen05.mma kind::f8f6f4 (M=128, N=128).
// Case r uses A row r and B row r, so D[r][r] = sum_k A[r][k] B[r][k]; the two
// MMAs read K bytes [0, 32) then [32, 64) (accumulating), so cases 5-7 test
// the carry of the FP32 accumulator across instructions.  Operands are E4M3:
//   0: [1, 2^-9].[1, 2^-9]            = 1 + 2^-18      (18 bits)
//   1: [1, 2^-8].[1, 2^-6]            = 1 + 2^-14
//   2: [1, 2^-6].[1, 2^-6]            = 1 + 2^-12
//   3: [256, 2^-9].[1, 2^-9]          = 256 + 2^-18    (below fp32 ulp: 256)
//   4: 32 x [1].[1]                   = 32
//   5: [64].[64]  then [2^-5].[2^-5]  = 4096 + 2^-10   (22 bits, across MMAs)
//   6: [1].[1]    then [2^-9].[2^-9]  = 1 + 2^-18      (across MMAs)
//   7: [1].[1]    then 32 x 2^-9.2^-9 = 1 + 2^-13      (across MMAs)
// out[r] = D[r][r] for r < 8.
__global__ void __launch_bounds__(128, 1) f8_accum_probe_kernel(float* out) {
  constexpr uint32_t kIdesc = make_idesc(/*F32*/ 1, /*E4M3*/ 0, /*E4M3*/ 0, 128, 128);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + 16384;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + 32768);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
  const int r = threadIdx.x, warp = r / 32, lane = r % 32;
  uint8_t a[64], bb[64];
#pragma unroll
  for (int k = 0; k < 64; ++k) { a[k] = 0; bb[k] = 0; }
  const uint8_t one = 0x38, m9 = 0x01, m8 = 0x02, m6 = 0x08, c64 = 0x68, m5 = 0x10, c256 = 0x78;
  switch (r) {
    case 0: a[0] = one; a[1] = m9; bb[0] = one; bb[1] = m9; break;
    case 1: a[0] = one; a[1] = m8; bb[0] = one; bb[1] = m6; break;
    case 2: a[0] = one; a[1] = m6; bb[0] = one; bb[1] = m6; break;
    case 3: a[0] = c256; a[1] = m9; bb[0] = one; bb[1] = m9; break;
    case 4: for (int k = 0; k < 32; ++k) { a[k] = one; bb[k] = one; } break;
    case 5: a[0] = c64; bb[0] = c64; a[32] = m5; bb[32] = m5; break;
    case 6: a[0] = one; bb[0] = one; a[32] = m9; bb[32] = m9; break;
    case 7: a[0] = one; bb[0] = one; for (int k = 32; k < 64; ++k) { a[k] = m9; bb[k] = m9; } break;
    default: break;
  }
  // row r of a 128-byte-swizzled K-major tile: 16-byte chunk c at (c ^ (r & 7))
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t wa[4] = {0, 0, 0, 0}, wb[4] = {0, 0, 0, 0};
    if (c < 4) {
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        wa[u / 4] |= (uint32_t)a[c * 16 + u] << (8 * (u % 4));
        wb[u / 4] |= (uint32_t)bb[c * 16 + u] << (8 * (u % 4));
      }
    }
    *reinterpret_cast<uint4*>(sA + r * 128 + ((c ^ (r & 7)) << 4)) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
    *reinterpret_cast<uint4*>(sB + r * 128 + ((c ^ (r & 7)) << 4)) = make_uint4(wb[0], wb[1], wb[2], wb[3]);
  }
  fence_proxy_async_smem();
  if (r == 0) {
    mbar_init(bar, 1);
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
  if (r == 0) {
    const uint32_t aA = smem_u32(sA), aB = smem_u32(sB);
    mma_f8f6f4(tmem, make_sdesc(aA, 1024, kSwizzle128B), make_sdesc(aB, 1024, kSwizzle128B), kIdesc, 0u);
    mma_f8f6f4(tmem, make_sdesc(aA + 32, 1024, kSwizzle128B), make_sdesc(aB + 32, 1024, kSwizzle128B), kIdesc, 1u);
    mma_commit(bar);
  }
  __syncwarp();
  if (mbar_wait_warp(bar, 0)) {
    tc_fence_after();
    uint32_t v[32];
    tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16), v);
    tmem_ld_wait();
    if (warp == 0 && lane < 8) {
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (u == lane) out[lane] = __uint_as_float(v[u]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// exp2_poly2 on an array (accuracy test of the FMA-pipe exponential).
__global__ void exp2_poly_probe_kernel(const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 r = exp2_poly2(make_float2(x[i], x[i + 1]));
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = exp2_poly2(make_float2(x[i], x[i])).x;
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

template <int D, bool CAUSAL, bool HAS_DS, bool TWO_LEVEL, typename TO>
cudaError_t launch_attn_t(const AttnArgs& a, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                          const CUtensorMap& tmO, cudaStream_t st) {
  // with delta_S the split-row kernel, else the one-warp-per-row kernel
  auto kern = HAS_DS ? (a.lse ? attn_i8f8_split_kernel<D, CAUSAL, true, TWO_LEVEL, TO, true>
                              : attn_i8f8_split_kernel<D, CAUSAL, true, TWO_LEVEL, TO, false>)
                     : (a.lse ? attn_i8f8_kernel<D, CAUSAL, false, TWO_LEVEL, TO, true>
                              : attn_i8f8_kernel<D, CAUSAL, false, TWO_LEVEL, TO, false>);
  const int smem = HAS_DS ? (int)SmemSplit<D>::kBytes : (int)Smem<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const unsigned n_pairs = (unsigned)(a.n_qtiles + 1) / 2;
  const unsigned grid = n_pairs * (unsigned)(a.B * a.Hq);
  kern<<<grid, HAS_DS ? kThreadsSplit : kThreadsAttn, smem, st>>>(tmQ, tmK, tmV, tmO, a);
  return cudaGetLastError();
}

template <int D, bool CAUSAL, bool TWO_LEVEL>
cudaError_t launch_attn_m(const AttnArgs& a, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                          const CUtensorMap& o, cudaStream_t st) {
  if (a.dS) {
    return a.out_fp16 ? launch_attn_t<D, CAUSAL, true, TWO_LEVEL, __half>(a, q, k, v, o, st)
                      : launch_attn_t<D, CAUSAL, true, TWO_LEVEL, __nv_bfloat16>(a, q, k, v, o, st);
  }
  return a.out_fp16 ? launch_attn_t<D, CAUSAL, false, TWO_LEVEL, __half>(a, q, k, v, o, st)
                    : launch_attn_t<D, CAUSAL, false, TWO_LEVEL, __nv_bfloat16>(a, q, k, v, o, st);
}

template <int D, bool CAUSAL>
cudaError_t launch_attn_d(const AttnArgs& a, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                          const CUtensorMap& o, cudaStream_t st) {
  return a.two_level ? launch_attn_m<D, CAUSAL, true>(a, q, k, v, o, st)
                     : launch_attn_m<D, CAUSAL, false>(a, q, k, v, o, st);
}

}  // namespace

cudaError_t launch_attn_i8f8(const AttnArgs& a, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                             const CUtensorMap& tmV, const CUtensorMap& tmO, cudaStream_t st) {
  if (a.D == 128)
    return a.causal ? launch_attn_d<128, true>(a, tmQ, tmK, tmV, tmO, st)
                    : launch_attn_d<128, false>(a, tmQ, tmK, tmV, tmO, st);
  return a.causal ? launch_attn_d<64, true>(a, tmQ, tmK, tmV, tmO, st)
                  : launch_attn_d<64, false>(a, tmQ, tmK, tmV, tmO, st);
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

cudaError_t launch_f8_accum_probe(float* out, cudaStream_t st) {
  const int smem = 32768 + 64 + 1024;
  cudaError_t e = cudaFuncSetAttribute(f8_accum_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  f8_accum_probe_kernel<<<1, 128, smem, st>>>(out);
  return cudaGetLastError();
}

cudaError_t launch_exp2_poly_probe(const float* x, float* y, int n, cudaStream_t st) {
  const int pairs = (n + 1) / 2;
  exp2_poly_probe_kernel<<<(pairs + 255) / 256, 256, 0, st>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_bounded_wait_probe(cudaStream_t st) {
  bounded_wait_probe_kernel<<<1, 32, 0, st>>>();
  return cudaGetLastError();
}

}  // namespace sage
