// attn_nvfp4.cu -- fused NVFP4 attention forward on sm_100a (SageAttention3
// style): block-scaled FP4 Q K^T and FP4 P V on tcgen05 (kind::mxf4nvf4,
// one UE4M3 scale per 16 elements), accumulators in TMEM.
//
// Method (SageAttention3 reading note, zhaifeiyue.github.io/papers/2505.11594,
// "Microscaling FP4 attention" and the two-level quantisation of P), per
// 128-row Q tile and 128-key tile j, scores in base 2 (t = S sm_scale log2 e):
//   S     = (Q^ sq)(K^ sk)^T + delta_S                  FP4 MMA, f32 in TMEM
//   m_t   = rowmax_j t,  m = max(m_old, m_t)
//   P~    = exp2(t - m),  l = exp2(m_old - m) l + rowsum P~
//   s_P1  = rowmax P~ / 2688 = exp2(m_t - m) / 2688      per row, per tile
//   P2    = P~ / s_P1 = 2688 exp2(t - m_t)               in [0, 2688]
//   s_P2  = E4M3(amax16(P2) / 6),  P^ = E2M1(P2 / s_P2)  per 16 keys
//   O     = exp2(m_old - m) O + s_P1 (P^ s_P2)(V^ sv)    FP4 MMA
//   out   = O / l
// P2 is computed directly as exp2(t - m_t + log2 2688), so no division by
// s_P1 is needed, and rowsum P~ = s_P1 rowsum P2.
//
// Accumulation.  O_i lives in one FP32 TMEM accumulator per Q tile that holds
// A = 2688 exp2(-E) U, U = sum over keys of exp2(t) v (absolute scale), where E
// is the tile max m_t of the last tile added.  Adding tile j multiplies A by
// r = exp2(E_old - m_t) on CUDA cores and lets the MMA add P^ V^ (the block
// scales s_P2 and sv ride in the MMA).  Then out = A exp2(E - m) / (2688 l).
// This equals the SageAttention2 two-level form (fresh O_t, then
// O = alpha O + s_P1 O_t) in exact arithmetic.  A tile whose row max lies more
// than 2^32 below the running max would need r > 2^32; its 128 values of P~ sum
// to less than 2^-25 of l (l >= 1), under half an fp32 ulp, so that row of the
// tile is dropped (P^ = 0, r = 1, l unchanged).  This keeps
// |A| <= 2^32 * 2688 * N * 2688 (|V^ sv| <= 6 * 448).
//
// CTA = one (batch, head) and two consecutive 128-row Q tiles sharing every
// K / V tile; 512 threads: warp 0 TMA producer, warp 1 MMA issuer and TMEM
// owner, WG1 / WG2 softmax of tile 0 / 1 (thread = row = TMEM lane), WG3
// rescale of A and the epilogue.  TMEM (512 columns): S [0,128) shared by the
// two tiles (their Q K^T alternate; a softmax releases S as soon as it has it
// in registers), A_i [128 + 128 i, +128), block scales from column 384.
// Head dim 128 only.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace sage {

namespace {

constexpr int kStF4 = 3;  // K / V ring stages
constexpr int kThreadsF4 = 512;
constexpr float kLog2_2688 = 11.392317422778762f;  // log2(448 * 6)
constexpr float kDropLog2 = 32.0f;                 // drop a tile row whose max is 2^32 below m

// TMEM columns
constexpr uint32_t kColS = 0, kColA = 128;
__host__ __device__ constexpr uint32_t col_sfq(int i, int kk) { return 384 + 8 * i + 4 * kk; }
__host__ __device__ constexpr uint32_t col_sfk(int s, int kk) { return 400 + 8 * s + 4 * kk; }
__host__ __device__ constexpr uint32_t col_sfp(int i, int kk) { return 400 + 8 * kStF4 + 8 * i + 4 * kk; }
__host__ __device__ constexpr uint32_t col_sfv(int s, int kk) { return 416 + 8 * kStF4 + 8 * s + 4 * kk; }
static_assert(col_sfv(kStF4 - 1, 1) + 4 <= 512, "TMEM columns");

constexpr uint32_t kRegsF4Producer = 56, kRegsF4Softmax = 184, kRegsF4Correction = 88;
static_assert(kRegsF4Producer + 2 * kRegsF4Softmax + kRegsF4Correction <= 512, "register split exceeds the launch");

struct SmemF4 {
  static constexpr uint32_t kT = 128 * 64;  // one 128 x 128 FP4 tile (64-byte rows)
  static constexpr uint32_t kSF = 1024;     // its scale block
  static constexpr uint32_t oQ = 0;
  static constexpr uint32_t oK = oQ + 2 * kT;
  static constexpr uint32_t oV = oK + kStF4 * kT;
  static constexpr uint32_t oP = oV + kStF4 * kT;
  static constexpr uint32_t oSFQ = oP + 4 * kT;  // P: [tile][2 buffers]
  static constexpr uint32_t oSFK = oSFQ + 2 * kSF;
  static constexpr uint32_t oSFV = oSFK + kStF4 * kSF;
  static constexpr uint32_t oSFP = oSFV + kStF4 * kSF;
  static constexpr uint32_t kDS = 2 * 2 * 128 * 4;  // delta_S rows of one key tile: [tile][Q block][128]
  static constexpr uint32_t oDS = oSFP + 4 * kSF;   // kStF4
  static constexpr uint32_t oR = oDS + kStF4 * kDS;  // float[tile][buffer][128] rescale factor r
  static constexpr uint32_t oL = oR + 4 * 128 * 4;  // float[2][128] final 1 / (2688 l exp2(m - E))
  static constexpr uint32_t oBar = oL + 2 * 128 * 4;
  static constexpr uint32_t kNumBars = 1 + 3 * kStF4 + 1 + 2 + 4 + 4 + 2 + 2 + 2 + 1;
  static constexpr uint32_t oTmem = oBar + 8 * kNumBars;
  static constexpr uint32_t kBytes = oTmem + 16 + 1024;
};

struct BarsF4 {
  uint64_t* q_full;
  uint64_t* k_full;    // [kStF4] K codes + scales landed
  uint64_t* v_full;    // [kStF4] V^T codes + scales landed
  uint64_t* kv_empty;  // [kStF4]
  uint64_t* s_free;    // S columns read by the softmax that owned them (128 arrivals)
  uint64_t* s_full;    // [2] Q K^T of tile i in S
  uint64_t* p_full;    // [tile][buffer j & 1] P^_i(j), its scales and r_i(j) written (128 arrivals)
  uint64_t* p_empty;   // [tile][buffer] the P V that read that buffer retired
  uint64_t* ot_full;   // [2] P V of tile i retired
  uint64_t* o_ready;   // [2] A_i rescaled for the next P V (128 arrivals)
  uint64_t* l_ready;   // [2] final normaliser of tile i in shared memory (128 arrivals)
  uint64_t* mma_done;
};

template <typename TO>
__device__ __forceinline__ uint32_t pack2f4(float a, float b);
template <>
__device__ __forceinline__ uint32_t pack2f4<__nv_bfloat16>(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <>
__device__ __forceinline__ uint32_t pack2f4<__half>(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) { return make_sdesc(saddr, 128, kSwizzleNone); }

// NHD: o is [B, N, Hq, 128] (else [B, Hq, N, 128]); a template choice, so that
// the register-tight epilogue computes one fixed address formula
template <bool CAUSAL, bool HAS_DS, typename TO, bool NHD>
__global__ void __launch_bounds__(kThreadsF4, 1)
    attn_nvfp4_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
  using L = SmemF4;
  constexpr uint32_t kIdesc = make_idesc_nvf4(128, 128);
  constexpr uint32_t kTmemCols = 512;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::oQ;
  uint8_t* sK = smem + L::oK;
  uint8_t* sV = smem + L::oV;
  uint8_t* sP = smem + L::oP;
  uint8_t* sSFQ = smem + L::oSFQ;
  uint8_t* sSFK = smem + L::oSFK;
  uint8_t* sSFV = smem + L::oSFV;
  uint8_t* sSFP = smem + L::oSFP;
  float* s_r = reinterpret_cast<float*>(smem + L::oR);
  float* s_l = reinterpret_cast<float*>(smem + L::oL);
  uint64_t* bar0 = reinterpret_cast<uint64_t*>(smem + L::oBar);
  BarsF4 bar;
  bar.q_full = bar0;
  bar.k_full = bar0 + 1;
  bar.v_full = bar.k_full + kStF4;
  bar.kv_empty = bar.v_full + kStF4;
  bar.s_free = bar.kv_empty + kStF4;
  bar.s_full = bar.s_free + 1;
  bar.p_full = bar.s_full + 2;
  bar.p_empty = bar.p_full + 4;
  bar.ot_full = bar.p_empty + 4;
  bar.o_ready = bar.ot_full + 2;
  bar.l_ready = bar.o_ready + 2;
  bar.mma_done = bar.l_ready + 2;
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
  const int bg = b * a.Hkv + g;
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
    for (int s = 0; s < kStF4; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.kv_empty[s], 1);
    }
    mbar_init(bar.s_free, 128);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar.s_full[i], 1);
      mbar_init(&bar.p_full[2 * i], 128);
      mbar_init(&bar.p_full[2 * i + 1], 128);
      mbar_init(&bar.p_empty[2 * i], 1);
      mbar_init(&bar.p_empty[2 * i + 1], 1);
      mbar_init(&bar.ot_full[i], 1);
      mbar_init(&bar.o_ready[i], 128);
      mbar_init(&bar.l_ready[i], 128);
    }
    mbar_init(bar.mma_done, 1);
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
  const int64_t tiles_per_head = a.Np / kTile;

  if (wg == 0) {
    regs_dec<kRegsF4Producer>();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------ TMA producer
      tma_prefetch_map(&tmQ);
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      const int64_t qhead = (int64_t)bh * a.Np;
      const int krow0 = (int)((int64_t)bg * a.Np);
      const int vrow = bg * 128;
      const int ds_rows = kTile / a.bq;  // Q blocks per tile (1 or 2)
      const uint32_t ds_bytes = (uint32_t)((nTi[0] > 0) + (nTi[1] > 0)) * ds_rows * 512;
      mbar_expect_tx(bar.q_full, (nTi[0] > 0 ? L::kT + L::kSF : 0u) + (nTi[1] > 0 ? L::kT + L::kSF : 0u));
      for (int i = 0; i < 2; ++i)
        if (nTi[i] > 0) {
          const int qt = 2 * pr + i;
          tma_load_2d(sQ + i * L::kT, &tmQ, bar.q_full, 0, (int)(qhead + (int64_t)qt * kTile));
          bulk_load_1d(sSFQ + i * L::kSF, a.sfq + ((int64_t)bh * tiles_per_head + qt) * 1024, L::kSF, bar.q_full);
        }
      bool ok = true;
      int j = 0;
      for (; j < nT && ok; ++j) {
        const int s = j % kStF4;
        if (j >= kStF4) ok = mbar_wait(&bar.kv_empty[s], ((j / kStF4) + 1) & 1);
        if (!ok) break;
        const int64_t kvt = (int64_t)bg * tiles_per_head + j;
        mbar_expect_tx(&bar.k_full[s], L::kT + L::kSF + (HAS_DS ? ds_bytes : 0u));
        tma_load_2d(sK + s * L::kT, &tmK, &bar.k_full[s], 0, krow0 + j * kTile);
        bulk_load_1d(sSFK + s * L::kSF, a.sfk + kvt * 1024, L::kSF, &bar.k_full[s]);
        if (HAS_DS) {
          // delta_S[b, h, Q block, keys of tile j] for the Q blocks of both tiles
          for (int i = 0; i < 2; ++i)
            for (int hb = 0; hb < ds_rows; ++hb)
              if (nTi[i] > 0) {
                const int blk = min((2 * pr + i) * ds_rows + hb, a.Tm - 1);
                bulk_load_1d(smem + L::oDS + s * L::kDS + (i * 2 + hb) * 512,
                             a.dS + ((int64_t)bh * a.Tm + blk) * a.Np + (int64_t)j * kTile, 512, &bar.k_full[s]);
              }
        }
        mbar_expect_tx(&bar.v_full[s], L::kT + L::kSF);
        tma_load_2d(sV + s * L::kT, &tmV, &bar.v_full[s], j * (kTile / 2), vrow);
        bulk_load_1d(sSFV + s * L::kSF, a.sfv + kvt * 1024, L::kSF, &bar.v_full[s]);
      }
      // never leave a copy in flight
      for (int jj = (j - kStF4 > 0 ? j - kStF4 : 0); jj < j; ++jj) {
        mbar_wait(&bar.k_full[jj % kStF4], (jj / kStF4) & 1);
        mbar_wait(&bar.v_full[jj % kStF4], (jj / kStF4) & 1);
      }
      mbar_wait(bar.q_full, 0);
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        bool ok = mbar_wait(bar.q_full, 0);
        if (ok) {
          for (int i = 0; i < 2; ++i)
            if (nTi[i] > 0)
              for (int kk = 0; kk < 2; ++kk) tmem_cp_sf(tmem + col_sfq(i, kk), sf_desc(smem_u32(sSFQ + i * L::kSF + kk * 512)));
        }
        // Q K^T of the two tiles alternate through the one S region:
        // (j=0,i=0), (0,1), (1,0), (1,1), ... skipping inactive tiles.  The n-th
        // needs the (n-1)-th consumed (s_free phase n-1).
        int qk_j = 0, qk_i = 0, n_qk = 0;
        auto qk_advance = [&]() {
          do {
            if (qk_i == 0) {
              qk_i = 1;
            } else {
              qk_i = 0;
              ++qk_j;
            }
          } while (qk_j < nT && qk_j >= nTi[qk_i]);
        };
        if (nTi[0] == 0) qk_i = 1;
        int issued_qk[2] = {0, 0}, next_pv[2] = {0, 0};
        int sfk_next = 0, sfv_next = 0, released = 0;
        uint64_t t_idle = 0;
        while (ok) {
          bool progress = false;
          // ---- next Q K^T
          if (qk_j < nT) {
            const int s = qk_j % kStF4;
            if (mbar_test_wait(smem_u32(&bar.k_full[s]), (qk_j / kStF4) & 1) &&
                (n_qk == 0 || mbar_test_wait(smem_u32(bar.s_free), (n_qk - 1) & 1))) {
              tc_fence_after();
              if (qk_j >= sfk_next) {
                for (int kk = 0; kk < 2; ++kk)
                  tmem_cp_sf(tmem + col_sfk(s, kk), sf_desc(smem_u32(sSFK + s * L::kSF + kk * 512)));
                sfk_next = qk_j + 1;
              }
              const uint32_t aQ = smem_u32(sQ + qk_i * L::kT), aK = smem_u32(sK + s * L::kT);
#pragma unroll
              for (int kk = 0; kk < 2; ++kk)
                mma_nvf4(tmem + kColS, make_sdesc(aQ + kk * 32, 512, kSwizzle64B),
                         make_sdesc(aK + kk * 32, 512, kSwizzle64B), kIdesc, tmem + col_sfq(qk_i, kk),
                         tmem + col_sfk(s, kk), kk > 0 ? 1u : 0u);
              mma_commit(&bar.s_full[qk_i]);
              ++issued_qk[qk_i];
              ++n_qk;
              qk_advance();
              progress = true;
            }
          }
          // ---- P V of either tile
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int jp = next_pv[i];
            const int s = jp % kStF4;
            if (jp < nTi[i] && issued_qk[i] > jp &&
                mbar_test_wait(smem_u32(&bar.p_full[i * 2 + (jp & 1)]), (jp >> 1) & 1) &&
                mbar_test_wait(smem_u32(&bar.v_full[s]), (jp / kStF4) & 1) &&
                (jp == 0 || mbar_test_wait(smem_u32(&bar.o_ready[i]), (jp - 1) & 1))) {
              tc_fence_after();
              if (jp >= sfv_next) {
                for (int kk = 0; kk < 2; ++kk)
                  tmem_cp_sf(tmem + col_sfv(s, kk), sf_desc(smem_u32(sSFV + s * L::kSF + kk * 512)));
                sfv_next = jp + 1;
              }
              for (int kk = 0; kk < 2; ++kk)
                tmem_cp_sf(tmem + col_sfp(i, kk), sf_desc(smem_u32(sSFP + (i * 2 + (jp & 1)) * L::kSF + kk * 512)));
              const uint32_t aP = smem_u32(sP + (i * 2 + (jp & 1)) * L::kT), aV = smem_u32(sV + s * L::kT);
#pragma unroll
              for (int kk = 0; kk < 2; ++kk)
                mma_nvf4(tmem + kColA + 128 * i, make_sdesc(aP + kk * 32, 512, kSwizzle64B),
                         make_sdesc(aV + kk * 32, 512, kSwizzle64B), kIdesc, tmem + col_sfp(i, kk),
                         tmem + col_sfv(s, kk), (jp > 0 || kk > 0) ? 1u : 0u);
              mma_commit(&bar.ot_full[i]);
              mma_commit(&bar.p_empty[i * 2 + (jp & 1)]);
              next_pv[i] = jp + 1;
              progress = true;
            }
          }
          while (released < nT && (next_pv[0] > released || released >= nTi[0]) &&
                 (next_pv[1] > released || released >= nTi[1])) {
            mma_commit(&bar.kv_empty[released % kStF4]);
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
        mma_commit(bar.mma_done);
        mbar_wait(bar.mma_done, 0);
      }
      __syncwarp();
    }
  } else if (wg == 1 || wg == 2) {
    // ------------------------------------------------------------ softmax + P quantisation
    regs_inc<kRegsF4Softmax>();
    const int ti = wg - 1;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int qtile = 2 * pr + ti;
    const int64_t qrow = (int64_t)qtile * kTile + row;
    const uint32_t tS = tmem + kColS + ((uint32_t)(quarter * 32) << 16);
    const int ds_half = (a.bq == 64 && row >= 64) ? 1 : 0;  // warp-uniform
    const float* sDS = reinterpret_cast<const float*>(smem + L::oDS);
    uint8_t* myP0 = sP + ti * 2 * L::kT + row * 64;  // buffer b at + b * kT
    uint32_t* mySF0 = reinterpret_cast<uint32_t*>(sSFP + ti * 2 * L::kSF) + 4 * lane + quarter;
    const float sl2 = a.scale_log2;
    float m = -INFINITY, l = 0.0f, E = 0.0f;
    bool ok = true;
    for (int j = 0; j < nTi[ti] && ok; ++j) {
      if (!(ok = mbar_wait_warp(&bar.s_full[ti], j & 1))) break;
      tc_fence_after();
      uint32_t s[128];
      tmem_ld32p(tS + 0, s + 0);
      tmem_ld32p(tS + 32, s + 32);
      tmem_ld32p(tS + 64, s + 64);
      tmem_ld32p(tS + 96, s + 96);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bar.s_free);
      const int col0 = j * kTile;
      // x = S + delta_S (the scores are t = x sm_scale log2 e; the scale is
      // applied to the max and inside the exponent's FMA)
      if (HAS_DS) {
        const float* dsr = sDS + (j % kStF4) * (L::kDS / 4) + (ti * 2 + ds_half) * 128;
        if (!(ok = mbar_wait_warp(&bar.k_full[j % kStF4], (j / kStF4) & 1))) break;
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          const float2 x = fadd2(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                                 *reinterpret_cast<const float2*>(dsr + c));
          s[c] = __float_as_uint(x.x);
          s[c + 1] = __float_as_uint(x.y);
        }
      }
      const bool need_mask = (col0 + kTile > a.N) || (CAUSAL && j == qtile);
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const int col = col0 + c;
          if (col >= a.N || (CAUSAL && col > qrow)) s[c] = __float_as_uint(-INFINITY);
        }
      }
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; c += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mx8[k] = fmax3(mx8[k], __uint_as_float(s[c + 2 * k]), __uint_as_float(s[c + 2 * k + 1]));
      const float mt = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])) * sl2;
      const float m_new = fmaxf(m, mt);
      const float alpha = (m == -INFINITY) ? 0.0f : ex2_approx(m - m_new);
      const bool keep = mt >= m_new - kDropLog2;  // false only for a row far below the running max
      // P buffer (j & 1) and its scales are free once P V(j - 2) retired
      if (j >= 2 && !(ok = mbar_wait_warp(&bar.p_empty[ti * 2 + (j & 1)], ((j >> 1) - 1) & 1))) break;
      uint8_t* myP = myP0 + (j & 1) * L::kT;
      uint32_t* mySF = mySF0 + (j & 1) * (L::kSF / 4);
      const float mm = keep ? mt - kLog2_2688 : INFINITY;  // P2 = exp2(t - mm); dropped rows give 0
      float2 rs[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) rs[k] = make_float2(0.0f, 0.0f);
      uint32_t sfw0 = 0, sfw1 = 0;
#pragma unroll
      for (int pair = 0; pair < 4; ++pair) {
        uint32_t w[4];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int c0 = pair * 32 + half * 16;
          float p[16];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const float2 u = ffma2(make_float2(__uint_as_float(s[c0 + e]), __uint_as_float(s[c0 + e + 1])),
                                   make_float2(sl2, sl2), make_float2(-mm, -mm));
            p[e] = ex2_approx(u.x);
            p[e + 1] = ex2_approx(u.y);
            rs[e / 4] = fadd2(rs[e / 4], make_float2(p[e], p[e + 1]));
          }
          const float gm = fmax3(fmax3(fmax3(p[0], p[1], p[2]), fmax3(p[3], p[4], p[5]), fmax3(p[6], p[7], p[8])),
                                 fmax3(p[9], p[10], p[11]), fmax3(p[12], p[13], fmaxf(p[14], p[15])));
          // s_P2 = E4M3(amax16 / 6) and 1 / s_P2 without IEEE division steps (a
          // code can differ from the divided one only at an exact midpoint)
          const uint32_t sc = cvt_e4m3(gm * (1.0f / 6.0f));
          const float sd = e4m3_value(sc);
          const float inv = sd > 0.0f ? rcp_approx(sd) : 0.0f;
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const float2 q = fmul2(make_float2(p[e], p[e + 1]), make_float2(inv, inv));
            p[e] = q.x;
            p[e + 1] = q.y;
          }
          w[half * 2 + 0] = cvt_e2m1x8(p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7]);
          w[half * 2 + 1] = cvt_e2m1x8(p[8], p[9], p[10], p[11], p[12], p[13], p[14], p[15]);
          const int grp = pair * 2 + half;
          if (grp < 4)
            sfw0 |= sc << (8 * grp);
          else
            sfw1 |= sc << (8 * (grp - 4));
        }
        // 64-byte rows, 64-byte swizzle: 16-byte chunk c of row r at c ^ ((r >> 1) & 3)
        *reinterpret_cast<uint4*>(myP + ((pair ^ ((row >> 1) & 3)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      mySF[0] = sfw0;        // scale block kk = 0: byte 16 (row % 32) + 4 (row / 32) + k
      mySF[128] = sfw1;      // kk = 1 (+512 bytes)
      const float2 rs2 = fadd2(fadd2(rs[0], rs[1]), fadd2(rs[2], rs[3]));
      float r = 1.0f;
      if (keep) {
        // rowsum P~ = s_P1 rowsum P2 with s_P1 = exp2(m_t - m) / 2688
        l = fmaf(l, alpha, ex2_approx(mt - m_new - kLog2_2688) * (rs2.x + rs2.y));
        r = (j == 0) ? 1.0f : ex2_approx(E - mt);
        E = mt;
      }  // a dropped row leaves l as it is (alpha == 1 there; its share is < 2^-25 of l)
      s_r[(ti * 2 + (j & 1)) * 128 + row] = r;
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(&bar.p_full[ti * 2 + (j & 1)]);
      m = m_new;
    }
    // out = A exp2(E - m) / (2688 l)
    s_l[ti * 128 + row] = ex2_approx(E - m - kLog2_2688) / l;
    mbar_arrive(&bar.l_ready[ti]);
  } else {
    // ------------------------------------------------------------ rescale of A + epilogue
    regs_dec<kRegsF4Correction>();
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    uint32_t x[32];
    // (every phase of p_full is waited in order, j = 0 included)
    for (int j = 0; j < nT && ok; ++j) {
      for (int i = 0; i < 2; ++i) {
        if (j >= nTi[i]) continue;
        if (!(ok = mbar_wait_warp(&bar.p_full[i * 2 + (j & 1)], (j >> 1) & 1))) break;
        if (j == 0) continue;
        if (!(ok = mbar_wait_warp(&bar.ot_full[i], (j - 1) & 1))) break;
        tc_fence_after();
        const float r = s_r[(i * 2 + (j & 1)) * 128 + row];
        if (__any_sync(0xffffffffu, r != 1.0f)) {
          const uint32_t tA = tmem + kColA + 128 * i + lane_off;
#pragma unroll
          for (int c = 0; c < 128; c += 32) {
            tmem_ld32(tA + c, x);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 o = fmul2(make_float2(__uint_as_float(x[e]), __uint_as_float(x[e + 1])), make_float2(r, r));
              x[e] = __float_as_uint(o.x);
              x[e + 1] = __float_as_uint(o.y);
            }
            tmem_st32(tA + c, x);
          }
          tmem_st_wait();
        }
        tc_fence_before();
        mbar_arrive(&bar.o_ready[i]);
      }
    }
    for (int i = 0; i < 2 && ok; ++i) {
      if (nTi[i] == 0) continue;
      if (!(ok = mbar_wait_warp(&bar.l_ready[i], 0))) break;
      if (!(ok = mbar_wait_warp(&bar.ot_full[i], (nTi[i] - 1) & 1))) break;
      tc_fence_after();
      const float f = s_l[i * 128 + row];
      const int64_t qrow = (int64_t)(2 * pr + i) * kTile + row;
      TO* out = reinterpret_cast<TO*>(a.o) + (NHD ? ((int64_t)b * a.N + qrow) * a.Hq + h : (int64_t)bh * a.N + qrow) * 128;
      const uint32_t tA = tmem + kColA + 128 * i + lane_off;
#pragma unroll
      for (int c = 0; c < 128; c += 32) {
        tmem_ld32(tA + c, x);
        tmem_ld_wait();
        if (qrow < a.N) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = __uint_as_float(x[e + u]) * f;
            *reinterpret_cast<uint4*>(out + c + e) = make_uint4(pack2f4<TO>(v[0], v[1]), pack2f4<TO>(v[2], v[3]),
                                                                pack2f4<TO>(v[4], v[5]), pack2f4<TO>(v[6], v[7]));
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
// Probe: one FP32 tile (Q^ sq)(K^ sk)^T of rows [128 qtile, +128) of head
// (b, h) and keys [128 ktile, +128) through the same TMA staging, scale-block
// copies and block-scaled MMA as the attention kernel; out row-major 128x128.
__global__ void __launch_bounds__(128, 1)
    qk_probe_nvfp4_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const AttnArgs a, float* out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sQ = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = sQ + SmemF4::kT;
  uint8_t* sSFQ = sK + SmemF4::kT;
  uint8_t* sSFK = sSFQ + 1024;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSFK + 1024);
  uint32_t& tmem_slot = *reinterpret_cast<uint32_t*>(bars + 2);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = a.probe_b * a.Hq + a.probe_h;
  const int bg = a.probe_b * a.Hkv + a.probe_h / (a.Hq / a.Hkv);
  const int64_t tph = a.Np / kTile;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  bool ok = true;
  if (threadIdx.x == 0) {
    mbar_expect_tx(&bars[0], 2 * SmemF4::kT + 2048);
    tma_load_2d(sQ, &tmQ, &bars[0], 0, (int)((int64_t)bh * a.Np + (int64_t)a.probe_qtile * kTile));
    tma_load_2d(sK, &tmK, &bars[0], 0, (int)((int64_t)bg * a.Np + (int64_t)a.probe_ktile * kTile));
    bulk_load_1d(sSFQ, a.sfq + ((int64_t)bh * tph + a.probe_qtile) * 1024, 1024, &bars[0]);
    bulk_load_1d(sSFK, a.sfk + ((int64_t)bg * tph + a.probe_ktile) * 1024, 1024, &bars[0]);
    ok = mbar_wait(&bars[0], 0);
    if (ok) {
      tc_fence_after();
      for (int kk = 0; kk < 2; ++kk) {
        tmem_cp_sf(tmem + 128 + 4 * kk, sf_desc(smem_u32(sSFQ + kk * 512)));
        tmem_cp_sf(tmem + 136 + 4 * kk, sf_desc(smem_u32(sSFK + kk * 512)));
      }
      for (int kk = 0; kk < 2; ++kk)
        mma_nvf4(tmem, make_sdesc(smem_u32(sQ) + kk * 32, 512, kSwizzle64B),
                 make_sdesc(smem_u32(sK) + kk * 32, 512, kSwizzle64B), make_idesc_nvf4(128, 128),
                 tmem + 128 + 4 * kk, tmem + 136 + 4 * kk, kk > 0 ? 1u : 0u);
      mma_commit(&bars[1]);
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  ok = __syncthreads_and(ok);
  if (ok) ok = mbar_wait_warp(&bars[1], 0);
  if (ok) {
    tc_fence_after();
    uint32_t x[32];
    const uint32_t base = tmem + ((uint32_t)(warp * 32) << 16);
    for (int c = 0; c < 128; c += 32) {
      tmem_ld32(base + c, x);
      tmem_ld_wait();
      for (int e = 0; e < 32; ++e) out[(warp * 32 + lane) * 128 + c + e] = __uint_as_float(x[e]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <bool CAUSAL, bool HAS_DS, typename TO>
cudaError_t launch_nvfp4_t(const AttnArgs& a, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                           cudaStream_t st) {
  auto k = a.nhd ? attn_nvfp4_kernel<CAUSAL, HAS_DS, TO, true> : attn_nvfp4_kernel<CAUSAL, HAS_DS, TO, false>;
  const int smem = (int)SmemF4::kBytes;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int n_pairs = (a.n_qtiles + 1) / 2;
  k<<<dim3(n_pairs * a.B * a.Hq), kThreadsF4, smem, st>>>(tmQ, tmK, tmV, a);
  return cudaGetLastError();
}

template <bool CAUSAL, bool HAS_DS>
cudaError_t launch_nvfp4_o(const AttnArgs& a, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                           cudaStream_t st) {
  return a.out_fp16 ? launch_nvfp4_t<CAUSAL, HAS_DS, __half>(a, q, k, v, st)
                    : launch_nvfp4_t<CAUSAL, HAS_DS, __nv_bfloat16>(a, q, k, v, st);
}

template <bool CAUSAL>
cudaError_t launch_nvfp4_d(const AttnArgs& a, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                           cudaStream_t st) {
  return a.dS ? launch_nvfp4_o<CAUSAL, true>(a, q, k, v, st) : launch_nvfp4_o<CAUSAL, false>(a, q, k, v, st);
}

}  // namespace

cudaError_t launch_attn_nvfp4(const AttnArgs& a, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                              const CUtensorMap& tmV, cudaStream_t st) {
  if (a.D != 128) return cudaErrorInvalidValue;
  return a.causal ? launch_nvfp4_d<true>(a, tmQ, tmK, tmV, st) : launch_nvfp4_d<false>(a, tmQ, tmK, tmV, st);
}

cudaError_t launch_qk_probe_nvfp4(const AttnArgs& a, const CUtensorMap& tmQ, const CUtensorMap& tmK, float* out,
                                  cudaStream_t st) {
  constexpr int kProbeSmem = 2 * SmemF4::kT + 2048 + 32 + 1024;
  qk_probe_nvfp4_kernel<<<1, 128, kProbeSmem, st>>>(tmQ, tmK, a, out);
  return cudaGetLastError();
}

}  // namespace sage
