// quant.cu -- SageAttention preprocessing on sm_100a (HBM-bound kernels).
//
// Follows the "Preprocessing" part of Algorithm 1 in the SageAttention2 note
// (zhaifeiyue.github.io/papers/2411.10958/detail) and Figure 3 stages 1-3:
//   smooth K:  km = mean_n K,  gamma(K) = K - km               (exact shift)
//   smooth Q:  qbar_i = mean of Q block i,  Q_i - qbar_i
//   psi_Q/psi_K: per-block INT8, scale = amax / 127, code = rint(x / scale)
//   psi_V:     per-channel FP8 E4M3, scale = amax / 448
//   GEMV:      delta_S[i, j] = qbar_i . gamma(K_j)   (tcgen05 TF32, 3-term split)
// Bit-exactness with the plain definitions: column sums are accumulated in
// fp64 (the partial sums of bf16/fp16 inputs are exact -- 53 bits hold a sum
// of up to 2^15 tokens whose magnitudes in one column lie within about 2^30
// of each other, which attention inputs do -- so the order does not matter),
// divided in fp64 and rounded once to fp32; every division of
// the quantisers is an IEEE fp32 division (__fdiv_rn) -- per element it is
// replaced by a multiplication with the reciprocal wherever that provably
// gives the same code (quant8_i8 / quant_e4m3x2 below) -- and the INT8 rounding
// is round-half-to-even.  Do not build with fast-math.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "common.cuh"
#include "sm100.cuh"

namespace sage {

namespace {

constexpr int kThreads = 256;
constexpr int kStatRows = 256;  // tokens per CTA in the K/V statistics pass

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&x)[8]);

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&x)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void load8<__half>(const __half* p, float (&x)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
    const float2 f = __half22float2(h);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_float(__half x) { return __half2float(x); }

// rows of a [r0, r0 + rows) block that lie below N
__device__ __forceinline__ int rows_valid(int N, int64_t r0, int rows) {
  const int64_t v = (int64_t)N - r0;
  return v <= 0 ? 0 : (v < rows ? (int)v : rows);
}

// Codes of a quotient x / s without a division per element.  With r = RN(1/s),
// y = RN(x r) is within 1.5 ulp of RN(x / s) (the quotient the definition
// rounds).  Every code conversion is monotonic, so when y (1 - 2^-21) and
// y (1 + 2^-21) -- a bracket of at least +-3.5 ulp around y -- get the same code,
// RN(x / s) gets it too; otherwise (within ~4 ulp of a rounding boundary, about
// one value in 10^5) the exact quotient __fdiv_rn(x, s) decides.  Subnormal y
// only arise for codes that are 0 either way.
constexpr float kBracketLo = 1.0f - 0x1p-21f, kBracketHi = 1.0f + 0x1p-21f;

// Eight INT8 codes rint(RN(x[e] / s)) packed little-endian.  |RN(x / s)| <= 127
// holds by construction (s = RN(amax / 127)), so no clamp is needed, and the code byte is the low byte of the bits of
// RN(y + 1.5 * 2^23) = 0x4B400000 + rint(y).  s > 0, r = RN(1/s).
__device__ __forceinline__ uint2 quant8_i8(const float (&x)[8], float s, float r) {
  uint32_t b[8];
  bool same = true;
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    const float2 y = fmul2(make_float2(x[e], x[e + 1]), make_float2(r, r));
    const float2 lo = ffma2(y, make_float2(kBracketLo, kBracketLo), make_float2(12582912.0f, 12582912.0f));
    const float2 hi = ffma2(y, make_float2(kBracketHi, kBracketHi), make_float2(12582912.0f, 12582912.0f));
    b[e] = __float_as_uint(lo.x);
    b[e + 1] = __float_as_uint(lo.y);
    same = same && (b[e] == __float_as_uint(hi.x)) && (b[e + 1] == __float_as_uint(hi.y));
  }
  if (!same) {
#pragma unroll
    for (int e = 0; e < 8; ++e) b[e] = (uint32_t)__float2int_rn(__fdiv_rn(x[e], s));
  }
  const uint32_t w0 = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
  const uint32_t w1 = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
  return make_uint2(w0, w1);
}

// Two E4M3 codes of x0 / s, x1 / s (lo byte x0); s > 0, r = RN(1/s).
// (the products run as f32x2 pairs: each lane is the same IEEE RN product)
__device__ __forceinline__ uint32_t quant_e4m3x2(float x0, float x1, float s, float r) {
  const float2 y = fmul2(make_float2(x0, x1), make_float2(r, r));
  const float2 yl = fmul2(y, make_float2(kBracketLo, kBracketLo));
  const float2 yh = fmul2(y, make_float2(kBracketHi, kBracketHi));
  const uint32_t lo = cvt_e4m3x2(yl.x, yl.y), hi = cvt_e4m3x2(yh.x, yh.y);
  return lo == hi ? lo : cvt_e4m3x2(__fdiv_rn(x0, s), __fdiv_rn(x1, s));
}

// Eight E2M1 codes of x[e] / s (element e in bits 4e..4e+3); s > 0, r = RN(1/s).
__device__ __forceinline__ uint32_t quant_e2m1x8(const float (&x)[8], float s, float r) {
  float l[8], h[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float y = __fmul_rn(x[e], r);
    l[e] = __fmul_rn(y, kBracketLo);
    h[e] = __fmul_rn(y, kBracketHi);
  }
  const uint32_t lo = cvt_e2m1x8(l[0], l[1], l[2], l[3], l[4], l[5], l[6], l[7]);
  const uint32_t hi = cvt_e2m1x8(h[0], h[1], h[2], h[3], h[4], h[5], h[6], h[7]);
  if (lo == hi) return lo;
  float q[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) q[e] = __fdiv_rn(x[e], s);
  return cvt_e2m1x8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
}

// CTA-wide maxima of NB non-negative floats per thread, all in one pass (one
// pair of CTA barriers for the NB values): out[nb] = max over the CTA of v[nb].
// red holds NB x (warps) floats; out is visible to every thread on return.
template <int NB>
__device__ __forceinline__ void block_max_nonneg_n(float (&v)[NB], float* red, float* out) {
  constexpr int NW = kThreads / 32;
#pragma unroll
  for (int nb = 0; nb < NB; ++nb)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v[nb] = fmaxf(v[nb], __shfl_xor_sync(0xffffffffu, v[nb], o));
  const int w = threadIdx.x / 32;
  __syncthreads();  // red and out may still be read by an earlier reduction
  if ((threadIdx.x & 31) == 0)
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) red[nb * NW + w] = v[nb];
  __syncthreads();
  if (threadIdx.x < NB) {
    float r = 0.0f;
#pragma unroll
    for (int i = 0; i < NW; ++i) r = fmaxf(r, red[threadIdx.x * NW + i]);
    out[threadIdx.x] = r;
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// Pass 1: per (b, kv-head, channel) fp64 sum of K (smooth K) and max |V|
// (skipped when a.vamax is null).
// grid (ceil(N / kStatRows), B*Hkv)
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) kv_stats_kernel(QuantArgs a) {
  constexpr int CH = D / 8, RG = kThreads / CH;
  __shared__ double s_sum[kThreads][8];
  __shared__ float s_amax[kThreads][8];
  const int bg = blockIdx.y;
  const int64_t r0 = (int64_t)blockIdx.x * kStatRows;
  const int64_t r1 = (r0 + kStatRows < (int64_t)a.N) ? r0 + kStatRows : (int64_t)a.N;
  const int ch = threadIdx.x % CH, rg = threadIdx.x / CH;
  const int64_t rs = row_stride(a.Hkv, D, a.nhd);
  const T* K = reinterpret_cast<const T*>(a.k) + row_offset(bg, 0, a.Hkv, a.N, D, a.nhd);
  const T* V = reinterpret_cast<const T*>(a.v) + row_offset(bg, 0, a.Hkv, a.N, D, a.nhd);
  double ks[8];
  float va[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) { ks[e] = 0.0; va[e] = 0.0f; }
  for (int64_t r = r0 + rg; r < r1; r += RG) {
    float x[8];
    load8<T>(K + r * rs + ch * 8, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) ks[e] += (double)x[e];
    if (a.vamax) {
      load8<T>(V + r * rs + ch * 8, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) va[e] = fmaxf(va[e], fabsf(x[e]));
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) { s_sum[threadIdx.x][e] = ks[e]; s_amax[threadIdx.x][e] = va[e]; }
  __syncthreads();
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    double s = 0.0;
    float m = 0.0f;
    for (int g = 0; g < RG; ++g) {
      s += s_sum[g * CH + c / 8][c % 8];
      m = fmaxf(m, s_amax[g * CH + c / 8][c % 8]);
    }
    if (a.smooth_k) atomicAdd(&a.ksum[(int64_t)bg * D + c], s);
    if (a.vamax) atomicMax(&a.vamax[(int64_t)bg * D + c], __float_as_uint(m));
  }
}

// ---------------------------------------------------------------------------
// Pass 2: one 128-row tile of Q, K or V per CTA.  The tile arrives in shared
// memory by one TMA load (3D map (D, N, B H) for HND inputs, 4D (D, N, H, B)
// for NHD; rows past N read as zeros), so
// the registers hold no tile and several CTAs per SM keep HBM busy; the
// threads then sweep the tile in shared memory (block sums, block max, codes).
template <typename T, int D>
__device__ __forceinline__ bool load_tile(T* dst, const CUtensorMap* map, uint64_t* bar, int row0, int bh, int H,
                                          int nhd) {
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_expect_tx(bar, kTile * D * (uint32_t)sizeof(T));
    if (nhd)
      tma_load_4d(dst, map, bar, 0, row0, bh % H, bh / H);  // (d, N, H, B) map
    else
      tma_load_3d(dst, map, bar, 0, row0, bh);  // (d, N, B H) map
  }
  return mbar_wait(bar, 0);
}

__device__ __forceinline__ uint8_t* align128(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 127) & ~uintptr_t(127));
}

// 8 consecutive elements of a row in shared memory as floats (exact)
template <typename T>
__device__ __forceinline__ void lds8(const T* p, float (&x)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  if constexpr (sizeof(T) == 2 && std::is_same<T, __nv_bfloat16>::value) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
}

// INT8 codes of one 128-row tile in shared memory (rows past N are zero):
// (s_red: NB x 8 floats)
// per BQ-row block, scale = max |x - shift| / 127 over the valid rows, codes
// rint(RN((x - shift) / scale)); writes the scales (s_k or s_q) and the codes
// (k8 or q8).  SHIFT = false: the shift is zero and the block max runs on the
// raw 16-bit magnitudes.  Every thread of the CTA calls it.
template <typename T, int D, int BQ, bool IS_K, bool SHIFT>
__device__ __forceinline__ void qk_encode(const T* sX, const float (*s_shift)[D], float* s_red, float* s_bmax,
                                          int bh, int tile, const QuantArgs& a) {
  constexpr int CH = D / 8, RG = kThreads / CH, NP = kTile / RG, NB = kTile / BQ, PPB = BQ / RG;
  const int64_t r0 = (int64_t)tile * kTile;
  const int valid = rows_valid(a.N, r0, kTile);
  const int ch = threadIdx.x % CH, rg = threadIdx.x / CH;
  const int Tb = IS_K ? a.Tn : a.Tm;
  // block max of |x - shift| over the valid rows
  float bm[NB];
  if (SHIFT) {
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) bm[nb] = 0.0f;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const int r = rg + p * RG;
      if (r < valid) {
        float x[8];
        lds8(sX + r * D + ch * 8, x);
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          const float2 d = fadd2(make_float2(x[e], x[e + 1]),
                                 make_float2(-s_shift[p / PPB][ch * 8 + e], -s_shift[p / PPB][ch * 8 + e + 1]));
          bm[p / PPB] = fmax3(bm[p / PPB], fabsf(d.x), fabsf(d.y));
        }
      }
    }
  } else {
    // max |x| on the bit patterns: non-negative bf16 / fp16 values order as
    // their 16-bit integers (rows past N hold zeros and change nothing)
    uint32_t mb[NB];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) mb[nb] = 0u;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const uint4 u = *reinterpret_cast<const uint4*>(sX + (rg + p * RG) * D + ch * 8);
      mb[p / PPB] = __vmaxu2(mb[p / PPB], __vmaxu2(__vmaxu2(u.x & 0x7FFF7FFFu, u.y & 0x7FFF7FFFu),
                                                   __vmaxu2(u.z & 0x7FFF7FFFu, u.w & 0x7FFF7FFFu)));
    }
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const uint32_t m16 = max(mb[nb] & 0xFFFFu, mb[nb] >> 16);
      if constexpr (std::is_same<T, __nv_bfloat16>::value)
        bm[nb] = __uint_as_float(m16 << 16);
      else
        bm[nb] = __half2float(__ushort_as_half((unsigned short)m16));
    }
  }
  block_max_nonneg_n<NB>(bm, s_red, s_bmax);
  float sc[NB], rc[NB];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    sc[nb] = __fdiv_rn(s_bmax[nb], 127.0f);
    rc[nb] = sc[nb] == 0.0f ? 0.0f : __frcp_rn(sc[nb]);
    const int gb = tile * NB + nb;
    if (threadIdx.x == 0 && gb < Tb) (IS_K ? a.s_k : a.s_q)[(int64_t)bh * Tb + gb] = sc[nb];
  }
  int8_t* out = (IS_K ? a.k8 : a.q8) + ((int64_t)bh * a.Np + r0) * D;
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int r = rg + p * RG;
    uint2 codes = make_uint2(0u, 0u);
    if (r < valid && sc[p / PPB] != 0.0f) {
      float x[8];
      lds8(sX + r * D + ch * 8, x);
      if (SHIFT) {
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          const float2 d = fadd2(make_float2(x[e], x[e + 1]),
                                 make_float2(-s_shift[p / PPB][ch * 8 + e], -s_shift[p / PPB][ch * 8 + e + 1]));
          x[e] = d.x;
          x[e + 1] = d.y;
        }
      }
      codes = quant8_i8(x, sc[p / PPB], rc[p / PPB]);
    }
    *reinterpret_cast<uint2*>(out + r * D + ch * 8) = codes;
  }
}

// smooth Q: the column means of each BQ-row block of a 128-row tile in shared
// memory (rows past N are zero): fp64 sums over the block, one fp64 division
// by its number of valid rows, one rounding to fp32 -> s_mean[nb][c], also
// written to qbar (when the block has rows).  Every thread of the CTA calls it.
template <typename T, int D, int BQ>
__device__ __forceinline__ void block_means(const T* sX, double (*s_sum)[8], float (*s_mean)[D], int bh, int tile,
                                            const QuantArgs& a) {
  constexpr int CH = D / 8, RG = kThreads / CH, NB = kTile / BQ, PPB = BQ / RG;
  const int64_t r0 = (int64_t)tile * kTile;
  const int ch = threadIdx.x % CH, rg = threadIdx.x / CH;
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    const int vb = rows_valid(a.N, r0 + nb * BQ, BQ);
    double cs[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) cs[e] = 0.0;
#pragma unroll
    for (int p = nb * PPB; p < (nb + 1) * PPB; ++p) {
      float x[8];
      lds8(sX + (rg + p * RG) * D + ch * 8, x);  // rows past N are zero
#pragma unroll
      for (int e = 0; e < 8; ++e) cs[e] += (double)x[e];
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 8; ++e) s_sum[threadIdx.x][e] = cs[e];
    __syncthreads();
    if (threadIdx.x < D) {
      const int c = threadIdx.x;
      double s = 0.0;
      for (int g = 0; g < RG; ++g) s += s_sum[g * CH + c / 8][c % 8];
      const float mu = vb > 0 ? __double2float_rn(__ddiv_rn(s, (double)vb)) : 0.0f;
      s_mean[nb][c] = mu;
      if (vb > 0) a.qbar[((int64_t)bh * a.Tm + tile * NB + nb) * D + c] = mu;
    }
  }
}

// Q (BQ-row blocks, optional block mean) or K (BQ = bk-row blocks, minus km):
// INT8 codes of x - shift with scale amax_block / 127.
//   IS_K = false: shift = qbar of the block when smooth_q (written to a.qbar)
//   IS_K = true:  shift = km = mean_n K (from the fp64 column sums)
// grid (Np/128, B*H), 256 threads, dynamic smem: 128 x D elements + 128
//   SHIFT: the shift is applied (smooth_q for Q, smooth_k for K); otherwise it
//   is identically zero and the block max runs on the raw 16-bit magnitudes.
//   QKM (Q only): also write Q_i . km per row (for the log-sum-exp); a template
//   choice so that the plain kernel carries none of it.
template <typename T, int D, int BQ, bool IS_K, bool SHIFT, bool QKM = false>
__global__ void __launch_bounds__(kThreads) qk_quant_kernel(const __grid_constant__ CUtensorMap tmX, QuantArgs a) {
  constexpr int NB = kTile / BQ;
  extern __shared__ uint8_t qk_smem_raw[];
  T* sX = reinterpret_cast<T*>(align128(qk_smem_raw));
  __shared__ double s_sum[kThreads][8];
  __shared__ float s_shift[NB][D], s_red[NB * (kThreads / 32)], s_bmax[NB];
  __shared__ uint64_t bar;
  const int bh = blockIdx.y, tile = blockIdx.x;
  const int64_t r0 = (int64_t)tile * kTile;
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    if (IS_K) {
      const float km = a.smooth_k ? __double2float_rn(__ddiv_rn(a.ksum[(int64_t)bh * D + c], (double)a.N)) : 0.0f;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) s_shift[nb][c] = km;
      if (tile == 0) a.km[(int64_t)bh * D + c] = km;
    } else {
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) s_shift[nb][c] = 0.0f;
    }
  }
  if (!load_tile<T, D>(sX, &tmX, &bar, (int)r0, bh, IS_K ? a.Hkv : a.Hq, a.nhd)) return;
  if (!IS_K && QKM) {
    // Q_i . km of every row of the tile (fp32), from the unshifted rows: the
    // constant by which smooth K shifts row i's scores (log-sum-exp correction)
    constexpr int CH = D / 8, RG = kThreads / CH;
    const int ch = threadIdx.x % CH, rg = threadIdx.x / CH;
    const float* km = a.km + (int64_t)((bh / a.Hq) * a.Hkv + (bh % a.Hq) / (a.Hq / a.Hkv)) * D + ch * 8;
    float kmc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) kmc[e] = km[e];
#pragma unroll 4
    for (int p = 0; p < kTile / RG; ++p) {
      const int r = rg + p * RG;
      float x[8];
      lds8(sX + r * D + ch * 8, x);  // rows past N are zero
      float dot = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) dot = fmaf(x[e], kmc[e], dot);
#pragma unroll
      for (int o = CH / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      if (ch == 0) a.qkm[(int64_t)bh * a.Np + r0 + r] = dot;
    }
  }
  if (!IS_K && SHIFT) block_means<T, D, BQ>(sX, s_sum, s_shift, bh, tile, a);
  __syncthreads();
  qk_encode<T, D, BQ, IS_K, SHIFT>(sX, s_shift, s_red, s_bmax, bh, tile, a);
}

// E4M3 codes of one 128-token V tile in shared memory (rows past N are zero),
// V / s_v[c] per channel, transposed: each thread encodes 16-token runs of one
// channel into registers; after a CTA barrier they are written as a
// 128-byte-swizzled [D x 128] tile at sVt (1024-byte aligned; it may overlay
// the V tile, which is consumed by then), and one TMA store writes that to
// v8t (the layout the attention kernel's TMA loads read).  Every thread of
// the CTA calls it; s_sv holds s_v of the head.
template <typename T, int D>
__device__ __forceinline__ void v_encode(const T* sV, uint8_t* sVt, const float* s_sv, const CUtensorMap* tmVt,
                                         int tile, int bg) {
  constexpr int TG = kThreads / D;       // token groups
  constexpr int RUNS = kTile / 16 / TG;  // 16-token runs per thread
  const int c = threadIdx.x % D, tg = threadIdx.x / D;
  const float sv = s_sv[c];
  const float rv = sv == 0.0f ? 0.0f : __frcp_rn(sv);
  uint4 codes[RUNS];
#pragma unroll
  for (int q = 0; q < RUNS; ++q) {
    const int run = tg * RUNS + q;
    uint32_t w[4];
#pragma unroll
    for (int u = 0; u < 16; u += 4) {
      float f[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) f[e] = to_float(sV[(run * 16 + u + e) * D + c]);
      w[u / 4] = sv == 0.0f ? 0u : quant_e4m3x2(f[0], f[1], sv, rv) | (quant_e4m3x2(f[2], f[3], sv, rv) << 16);
    }
    codes[q] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  __syncthreads();  // every thread has read the V tile
#pragma unroll
  for (int q = 0; q < RUNS; ++q) {
    const int run = tg * RUNS + q;
    *reinterpret_cast<uint4*>(sVt + c * kTile + ((run ^ (c & 7)) << 4)) = codes[q];
  }
  fence_proxy_async_smem();
  __syncthreads();
  if (threadIdx.x == 0) {
    tma_store_2d(tmVt, sVt, tile * kTile, bg * D);
    tma_store_commit_and_wait_read();
  }
}

// V: E4M3(V / s_v[c]) per channel, transposed to [D][Np] (v_encode; the codes
// overlay the tile).  grid (Np/128, B*Hkv), 256 threads, dynamic smem:
// 128 x D elements + 1024
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
    v_quant_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmVt, QuantArgs a) {
  extern __shared__ uint8_t v_smem_raw[];
  uint8_t* sVt = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(v_smem_raw) + 1023) & ~uintptr_t(1023));
  T* sV = reinterpret_cast<T*>(sVt);
  __shared__ float s_sv[D];
  __shared__ uint64_t bar;
  const int bg = blockIdx.y, tile = blockIdx.x;
  const int64_t r0 = (int64_t)tile * kTile;
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    const float sv = __fdiv_rn(__uint_as_float(a.vamax[(int64_t)bg * D + c]), 448.0f);
    s_sv[c] = sv;
    if (tile == 0) a.s_v[(int64_t)bg * D + c] = sv;
  }
  if (!load_tile<T, D>(sV, &tmX, &bar, (int)r0, bg, a.Hkv, a.nhd)) return;
  v_encode<T, D>(sV, sVt, s_sv, &tmVt, tile, bg);
}

// ---------------------------------------------------------------------------
// One-read K and V quantisation.  smooth K needs the mean of K over all N
// tokens and psi_V the max |V| of each channel over all N, so the two-pass
// path reads K and V twice (statistics, then codes).  Here a CTA loads one
// 128-token tile of K or V once, adds the tile's column sums (fp64) or
// column max |V| into its head's totals (the atomics of the statistics pass:
// fp64 sums of 16-bit inputs are exact in the range described at the top of
// this file, so the order does not matter),
// counts itself as published, and keeps the tile in shared memory until all
// tiles of its (head, K|V) group have published; then it reads km or s_v
// from the totals and writes its codes.
//
// Work items are handed out by ticket (one atomic increment per CTA), so
// tickets follow the order in which CTAs start: every lower ticket belongs to
// a CTA that is running or has finished.  A group's tiles hold consecutive
// tickets and wait only on each other, so every wait ends as long as one
// group fits in the CTAs resident at once (the launcher checks
// tiles <= resident / 2 and otherwise takes the two-pass path).
// Ticket t: group g = t / tiles = 2 (b Hkv + h) + (0: K, 1: V), tile t % tiles.
// grid (2 tiles B Hkv), 256 threads, dynamic smem: 128 x D elements + 1024
// (the V codes overlay the tile)
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait (one thread) for *counter >= target; false (and the timeout
// error recorded) when the limit ran out.
__device__ __noinline__ bool wait_count(const int* counter, int target) {
  if (ld_acquire_gpu(counter) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  const uint64_t limit = g_wait_limit_ns;
  while (true) {
    __nanosleep(100);
    if (ld_acquire_gpu(counter) >= target) return true;
    if (globaltimer_ns() - t0 > limit) {
      record_error(kDevErrTimeout);
      return false;
    }
  }
}

template <typename T>
__device__ __forceinline__ float half_bits_to_float(uint32_t m16) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value)
    return __uint_as_float(m16 << 16);
  else
    return __half2float(__ushort_as_half((unsigned short)m16));
}

template <typename T, int D, int BK, bool SMOOTH_K>
__global__ void __launch_bounds__(kThreads)
    kv_fused_quant_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const __grid_constant__ CUtensorMap tmVt, QuantArgs a) {
  constexpr int CH = D / 8, RG = kThreads / CH, NP = kTile / RG, NB = kTile / BK, NW = kThreads / 32;
  extern __shared__ uint8_t kvf_smem_raw[];
  uint8_t* sVt = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(kvf_smem_raw) + 1023) & ~uintptr_t(1023));
  T* sX = reinterpret_cast<T*>(sVt);
  __shared__ double s_pk[NW * D];                       // per-warp column sums (K group)
  unsigned* s_pv = reinterpret_cast<unsigned*>(s_pk);  // per-warp column max |V| bits (V group)
  __shared__ float s_shift[NB][D], s_red[NB * NW], s_bmax[NB];
  __shared__ uint64_t bar;
  __shared__ int s_item, s_ok;
  const int tiles = (int)(a.Np / kTile);
  int* published = a.kv_sync + 1;
  if (threadIdx.x == 0) s_item = atomicAdd(a.kv_sync, 1);
  __syncthreads();
  const int grp = s_item / tiles, tile = s_item % tiles;
  const int bh = grp >> 1;
  const bool is_v = (grp & 1) != 0;
  if (!load_tile<T, D>(sX, is_v ? &tmV : &tmK, &bar, tile * kTile, bh, a.Hkv, a.nhd)) return;
  if (!is_v && !SMOOTH_K) {  // km = 0: nothing to wait for
    if (tile == 0 && threadIdx.x < D) a.km[(int64_t)bh * D + threadIdx.x] = 0.0f;
    qk_encode<T, D, BK, true, false>(sX, s_shift, s_red, s_bmax, bh, tile, a);
    return;
  }
  // ---- this tile's column statistics (rows past N are zero and change nothing)
  const int ch = threadIdx.x % CH, rg = threadIdx.x / CH, warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (!is_v) {
    double cs[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) cs[e] = 0.0;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      float x[8];
      lds8(sX + (rg + p * RG) * D + ch * 8, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) cs[e] += (double)x[e];
    }
    // lanes l, l + CH, ... of a warp hold the same channels
#pragma unroll
    for (int o = CH; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) cs[e] += __shfl_xor_sync(0xffffffffu, cs[e], o);
    if (lane < CH)
#pragma unroll
      for (int e = 0; e < 8; ++e) s_pk[warp * D + ch * 8 + e] = cs[e];
  } else {
    // max |v| on the bit patterns (non-negative 16-bit floats order as integers)
    uint32_t mv[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const uint4 u = *reinterpret_cast<const uint4*>(sX + (rg + p * RG) * D + ch * 8);
      mv[0] = __vmaxu2(mv[0], u.x & 0x7FFF7FFFu);
      mv[1] = __vmaxu2(mv[1], u.y & 0x7FFF7FFFu);
      mv[2] = __vmaxu2(mv[2], u.z & 0x7FFF7FFFu);
      mv[3] = __vmaxu2(mv[3], u.w & 0x7FFF7FFFu);
    }
#pragma unroll
    for (int o = CH; o < 32; o <<= 1)
#pragma unroll
      for (int i = 0; i < 4; ++i) mv[i] = __vmaxu2(mv[i], __shfl_xor_sync(0xffffffffu, mv[i], o));
    if (lane < CH)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        s_pv[warp * D + ch * 8 + 2 * i] = __float_as_uint(half_bits_to_float<T>(mv[i] & 0xFFFFu));
        s_pv[warp * D + ch * 8 + 2 * i + 1] = __float_as_uint(half_bits_to_float<T>(mv[i] >> 16));
      }
  }
  __syncthreads();
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    if (!is_v) {
      double s = 0.0;
#pragma unroll
      for (int w = 0; w < NW; ++w) s += s_pk[w * D + c];
      atomicAdd(a.ksum + (int64_t)bh * D + c, s);
    } else {
      unsigned m = 0u;
#pragma unroll
      for (int w = 0; w < NW; ++w) m = max(m, s_pv[w * D + c]);
      atomicMax(a.vamax + (int64_t)bh * D + c, m);
    }
    __threadfence();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    atomicAdd(published + grp, 1);
    s_ok = wait_count(published + grp, tiles) ? 1 : 0;  // every tile of the group added its part
  }
  __syncthreads();
  if (!s_ok) return;  // timeout recorded; the codes of this tile are not written
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    if (!is_v) {
      const float km = __double2float_rn(__ddiv_rn(__ldcg(a.ksum + (int64_t)bh * D + c), (double)a.N));
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) s_shift[nb][c] = km;
      if (tile == 0) a.km[(int64_t)bh * D + c] = km;
    } else {
      const float sv = __fdiv_rn(__uint_as_float(__ldcg(a.vamax + (int64_t)bh * D + c)), 448.0f);
      s_shift[0][c] = sv;
      if (tile == 0) a.s_v[(int64_t)bh * D + c] = sv;
    }
  }
  __syncthreads();
  if (!is_v)
    qk_encode<T, D, BK, true, SMOOTH_K>(sX, s_shift, s_red, s_bmax, bh, tile, a);
  else
    v_encode<T, D>(sX, sVt, s_shift[0], &tmVt, tile, bh);
}

// ---------------------------------------------------------------------------
// delta_S on the tensor cores.  Per (b, h) and 128-key tile j:
//   delta_S^T[key, i] = sum_c gamma(K)[key, c] qbar[i, c]
// is a [128 x d] x [d x Tm] contraction, so it runs as tcgen05.mma kind::tf32
// with the keys as M (the accumulator's TMEM lanes) and the Q blocks as N.
// TF32 keeps 10 of fp32's 23 mantissa bits, so each operand is split exactly
// into x = hi + lo (hi: x with the low 13 mantissa bits cleared, a TF32 value;
// lo = x - hi, exact in fp32) and three products accumulate in FP32:
// hi lo + lo hi first (the small terms), then hi hi; the dropped lo lo term
// and the TF32 rounding of lo are below 2^-20 of |x y| per product.
// The channels go through in passes of 64 (operands of 128 keys and of
// kDsTcBlocks Q blocks, hi and lo: 104 KB, so two CTAs share an SM and one's
// loads overlap the other's MMAs and stores); the Q blocks in chunks of
// kDsTcBlocks (the accumulator's columns).
// Operands in shared memory, K-major with the 128-byte swizzle: element
// (r, c) of an R-row operand sits in 32-channel column block c / 32 (R x 128
// bytes), row r, 16-byte unit ((c % 32) / 4) ^ (r % 8).
// grid (Np/128, B*Hq), 256 threads; dynamic smem ds_tc_smem().  Keys past N
// give gamma = 0, so their delta_S columns are written as zeros, like the rest
// of the padding.
constexpr int kDsTcBlocks = 80;  // Q blocks per chunk (MMA N <= 80)
constexpr int kDsTcCh = 64;      // channels per pass

constexpr size_t ds_tc_smem() { return (size_t)2 * (kTile + kDsTcBlocks) * kDsTcCh * 4 + 1024; }

__device__ __forceinline__ uint32_t swz128_offset(int r, int c, int rows) {
  return (uint32_t)((c >> 5) * rows * 128 + r * 128 + ((((c & 31) >> 2) ^ (r & 7)) << 4) + (c & 3) * 4);
}

// split 8 consecutive fp32 (channels c .. c + 7 of the pass, c % 8 == 0) of
// row r into the hi / lo operands
__device__ __forceinline__ void store_split8(uint8_t* hi, uint8_t* lo, int r, int c, int rows, const float (&x)[8]) {
  float h[8], l[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    h[e] = __uint_as_float(__float_as_uint(x[e]) & 0xFFFFE000u);
    l[e] = __fsub_rn(x[e], h[e]);
  }
  const uint32_t o0 = swz128_offset(r, c, rows), o1 = swz128_offset(r, c + 4, rows);
  *reinterpret_cast<float4*>(hi + o0) = make_float4(h[0], h[1], h[2], h[3]);
  *reinterpret_cast<float4*>(hi + o1) = make_float4(h[4], h[5], h[6], h[7]);
  *reinterpret_cast<float4*>(lo + o0) = make_float4(l[0], l[1], l[2], l[3]);
  *reinterpret_cast<float4*>(lo + o1) = make_float4(l[4], l[5], l[6], l[7]);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 2) delta_s_tc_kernel(QuantArgs a) {
  constexpr int NBK = kDsTcBlocks, CP = kDsTcCh, G8 = CP / 8;  // 8-channel groups per pass row
  constexpr uint32_t kA = kTile * CP * 4, kB = NBK * CP * 4;
  constexpr uint32_t kCols = 128;
  static_assert(D % CP == 0 && NBK % 16 == 0 && NBK <= (int)kCols, "delta_S tile shape");
  extern __shared__ uint8_t ds_tc_raw[];
  uint8_t* sAh = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ds_tc_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sAl = sAh + kA;
  uint8_t* sBh = sAl + kA;
  uint8_t* sBl = sBh + kB;
  __shared__ uint64_t mma_bar;
  __shared__ uint32_t tmem_slot;
  const int bh = blockIdx.y, tile = blockIdx.x;
  const int b = bh / a.Hq, h = bh % a.Hq;
  const int bg = b * a.Hkv + h / (a.Hq / a.Hkv);
  const int64_t r0 = (int64_t)tile * kTile;
  const int valid = rows_valid(a.N, r0, kTile);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (warp == 0) {
    tmem_alloc(&tmem_slot, kCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    mbar_init(&mma_bar, 1);
    mbar_fence_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const T* K = reinterpret_cast<const T*>(a.k) + row_offset(bg, r0, a.Hkv, a.N, D, a.nhd);
  const int64_t krs = row_stride(a.Hkv, D, a.nhd);
  const float* km = a.km + (int64_t)bg * D;
  const float* qb = a.qbar + (int64_t)bh * a.Tm * D;
  float* out = a.dS + (int64_t)bh * a.Tm * a.Np + r0;
  const int quarter = warp & 3, half = warp >> 2;
  const int cl = (threadIdx.x % G8) * 8;  // this thread's channels within a pass (every step)
  // Passes (chunk of NBK Q blocks, 64 channels) run in order; the global loads
  // of pass p + 1 are issued as soon as pass p's operands are in shared memory,
  // so they are in flight during pass p's MMAs and stores (the registers that
  // hold them are free by then).
  constexpr int NPC = D / CP;  // passes per chunk
  constexpr int ITA = kTile * G8 / kThreads, ITB = (NBK * G8 + kThreads - 1) / kThreads;
  const int n_pass = ((a.Tm + NBK - 1) / NBK) * NPC;
  uint4 ka[ITA];
  float4 qv[ITB][2];
  // A = gamma(K)[:, c0 .. c0 + 64) (rows past N zero; with a single pass per
  // chunk (d = 64) A stays from the first chunk), B = qbar[i0 .., c0 ..) (rows
  // past Tm zero)
  auto load_pass = [&](int pass) {
    const int pi0 = (pass / NPC) * NBK, pc0 = (pass % NPC) * CP;
    const int pnb = min(NBK, a.Tm - pi0);
    const bool load_a = D > CP || pi0 == 0;
#pragma unroll
    for (int it = 0; it < ITA; ++it) {
      const int r = (threadIdx.x + it * kThreads) / G8;
      ka[it] = (load_a && r < valid) ? __ldg(reinterpret_cast<const uint4*>(K + (int64_t)r * krs + pc0 + cl))
                                     : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int it = 0; it < ITB; ++it) {
      const int r = (threadIdx.x + it * kThreads) / G8;
      const float* src = qb + (int64_t)(pi0 + r) * D + pc0 + cl;
      qv[it][0] = r < pnb ? __ldg(reinterpret_cast<const float4*>(src)) : make_float4(0.f, 0.f, 0.f, 0.f);
      qv[it][1] = r < pnb ? __ldg(reinterpret_cast<const float4*>(src + 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  bool ok = true;
  uint32_t phase = 0;
  load_pass(0);
  for (int pass = 0; pass < n_pass && ok; ++pass, phase ^= 1u) {
    const int i0 = (pass / NPC) * NBK, c0 = (pass % NPC) * CP;
    const int nb = min(NBK, a.Tm - i0);
    const int nbp = (nb + 15) & ~15;  // MMA N: a multiple of 16
    const uint32_t idesc = make_idesc(/*F32*/ 1, /*TF32*/ 2, /*TF32*/ 2, kTile, nbp);
    const bool load_a = D > CP || i0 == 0;
    float kmc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) kmc[e] = km[c0 + cl + e];
    // the previous pass's MMAs have read the operands (waited on below)
    if (load_a) {
#pragma unroll
      for (int it = 0; it < ITA; ++it) {
        const int r = (threadIdx.x + it * kThreads) / G8;
        float x[8];
        lds8(reinterpret_cast<const T*>(&ka[it]), x);
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = r < valid ? __fsub_rn(x[e], kmc[e]) : 0.0f;
        store_split8(sAh, sAl, r, cl, kTile, x);
      }
    }
#pragma unroll
    for (int it = 0; it < ITB; ++it) {
      const int r = (threadIdx.x + it * kThreads) / G8;
      if (r < nbp) {
        const float x[8] = {qv[it][0].x, qv[it][0].y, qv[it][0].z, qv[it][0].w,
                            qv[it][1].x, qv[it][1].y, qv[it][1].z, qv[it][1].w};
        store_split8(sBh, sBl, r, cl, NBK, x);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
      const uint32_t aH = smem_u32(sAh), aL = smem_u32(sAl), bH = smem_u32(sBh), bL = smem_u32(sBl);
      // K step kk: 8 channels = 32 bytes inside 32-channel column block kk / 4
#pragma unroll
      for (int kk = 0; kk < CP / 8; ++kk) {
        const uint32_t oa = (kk >> 2) * kTile * 128 + (kk & 3) * 32, ob = (kk >> 2) * NBK * 128 + (kk & 3) * 32;
        mma_tf32(tmem, make_sdesc(aH + oa, 1024, kSwizzle128B), make_sdesc(bL + ob, 1024, kSwizzle128B), idesc,
                 (c0 > 0 || kk > 0) ? 1u : 0u);
        mma_tf32(tmem, make_sdesc(aL + oa, 1024, kSwizzle128B), make_sdesc(bH + ob, 1024, kSwizzle128B), idesc,
                 1u);
      }
#pragma unroll
      for (int kk = 0; kk < CP / 8; ++kk) {
        const uint32_t oa = (kk >> 2) * kTile * 128 + (kk & 3) * 32, ob = (kk >> 2) * NBK * 128 + (kk & 3) * 32;
        mma_tf32(tmem, make_sdesc(aH + oa, 1024, kSwizzle128B), make_sdesc(bH + ob, 1024, kSwizzle128B), idesc,
                 1u);
      }
      mma_commit(&mma_bar);
    }
    if (pass + 1 < n_pass) load_pass(pass + 1);
    __syncwarp();
    ok = mbar_wait_warp(&mma_bar, phase);
    tc_fence_after();
    ok = __syncthreads_and(ok);
    if (ok && c0 + CP == D) {
      // the chunk's accumulator is complete.  Lanes 32 quarter ..: keys; the two
      // halves of the CTA take alternate 16-block groups
      const uint32_t tq = tmem + ((uint32_t)(quarter * 32) << 16);
      const int key = quarter * 32 + lane;
      for (int g = half; g < nbp / 16; g += 2) {
        uint32_t v[16];
        tmem_ld16p(tq + g * 16, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int i = i0 + g * 16 + e;
          if (i < a.Tm) out[(int64_t)i * a.Np + key] = __uint_as_float(v[e]);
        }
      }
      // every warp has read the accumulator before the next chunk's MMAs
      tc_fence_before();
      ok = __syncthreads_and(ok);
      tc_fence_after();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

template <typename T, int D>
cudaError_t launch_delta_s(const QuantArgs& a, cudaStream_t st) {
  const int tiles = (int)(a.Np / kTile);
  const int smem = (int)ds_tc_smem();
  cudaError_t e = cudaFuncSetAttribute(delta_s_tc_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  delta_s_tc_kernel<T, D><<<dim3(tiles, a.B * a.Hq), kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

// The one-read K/V kernel for (bk, smooth_k), or nullptr if a (head, K|V)
// group of `tiles` CTAs might not fit in half of the CTAs resident at once
// (then the two-pass path runs).  head_dim 64 also takes the two-pass path:
// a 16 KB tile per CTA does not amortise the ticket, fence and wait (measured
// 2.5 % slower than two passes on B=2, H=48, N=17776; head_dim 128: 12 % and
// 6 % faster on N=4096 and N=32768).
template <typename T, int D>
void (*kv_fused_kernel(const QuantArgs& a, int tiles, int smem))(CUtensorMap, CUtensorMap, CUtensorMap, QuantArgs) {
  if (D != 128) return nullptr;
  auto kf = a.bk == 64 ? (a.smooth_k ? kv_fused_quant_kernel<T, D, 64, true> : kv_fused_quant_kernel<T, D, 64, false>)
                       : (a.smooth_k ? kv_fused_quant_kernel<T, D, 128, true> : kv_fused_quant_kernel<T, D, 128, false>);
  if (cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return nullptr;
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kf, kThreads, smem) != cudaSuccess)
    return nullptr;
  return (a.force_one_read || (int64_t)tiles * 2 <= (int64_t)sms * per_sm) ? kf : nullptr;
}

template <typename T, int D, bool QKM>
auto q_quant_pick(const QuantArgs& a) {
  return a.bq == 32   ? (a.smooth_q ? qk_quant_kernel<T, D, 32, false, true, QKM> : qk_quant_kernel<T, D, 32, false, false, QKM>)
         : a.bq == 64 ? (a.smooth_q ? qk_quant_kernel<T, D, 64, false, true, QKM> : qk_quant_kernel<T, D, 64, false, false, QKM>)
                      : (a.smooth_q ? qk_quant_kernel<T, D, 128, false, true, QKM> : qk_quant_kernel<T, D, 128, false, false, QKM>);
}

template <typename T, int D>
cudaError_t launch_quant_t(const QuantArgs& a, const QuantMaps& m, cudaStream_t st) {
  cudaError_t e;
  const int BHkv = a.B * a.Hkv, BHq = a.B * a.Hq;
  const int tiles = (int)(a.Np / kTile);
  const int smem_kvf = kTile * D * (int)sizeof(T) + 1024;
  auto kf = a.kv_sync ? kv_fused_kernel<T, D>(a, tiles, smem_kvf) : nullptr;
  if (kf) {
    // ksum, vamax and kv_sync are consecutive in the workspace: one memset
    e = cudaMemsetAsync(a.ksum, 0, a.kv_zero_bytes, st);
    if (e != cudaSuccess) return e;
    kf<<<dim3(2 * tiles * BHkv), kThreads, smem_kvf, st>>>(m.k, m.v, m.vt, a);
  }
  const int smem_qk = kTile * D * (int)sizeof(T) + 128;
  if (!kf) {  // two passes: column statistics, then the K and V codes
    if (a.smooth_k) {
      e = cudaMemsetAsync(a.ksum, 0, sizeof(double) * (size_t)BHkv * D, st);
      if (e != cudaSuccess) return e;
    }
    e = cudaMemsetAsync(a.vamax, 0, sizeof(unsigned) * (size_t)BHkv * D, st);
    if (e != cudaSuccess) return e;
    kv_stats_kernel<T, D><<<dim3((a.N + kStatRows - 1) / kStatRows, BHkv), kThreads, 0, st>>>(a);
    auto kq = a.bk == 64 ? (a.smooth_k ? qk_quant_kernel<T, D, 64, true, true> : qk_quant_kernel<T, D, 64, true, false>)
                         : (a.smooth_k ? qk_quant_kernel<T, D, 128, true, true> : qk_quant_kernel<T, D, 128, true, false>);
    e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_qk);
    if (e != cudaSuccess) return e;
    kq<<<dim3(tiles, BHkv), kThreads, smem_qk, st>>>(m.k, a);
    const int smem = kTile * D * (int)sizeof(T) + 1024;
    e = cudaFuncSetAttribute(v_quant_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    v_quant_kernel<T, D><<<dim3(tiles, BHkv), kThreads, smem, st>>>(m.v, m.vt, a);
  }
  {
    auto qq = a.qkm ? q_quant_pick<T, D, true>(a) : q_quant_pick<T, D, false>(a);
    e = cudaFuncSetAttribute(qq, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_qk);
    if (e != cudaSuccess) return e;
    qq<<<dim3(tiles, BHq), kThreads, smem_qk, st>>>(m.q, a);
  }
  if (a.smooth_q) {
    e = launch_delta_s<T, D>(a, st);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

template <typename T, int D>
int quant_kernel_count_t(const QuantArgs& a, bool allow_one_read) {
  const int tiles = (int)(a.Np / kTile);
  const bool one_read = allow_one_read && kv_fused_kernel<T, D>(a, tiles, kTile * D * (int)sizeof(T) + 1024);
  return (one_read ? 2 : 4) + (a.smooth_q ? 1 : 0);
}

}  // namespace

int quant_kernel_count(const QuantArgs& a, int is_fp16, bool allow_one_read) {
  if (is_fp16)
    return a.D == 128 ? quant_kernel_count_t<__half, 128>(a, allow_one_read)
                      : quant_kernel_count_t<__half, 64>(a, allow_one_read);
  return a.D == 128 ? quant_kernel_count_t<__nv_bfloat16, 128>(a, allow_one_read)
                    : quant_kernel_count_t<__nv_bfloat16, 64>(a, allow_one_read);
}

cudaError_t launch_quant(const QuantArgs& a, const QuantMaps& m, int is_fp16, cudaStream_t st) {
  if (is_fp16) return a.D == 128 ? launch_quant_t<__half, 128>(a, m, st) : launch_quant_t<__half, 64>(a, m, st);
  return a.D == 128 ? launch_quant_t<__nv_bfloat16, 128>(a, m, st) : launch_quant_t<__nv_bfloat16, 64>(a, m, st);
}

}  // namespace sage
