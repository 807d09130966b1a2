// quant_nvfp4.cu -- NVFP4 preprocessing on sm_100a (HBM-bound kernels).
//
// SageAttention3 as summarised in its reading note
// (zhaifeiyue.github.io/papers/2505.11594), "Microscaling FP4 attention": Q and
// K are smoothed (K by its token mean, Q by its per-block mean with the delta_S
// compensation of SageAttention2), then every group of 16 consecutive elements
// along the head dimension gets one E4M3 scale, sb = E4M3(amax16 / 6), and E2M1
// codes E2M1(x / sb).  V is grouped the same way along tokens (the reduction
// axis of P V).  Every division is an IEEE fp32 division (__fdiv_rn; per
// element a reciprocal multiply where it provably gives the same code); E2M1 and
// E4M3 use round-to-nearest-even with saturation (cvt.rn.satfinite), so codes
// and scales are bit-exact with the plain definitions.
//
// Output layouts (what the attention kernel's TMA / bulk copies read):
//   q4 [B,Hq,Np,64], k4 [B,Hkv,Np,64]: E2M1 codes of a row, two per byte, the
//     even element in the low nibble.
//   v4t [B,Hkv,128,Np/2]: V transposed, codes along tokens, same packing.
//   sfq / sfk / sfv [.., Np/128, 1024]: per 128-row tile, two 512-byte blocks
//     (K chunks of 64 elements); in block kk the scale of row m (Q row, key, or
//     V channel) for its 16-element group kk*4 + k sits at byte
//     16 (m % 32) + 4 (m / 32) + k -- the order tcgen05.cp broadcasts into TMEM.
// Only head_dim 128 is supported on this path.

namespace sage {

namespace {

constexpr int kF4D = 128;

__device__ __forceinline__ int sf_byte(int m, int grp) {
  return (grp >> 2) * 512 + 16 * (m & 31) + 4 * (m >> 5) + (grp & 3);
}

// E2M1 codes of x / sd for 8 values (0 when sd == 0), packed low nibble first.
__device__ __forceinline__ uint32_t encode8_e2m1(const float (&x)[8], float sd) {
  return sd == 0.0f ? 0u : quant_e2m1x8(x, sd, __frcp_rn(sd));
}

// Encodes row chunk x (8 channels) of a 16-group shared with the partner lane
// (lane ^ 1): returns the 4 code bytes, writes the group's scale code to *sc.
__device__ __forceinline__ uint32_t encode_pair(const float (&x)[8], uint32_t* sc) {
  float am = 0.0f;
#pragma unroll
  for (int e = 0; e < 8; ++e) am = fmaxf(am, fabsf(x[e]));
  am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
  const uint32_t c = cvt_e4m3(__fdiv_rn(am, 6.0f));
  *sc = c;
  return encode8_e2m1(x, e4m3_value(c));
}

// ---------------------------------------------------------------------------
// K: gamma(K) = K - km, NVFP4 along d.  grid (Np/128, B*Hkv), 256 threads.
template <typename T>
__global__ void __launch_bounds__(kThreads) k_quant_nvfp4_kernel(QuantArgs a) {
  constexpr int D = kF4D, CH = D / 8, RG = kThreads / CH, NP = kTile / RG;
  __shared__ float s_km[D];
  __shared__ __align__(16) uint8_t s_sf[1024];
  const int bg = blockIdx.y, tile = blockIdx.x;
  const int64_t r0 = (int64_t)tile * kTile;
  const int valid = rows_valid(a.N, r0, kTile);
  const int ch = threadIdx.x % CH, rg = threadIdx.x / CH;
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    const float km = a.smooth_k ? __double2float_rn(__ddiv_rn(a.ksum[(int64_t)bg * D + c], (double)a.N)) : 0.0f;
    s_km[c] = km;
    if (tile == 0) a.km[(int64_t)bg * D + c] = km;
  }
  __syncthreads();
  const T* K = reinterpret_cast<const T*>(a.k) + row_offset(bg, 0, a.Hkv, a.N, D, a.nhd);
  const int64_t rs = row_stride(a.Hkv, D, a.nhd);
  uint8_t* k4 = a.k4 + ((int64_t)bg * a.Np + r0) * (D / 2);
#pragma unroll 2
  for (int p = 0; p < NP; ++p) {
    const int r = rg + p * RG;
    float x[8];
    if (r < valid) {
      load8<T>(K + (r0 + r) * rs + ch * 8, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = __fsub_rn(x[e], s_km[ch * 8 + e]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = 0.0f;
    }
    uint32_t sc;
    const uint32_t codes = encode_pair(x, &sc);
    *reinterpret_cast<uint32_t*>(k4 + r * (D / 2) + ch * 4) = codes;
    if ((ch & 1) == 0) s_sf[sf_byte(r, ch >> 1)] = (uint8_t)sc;
  }
  __syncthreads();
  reinterpret_cast<uint32_t*>(a.sfk + ((int64_t)bg * (a.Np / kTile) + tile) * 1024)[threadIdx.x] =
      reinterpret_cast<const uint32_t*>(s_sf)[threadIdx.x];
}

// ---------------------------------------------------------------------------
// NVFP4 codes of one 128-row tile in shared memory (rows past N are zero):
// x - shift[row block] for the valid rows (shift == nullptr: no shift), one
// E4M3 scale per 16 channels, codes to x4 (this tile's rows), scales to the
// tile's 1 KB block sf.  Every thread of the CTA calls it.
template <typename T, int BQ>
__device__ __forceinline__ void nvfp4_encode_tile(const T* sX, const float (*shift)[kF4D], uint8_t* s_sf, int valid,
                                                  uint8_t* x4, uint8_t* sf) {
  constexpr int D = kF4D, CH = D / 8, RG = kThreads / CH, NP = kTile / RG, PPB = BQ / RG;
  const int ch = threadIdx.x % CH, rg = threadIdx.x / CH;
#pragma unroll 4
  for (int p = 0; p < NP; ++p) {
    const int r = rg + p * RG;
    float x[8];
    lds8(sX + r * D + ch * 8, x);
    if (shift != nullptr && r < valid) {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = __fsub_rn(x[e], shift[p / PPB][ch * 8 + e]);
    }
    uint32_t sc;
    const uint32_t codes = encode_pair(x, &sc);
    *reinterpret_cast<uint32_t*>(x4 + r * (D / 2) + ch * 4) = codes;
    if ((ch & 1) == 0) s_sf[sf_byte(r, ch >> 1)] = (uint8_t)sc;
  }
  __syncthreads();
  reinterpret_cast<uint32_t*>(sf)[threadIdx.x] = reinterpret_cast<const uint32_t*>(s_sf)[threadIdx.x];
}

// Q: optional per-BQ-block mean (smooth Q), NVFP4 along d.  One 128-row tile
// per CTA, staged in shared memory by one TMA load (3D map, rows past N read
// as zeros).  grid (Np/128, B*Hq), 256 threads, dynamic smem 128 x 128
// elements + 128.
template <typename T, int BQ, bool SHIFT>
__global__ void __launch_bounds__(kThreads) q_quant_nvfp4_kernel(const __grid_constant__ CUtensorMap tmQ, QuantArgs a) {
  constexpr int D = kF4D, NB = kTile / BQ;
  extern __shared__ uint8_t q4_smem_raw[];
  T* sX = reinterpret_cast<T*>(align128(q4_smem_raw));
  __shared__ double s_sum[SHIFT ? kThreads : 1][8];
  __shared__ float s_mean[NB][D];
  __shared__ __align__(16) uint8_t s_sf[1024];
  __shared__ uint64_t bar;
  const int bh = blockIdx.y, tile = blockIdx.x;
  const int64_t r0 = (int64_t)tile * kTile;
  if (!load_tile<T, D>(sX, &tmQ, &bar, (int)r0, bh, a.Hq, a.nhd)) return;
  if (SHIFT) block_means<T, D, BQ>(sX, s_sum, s_mean, bh, tile, a);
  __syncthreads();
  nvfp4_encode_tile<T, BQ>(sX, SHIFT ? s_mean : nullptr, s_sf, rows_valid(a.N, r0, kTile),
                           a.q4 + ((int64_t)bh * a.Np + r0) * (D / 2),
                           a.sfq + ((int64_t)bh * (a.Np / kTile) + tile) * 1024);
}

// ---------------------------------------------------------------------------
// One-read K: each CTA loads one 128-token tile of K once and keeps it in
// shared memory while its head's column sums complete (the scheme of the
// INT8 path's one-read K/V kernel: tickets in CTA start order, fp64 atomics,
// a publish counter per head, bounded waits), then encodes gamma(K) = K - km.
// Ticket t: head t / tiles, tile t % tiles.  grid (tiles B Hkv), 256 threads,
// dynamic smem 128 x 128 elements + 128.
template <typename T, bool SMOOTH_K>
__global__ void __launch_bounds__(kThreads) k_fused_nvfp4_kernel(const __grid_constant__ CUtensorMap tmK, QuantArgs a) {
  constexpr int D = kF4D, CH = D / 8, RG = kThreads / CH, NP = kTile / RG, NW = kThreads / 32;
  extern __shared__ uint8_t k4_smem_raw[];
  T* sX = reinterpret_cast<T*>(align128(k4_smem_raw));
  __shared__ double s_pk[SMOOTH_K ? NW * D : 1];
  __shared__ float s_km[1][D];
  __shared__ __align__(16) uint8_t s_sf[1024];
  __shared__ uint64_t bar;
  __shared__ int s_item, s_ok;
  const int tiles = (int)(a.Np / kTile);
  if (threadIdx.x == 0) s_item = atomicAdd(a.kv_sync, 1);
  __syncthreads();
  const int bg = s_item / tiles, tile = s_item % tiles;
  if (!load_tile<T, D>(sX, &tmK, &bar, tile * kTile, bg, a.Hkv, a.nhd)) return;
  if constexpr (SMOOTH_K) {
    const int ch = threadIdx.x % CH, rg = threadIdx.x / CH, warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    double cs[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) cs[e] = 0.0;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      float x[8];
      lds8(sX + (rg + p * RG) * D + ch * 8, x);  // rows past N are zero
#pragma unroll
      for (int e = 0; e < 8; ++e) cs[e] += (double)x[e];
    }
#pragma unroll
    for (int o = CH; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) cs[e] += __shfl_xor_sync(0xffffffffu, cs[e], o);
    if (lane < CH)
#pragma unroll
      for (int e = 0; e < 8; ++e) s_pk[warp * D + ch * 8 + e] = cs[e];
    __syncthreads();
    if (threadIdx.x < D) {
      double sum = 0.0;
#pragma unroll
      for (int w = 0; w < NW; ++w) sum += s_pk[w * D + threadIdx.x];
      atomicAdd(a.ksum + (int64_t)bg * D + threadIdx.x, sum);
      __threadfence();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      atomicAdd(a.kv_sync + 1 + bg, 1);
      s_ok = wait_count(a.kv_sync + 1 + bg, tiles) ? 1 : 0;  // every tile of the head added its sums
    }
    __syncthreads();
    if (!s_ok) return;  // timeout recorded; this tile's codes are not written
    if (threadIdx.x < D) {
      const float km = __double2float_rn(__ddiv_rn(__ldcg(a.ksum + (int64_t)bg * D + threadIdx.x), (double)a.N));
      s_km[0][threadIdx.x] = km;
      if (tile == 0) a.km[(int64_t)bg * D + threadIdx.x] = km;
    }
  } else {
    if (threadIdx.x < D && tile == 0) a.km[(int64_t)bg * D + threadIdx.x] = 0.0f;
  }
  __syncthreads();
  nvfp4_encode_tile<T, kTile>(sX, SMOOTH_K ? s_km : nullptr, s_sf, rows_valid(a.N, (int64_t)tile * kTile, kTile),
                              a.k4 + ((int64_t)bg * a.Np + (int64_t)tile * kTile) * (D / 2),
                              a.sfk + ((int64_t)bg * (a.Np / kTile) + tile) * 1024);
}

// ---------------------------------------------------------------------------
// V: NVFP4 along tokens (16-token groups per channel), transposed to
// [D][Np/2].  The tile arrives in shared memory by one TMA load; each thread
// encodes (channel, 16-token group) items, consecutive threads taking
// consecutive channels, and keeps the codes in registers; after a barrier they
// are written over the consumed tile so that the global stores are 16-byte
// rows.  grid (Np/128, B*Hkv), 256 threads, dynamic smem 128 x 128 elements + 128.
template <typename T>
__global__ void __launch_bounds__(kThreads) v_quant_nvfp4_kernel(const __grid_constant__ CUtensorMap tmV, QuantArgs a) {
  constexpr int D = kF4D, IT = (D * 8) / kThreads;  // (channel, group) items per thread
  extern __shared__ uint8_t v4_smem_raw[];
  T* sV = reinterpret_cast<T*>(align128(v4_smem_raw));
  uint8_t* sVt = reinterpret_cast<uint8_t*>(sV);  // [D][64] code bytes, over the consumed tile
  __shared__ __align__(16) uint8_t s_sf[1024];
  __shared__ uint64_t bar;
  const int bg = blockIdx.y, tile = blockIdx.x;
  const int64_t r0 = (int64_t)tile * kTile;
  if (!load_tile<T, D>(sV, &tmV, &bar, (int)r0, bg, a.Hkv, a.nhd)) return;  // rows past N are zero
  uint2 codes[IT];
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int item = threadIdx.x + it * kThreads;
    const int c = item % D, grp = item / D;
    float x[16];
    float am = 0.0f;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      x[u] = to_float(sV[(grp * 16 + u) * D + c]);
      am = fmaxf(am, fabsf(x[u]));
    }
    const uint32_t sc = cvt_e4m3(__fdiv_rn(am, 6.0f));
    const float sd = e4m3_value(sc);
    float lo[8], hi[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      lo[u] = x[u];
      hi[u] = x[8 + u];
    }
    const float rd = sd == 0.0f ? 0.0f : __frcp_rn(sd);
    codes[it] = sd == 0.0f ? make_uint2(0u, 0u) : make_uint2(quant_e2m1x8(lo, sd, rd), quant_e2m1x8(hi, sd, rd));
    s_sf[sf_byte(c, grp)] = (uint8_t)sc;
  }
  __syncthreads();  // every thread has read the tile
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int item = threadIdx.x + it * kThreads;
    const int c = item % D, grp = item / D;
    *reinterpret_cast<uint2*>(sVt + c * (kTile / 2) + grp * 8) = codes[it];
  }
  __syncthreads();
  uint8_t* v4t = a.v4t + (int64_t)bg * D * (a.Np / 2) + r0 / 2;
#pragma unroll
  for (int it = 0; it < (D * kTile / 2 / 16) / kThreads; ++it) {
    const int idx = threadIdx.x + it * kThreads;  // 16-byte chunk
    const int c = idx / 4, q = idx % 4;
    *reinterpret_cast<uint4*>(v4t + (int64_t)c * (a.Np / 2) + q * 16) =
        *reinterpret_cast<const uint4*>(sVt + c * (kTile / 2) + q * 16);
  }
  reinterpret_cast<uint32_t*>(a.sfv + ((int64_t)bg * (a.Np / kTile) + tile) * 1024)[threadIdx.x] =
      reinterpret_cast<const uint32_t*>(s_sf)[threadIdx.x];
}

using KNvfp4Fn = void (*)(CUtensorMap, QuantArgs);

// The one-read K kernel, or nullptr if one head's `tiles` CTAs might not fit
// in half of the CTAs resident at once (then statistics + K kernels run).
template <typename T>
KNvfp4Fn k_fused_nvfp4_for(const QuantArgs& a, int tiles, int smem) {
  KNvfp4Fn kf = a.smooth_k ? k_fused_nvfp4_kernel<T, true> : k_fused_nvfp4_kernel<T, false>;
  if (cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return nullptr;
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kf, kThreads, smem) != cudaSuccess)
    return nullptr;
  return (a.force_one_read || (int64_t)tiles * 2 <= (int64_t)sms * per_sm) ? kf : nullptr;
}

template <typename T>
int quant_nvfp4_kernel_count_t(const QuantArgs& a, bool allow_one_read) {
  const int tiles = (int)(a.Np / kTile);
  const bool one_read = allow_one_read && k_fused_nvfp4_for<T>(a, tiles, kTile * kF4D * (int)sizeof(T) + 128);
  return (one_read ? 1 : 2) + 2 + (a.smooth_q ? 1 : 0);
}

template <typename T>
cudaError_t launch_quant_nvfp4_t(const QuantArgs& a, const QuantMaps& m, cudaStream_t st) {
  cudaError_t e;
  const int BHkv = a.B * a.Hkv, BHq = a.B * a.Hq;
  const int tiles = (int)(a.Np / kTile);
  const int smem = kTile * kF4D * (int)sizeof(T) + 128;
  QuantArgs s = a;
  s.vamax = nullptr;  // no per-channel V statistics on this path
  auto kf = a.kv_sync ? k_fused_nvfp4_for<T>(a, tiles, smem) : nullptr;
  if (kf) {
    // ksum and kv_sync are consecutive in the workspace: one memset
    e = cudaMemsetAsync(a.ksum, 0, a.kv_zero_bytes, st);
    if (e != cudaSuccess) return e;
    kf<<<dim3(tiles * BHkv), kThreads, smem, st>>>(m.k, s);
  } else {
    if (a.smooth_k) {
      e = cudaMemsetAsync(a.ksum, 0, sizeof(double) * (size_t)BHkv * kF4D, st);
      if (e != cudaSuccess) return e;
    }
    kv_stats_kernel<T, kF4D><<<dim3((a.N + kStatRows - 1) / kStatRows, BHkv), kThreads, 0, st>>>(s);
    k_quant_nvfp4_kernel<T><<<dim3(tiles, BHkv), kThreads, 0, st>>>(s);
  }
  e = cudaFuncSetAttribute(v_quant_nvfp4_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  v_quant_nvfp4_kernel<T><<<dim3(tiles, BHkv), kThreads, smem, st>>>(m.v, s);
  {
    auto qq = a.bq == 64 ? (a.smooth_q ? q_quant_nvfp4_kernel<T, 64, true> : q_quant_nvfp4_kernel<T, 64, false>)
                         : (a.smooth_q ? q_quant_nvfp4_kernel<T, 128, true> : q_quant_nvfp4_kernel<T, 128, false>);
    e = cudaFuncSetAttribute(qq, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    qq<<<dim3(tiles, BHq), kThreads, smem, st>>>(m.q, s);
  }
  if (a.smooth_q) {
    e = launch_delta_s<T, kF4D>(s, st);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quant_nvfp4(const QuantArgs& a, const QuantMaps& m, int is_fp16, cudaStream_t st) {
  if (a.D != kF4D) return cudaErrorInvalidValue;
  return is_fp16 ? launch_quant_nvfp4_t<__half>(a, m, st) : launch_quant_nvfp4_t<__nv_bfloat16>(a, m, st);
}

int quant_nvfp4_kernel_count(const QuantArgs& a, int is_fp16, bool allow_one_read) {
  return is_fp16 ? quant_nvfp4_kernel_count_t<__half>(a, allow_one_read)
                 : quant_nvfp4_kernel_count_t<__nv_bfloat16>(a, allow_one_read);
}

}  // namespace sage
