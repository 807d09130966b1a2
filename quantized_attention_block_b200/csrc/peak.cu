// peak.cu -- tensor-core rate probe: every CTA (one per SM) issues back-to-back
// tcgen05.mma instructions of one kind on operand tiles that stay resident in
// shared memory, so the tensor pipe never waits for data.  The achieved rate
// is the measured peak of that kind on this GPU at the clocks of the run: the
// denominator of the attention kernels' roofline.
//   kind 0: kind::i8      (s8 x s8 -> s32),     M = 128, N = 64/128/256, K = 32 per instruction
//   kind 1: kind::f8f6f4  (E4M3 x E4M3 -> f32), M = 128, N = 64/128/256, K = 32
//   kind 2: kind::mxf4nvf4.block_scale.block16 (E2M1 x E2M1, UE4M3 scale per
//           16 elements -> f32), M = 128, N = 128, K = 64
// All instructions of a CTA accumulate into one TMEM accumulator (a GEMM's K
// loop); the values are pseudo-random and finite.
#include "sm100.cuh"

namespace sage {

namespace {

constexpr int kRateThreads = 128;

template <int KIND, int N>
__global__ void __launch_bounds__(kRateThreads, 1) mma_rate_kernel(int iters) {
  // i8 / f8: A [128][128 B], B [N][128 B], 128-byte swizzle (4 MMAs of K = 32 bytes per pass)
  // f4:      A [128][64 B],  B [128][64 B], 64-byte swizzle (2 MMAs of K = 64 elements per pass)
  constexpr bool kF4 = KIND == 2;
  constexpr uint32_t kRowBytes = kF4 ? 64 : 128;
  constexpr uint32_t kA = 128 * kRowBytes, kB = N * kRowBytes;
  constexpr uint32_t kSwz = kF4 ? kSwizzle64B : kSwizzle128B;
  constexpr uint32_t kSbo = 8 * kRowBytes;
  constexpr int kSteps = kF4 ? 2 : 4;
  constexpr uint32_t kIdesc = kF4 ? make_idesc_nvf4(128, N)
                                  : (KIND == 0 ? make_idesc(/*S32*/ 2, /*s8*/ 1, /*s8*/ 1, 128, N)
                                               : make_idesc(/*F32*/ 1, /*E4M3*/ 0, /*E4M3*/ 0, 128, N));
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sA = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = sA + kA;
  uint8_t* sSF = sB + kB;  // f4: 2 x 512-byte scale blocks (A and B share them)
  uint64_t* bar = reinterpret_cast<uint64_t*>(sSF + 1024);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
  const int t = threadIdx.x, warp = t / 32;

  // pseudo-random operand bytes (a 32-bit LCG per thread); E4M3 bytes keep
  // their exponent below 15 so every value is finite
  uint32_t x = 2654435761u * (uint32_t)(blockIdx.x * kRateThreads + t + 1);
  for (uint32_t i = t * 4; i < kA + kB; i += kRateThreads * 4) {
    x = x * 1664525u + 1013904223u;
    uint32_t w = x;
    if (KIND == 1) w &= 0xF7F7F7F7u;
    *reinterpret_cast<uint32_t*>(sA + i) = w;
  }
  if (kF4)
    for (uint32_t i = t * 4; i < 1024; i += kRateThreads * 4) *reinterpret_cast<uint32_t*>(sSF + i) = 0x38383838u;
  fence_proxy_async_smem();
  if (t == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (t == 0) {
    const uint32_t aA = smem_u32(sA), aB = smem_u32(sB);
    if (kF4) {
      // scale factors of A and B (4 TMEM columns per K step each)
      for (int kk = 0; kk < 2; ++kk) {
        tmem_cp_sf(tmem + 256 + 4 * kk, make_sdesc(smem_u32(sSF + kk * 512), 128, kSwizzleNone));
        tmem_cp_sf(tmem + 264 + 4 * kk, make_sdesc(smem_u32(sSF + kk * 512), 128, kSwizzleNone));
      }
    }
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int kk = 0; kk < kSteps; ++kk) {
        const uint64_t da = make_sdesc(aA + kk * 32, kSbo, kSwz), db = make_sdesc(aB + kk * 32, kSbo, kSwz);
        const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
        if (KIND == 0) mma_i8(tmem, da, db, kIdesc, acc);
        else if (KIND == 1) mma_f8f6f4(tmem, da, db, kIdesc, acc);
        else mma_nvf4(tmem, da, db, kIdesc, tmem + 256 + 4 * kk, tmem + 264 + 4 * kk, acc);
      }
    }
    mma_commit(bar);
  }
  __syncwarp();
  mbar_wait_warp(bar, 0);  // bounded; a timeout is recorded for sage_last_device_error
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int KIND, int N>
cudaError_t launch_rate(int iters, int ctas, cudaStream_t st) {
  constexpr uint32_t kRow = KIND == 2 ? 64 : 128;
  const int smem = (int)(128 * kRow + N * kRow + 1024 + 64 + 1024);
  cudaError_t e = cudaFuncSetAttribute(mma_rate_kernel<KIND, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  mma_rate_kernel<KIND, N><<<ctas, kRateThreads, smem, st>>>(iters);
  return cudaGetLastError();
}

}  // namespace

// ops (2 M N K per instruction) of one launch, or 0 for an unsupported (kind, n)
double mma_rate_ops(int kind, int n, int iters, int ctas) {
  if (kind == 2) return n == 128 ? 2.0 * 128 * 128 * 128 * (double)iters * ctas : 0.0;
  if (kind != 0 && kind != 1) return 0.0;
  if (n != 64 && n != 128 && n != 256) return 0.0;
  return 2.0 * 128 * n * 128 * (double)iters * ctas;
}

cudaError_t launch_mma_rate(int kind, int n, int iters, int ctas, cudaStream_t st) {
  if (kind == 0) {
    if (n == 64) return launch_rate<0, 64>(iters, ctas, st);
    if (n == 128) return launch_rate<0, 128>(iters, ctas, st);
    if (n == 256) return launch_rate<0, 256>(iters, ctas, st);
  } else if (kind == 1) {
    if (n == 64) return launch_rate<1, 64>(iters, ctas, st);
    if (n == 128) return launch_rate<1, 128>(iters, ctas, st);
    if (n == 256) return launch_rate<1, 256>(iters, ctas, st);
  } else if (kind == 2 && n == 128) {
    return launch_rate<2, 128>(iters, ctas, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace sage
