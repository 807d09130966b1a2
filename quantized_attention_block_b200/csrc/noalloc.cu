// noalloc.cu -- sage_attn_fwd_noalloc: the whole forward with its scratch in
// a fixed, library-owned device array instead of a caller workspace.
//
// Some callers cannot obtain device memory at all: a plugin or custom-op
// interface that hands the library only its input and output pointers, or a
// process whose device memory is entirely owned by another allocator (a
// serving runtime with a fixed budget), where calling cudaMalloc is either
// not allowed or would synchronise the device in the middle of its work.
// For them this entry point takes only Q, K, V and O.  The scratch lives in
// `g_static_scratch` below; every GPU that loads this library reserves it
// until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "sage.h"

namespace {

// Scratch for quantised Q/K/V, scales, statistics and delta_S.
static __device__ __align__(256) uint8_t g_static_scratch[SAGE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device.  In host code
// the name g_static_scratch is only a host-side stand-in, so the address is
// looked up once per device (with that device current) and cached.
sage_status static_scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SAGE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return SAGE_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SAGE_OK;
}

}  // namespace

extern "C" SAGE_API sage_status sage_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o,
                                                      const sage_params* p, void* stream) {
  const size_t need = sage_workspace_bytes(p);
  if (need == 0) return SAGE_ERR_INVALID_ARG;
  if (need > (size_t)SAGE_STATIC_SCRATCH_BYTES) return SAGE_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  const sage_status s = static_scratch_address(&scratch);
  if (s != SAGE_OK) return s;
  // sage_quant_qkv zeroes the statistics accumulators it needs on every call
  // and overwrites every other byte of the scratch it uses (padding included),
  // so nothing left by the previous call leaks into this one.
  return sage_attn_fwd(q, k, v, o, p, scratch, (size_t)SAGE_STATIC_SCRATCH_BYTES, stream);
}
