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
#include <cudaTypedefs.h>

#include <mutex>

#include "sage.h"

namespace {

// Scratch for quantised Q/K/V, scales, statistics and delta_S.
static __device__ __align__(256) uint8_t g_static_scratch[SAGE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
struct ScratchEntry {
  void* addr;
  unsigned long long ctx_id;  // unique id of the context the address was looked up in (0: unknown)
};
ScratchEntry g_scratch[kMaxDevices] = {};

// Unique id of the current context (ids are never reused within a process,
// so a context re-created after cudaDeviceReset gets a new one); 0 if the
// driver does not report it.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_ctx = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 4000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_ctx = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_ctx || !get_id || get_ctx(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_static_scratch on the current device.  In host code
// the name g_static_scratch is only a host-side stand-in, so the address is
// looked up with the device current and cached per device, together with
// the id of the context it belongs to; a different context on that device
// (after cudaDeviceReset) gets a fresh lookup.
sage_status static_scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SAGE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchEntry& e = g_scratch[dev];
  if (e.addr == nullptr || e.ctx_id != current_context_id()) {
    // the lookup creates the device's context if it does not exist yet, so the
    // context id is read after it
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return SAGE_ERR_CUDA;
    e.addr = p;
    e.ctx_id = current_context_id();
  }
  *out = e.addr;
  return SAGE_OK;
}

}  // namespace

extern "C" SAGE_API sage_status sage_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o,
                                                      const sage_params* p, void* stream) {
  // the same argument checks, in the same order, as sage_attn_fwd
  Dims d;
  sage_status s = check_params(p, &d);
  if (s != SAGE_OK) return s;
  if (sage_workspace_bytes(p) > (size_t)SAGE_STATIC_SCRATCH_BYTES) return SAGE_ERR_WORKSPACE_TOO_SMALL;
  if ((s = check_arch()) != SAGE_OK) return s;
  void* scratch = nullptr;
  if ((s = static_scratch_address(&scratch)) != SAGE_OK) return s;
  // sage_quant_qkv zeroes the statistics accumulators it needs on every call
  // and overwrites every other byte of the scratch it uses (padding included),
  // so nothing left by the previous call leaks into this one.
  return sage_attn_fwd(q, k, v, o, p, scratch, (size_t)SAGE_STATIC_SCRATCH_BYTES, stream);
}
