// api.cu -- the extern "C" entry points declared in include/sage.h: argument
// validation, workspace layout, TMA tensor maps, kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "sage.h"
#include "sm100.cuh"

namespace {

using namespace sage;

constexpr size_t kAlign = 1024;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Dims {
  int64_t B, Hq, Hkv, N, D, Np, Tm, Tn;
};

struct Layout {
  size_t q8, k8, v8t, s_q, s_k, s_v, km, qkm, ksum, vamax, kv_sync, kv_sync_end, qbar, dS, total;
};

// K/V path of sage_quant_qkv / sage_quant_nvfp4 (sage_debug_kv_quant_two_pass):
// 0: the default choice; 1: always two passes; 2: one read even when a group's
// tiles may not all be resident at once (a test of the bounded group waits)
int g_kv_two_pass = 0;

sage_status check_params(const sage_params* p, Dims* d) {
  if (!p) return SAGE_ERR_INVALID_ARG;
  if (p->B < 1 || p->Hq < 1 || p->Hkv < 1 || p->N < 1) return SAGE_ERR_INVALID_ARG;
  if (p->Hq % p->Hkv != 0) return SAGE_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return SAGE_ERR_UNSUPPORTED_HEADDIM;
  if (p->dtype != SAGE_BF16 && p->dtype != SAGE_FP16) return SAGE_ERR_UNSUPPORTED_DTYPE;
  if ((p->bq != 32 && p->bq != 64 && p->bq != 128) || (p->bk != 64 && p->bk != 128)) return SAGE_ERR_INVALID_ARG;
  if ((p->causal != 0 && p->causal != 1) || (p->smooth_k != 0 && p->smooth_k != 1) ||
      (p->smooth_q != 0 && p->smooth_q != 1))
    return SAGE_ERR_INVALID_ARG;
  if (std::isnan(p->sm_scale) || std::isinf(p->sm_scale)) return SAGE_ERR_INVALID_ARG;
  if (p->pv_accum != SAGE_PV_TWO_LEVEL && p->pv_accum != SAGE_PV_TMEM_FP32) return SAGE_ERR_INVALID_ARG;
  if (p->return_lse != 0 && p->return_lse != 1) return SAGE_ERR_INVALID_ARG;
  if (p->layout != SAGE_HND && p->layout != SAGE_NHD) return SAGE_ERR_INVALID_ARG;
  d->B = p->B;
  d->Hq = p->Hq;
  d->Hkv = p->Hkv;
  d->N = p->N;
  d->D = p->d;
  d->Np = (d->N + kTile - 1) / kTile * kTile;
  d->Tm = (d->N + p->bq - 1) / p->bq;
  d->Tn = (d->N + p->bk - 1) / p->bk;
  // TMA row coordinates are int32
  if (d->B * d->Hq * d->Np >= (int64_t(1) << 31) || d->B * d->Hkv * d->D >= (int64_t(1) << 31))
    return SAGE_ERR_INVALID_ARG;
  return SAGE_OK;
}

Layout make_layout(const sage_params* p, const Dims& d) {
  Layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, kAlign);
    return o;
  };
  L.q8 = take((size_t)(d.B * d.Hq * d.Np * d.D));
  L.k8 = take((size_t)(d.B * d.Hkv * d.Np * d.D));
  L.v8t = take((size_t)(d.B * d.Hkv * d.D * d.Np));
  L.s_q = take(4 * (size_t)(d.B * d.Hq * d.Tm));
  L.s_k = take(4 * (size_t)(d.B * d.Hkv * d.Tn));
  L.s_v = take(4 * (size_t)(d.B * d.Hkv * d.D));
  L.km = take(4 * (size_t)(d.B * d.Hkv * d.D));
  L.qkm = take(4 * (size_t)(d.B * d.Hq * d.Np));
  // ksum, vamax, kv_sync consecutive: the one-read K/V kernel zeroes them with one memset
  L.ksum = take(8 * (size_t)(d.B * d.Hkv * d.D));
  L.vamax = take(4 * (size_t)(d.B * d.Hkv * d.D));
  L.kv_sync = take(4 * (size_t)(1 + 2 * d.B * d.Hkv));
  L.kv_sync_end = L.kv_sync + 4 * (size_t)(1 + 2 * d.B * d.Hkv);
  if (p->smooth_q) {
    L.qbar = take(4 * (size_t)(d.B * d.Hq * d.Tm * d.D));
    L.dS = take(4 * (size_t)(d.B * d.Hq * d.Tm * d.Np));
  }
  L.total = off;
  return L;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

sage_status check_arch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return SAGE_ERR_CUDA;
  return (major == 10 && minor == 0) ? SAGE_OK : SAGE_ERR_UNSUPPORTED_ARCH;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// 2D uint8 tensor map: `rows` rows of `cols` bytes (row pitch `cols`), box
// box_cols x box_rows, with the given swizzle.
bool map_2d_u8(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
               uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [B*H][N][D] bf16/fp16 input as a 3D tensor (box 1 x 128 x D, no swizzle):
// a tile that runs past N reads zeros.
// A caller's 16-bit input as a TMA tensor: HND [B, H, N, D] as 3D (D, N, B H);
// NHD [B, N, H, D] as 4D (D, N, H, B) with the layout in the strides.  Box
// D x 128 (x 1 (x 1)); the quantisers pass matching coordinates.
bool map_input(CUtensorMap* m, const void* base, uint64_t D, uint64_t N, uint64_t H, uint64_t B, int nhd) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {D, N, nhd ? H : B * H, B};
  const cuuint64_t strides[3] = {(nhd ? H * D : D) * 2, (nhd ? D : N * D) * 2, H * N * D * 2};
  const cuuint32_t box[4] = {(cuuint32_t)D, kTile, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, nhd ? 4 : 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The caller's 16-bit output as a TMA tensor for bulk stores: 4D (d, N, Hq, B)
// with the strides of either layout, box 64 columns x 32 rows, 128-byte swizzle.
bool map_output(CUtensorMap* m, void* base, const AttnArgs& a) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)a.D, (cuuint64_t)a.N, (cuuint64_t)a.Hq, (cuuint64_t)a.B};
  const cuuint64_t strides[3] = {(cuuint64_t)a.o_rs * 2, (cuuint64_t)a.o_hs * 2, (cuuint64_t)a.o_bs * 2};
  const cuuint32_t box[4] = {64, 32, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

sage_status fill_view(const sage_params* p, const Dims& d, void* ws, sage_quant_view* v) {
  const Layout L = make_layout(p, d);
  uint8_t* base = static_cast<uint8_t*>(ws);
  v->q8 = reinterpret_cast<int8_t*>(base + L.q8);
  v->k8 = reinterpret_cast<int8_t*>(base + L.k8);
  v->v8t = base + L.v8t;
  v->s_q = reinterpret_cast<float*>(base + L.s_q);
  v->s_k = reinterpret_cast<float*>(base + L.s_k);
  v->s_v = reinterpret_cast<float*>(base + L.s_v);
  v->km = reinterpret_cast<float*>(base + L.km);
  v->qbar = p->smooth_q ? reinterpret_cast<float*>(base + L.qbar) : nullptr;
  v->dS = p->smooth_q ? reinterpret_cast<float*>(base + L.dS) : nullptr;
  v->Np = d.Np;
  v->qkm = p->return_lse ? reinterpret_cast<float*>(base + L.qkm) : nullptr;
  return SAGE_OK;
}

sage_status make_maps(const sage_quant_view* v, const Dims& d, CUtensorMap* mQ, CUtensorMap* mK,
                      CUtensorMap* mV) {
  const CUtensorMapSwizzle swz = d.D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!map_2d_u8(mQ, v->q8, (uint64_t)d.D, (uint64_t)(d.B * d.Hq * d.Np), (uint32_t)d.D, kTile, swz))
    return SAGE_ERR_CUDA;
  if (!map_2d_u8(mK, v->k8, (uint64_t)d.D, (uint64_t)(d.B * d.Hkv * d.Np), (uint32_t)d.D, kTile, swz))
    return SAGE_ERR_CUDA;
  if (mV && !map_2d_u8(mV, v->v8t, (uint64_t)d.Np, (uint64_t)(d.B * d.Hkv * d.D), kTile, (uint32_t)d.D,
                       CU_TENSOR_MAP_SWIZZLE_128B))
    return SAGE_ERR_CUDA;
  return SAGE_OK;
}

// element strides of the caller's o [B, Hq, N, d] (HND) or [B, N, Hq, d] (NHD)
void set_out_strides(AttnArgs* a, const sage_params* p, const Dims& d) {
  const int64_t D = d.D, N = d.N, Hq = d.Hq;
  a->o_bs = Hq * N * D;
  a->o_hs = p->layout == SAGE_NHD ? D : N * D;
  a->o_rs = p->layout == SAGE_NHD ? Hq * D : D;
  a->nhd = p->layout == SAGE_NHD;
}

AttnArgs attn_args(const sage_quant_view* v, const sage_params* p, const Dims& d) {
  AttnArgs a{};
  a.B = (int)d.B;
  a.Hq = (int)d.Hq;
  a.Hkv = (int)d.Hkv;
  a.N = (int)d.N;
  a.D = (int)d.D;
  a.Np = d.Np;
  a.Tm = (int)d.Tm;
  a.Tn = (int)d.Tn;
  a.bq = p->bq;
  a.bk = p->bk;
  a.causal = p->causal;
  a.n_qtiles = (int)(d.Np / kTile);
  const float sm = p->sm_scale > 0.0f ? p->sm_scale : 1.0f / std::sqrt((float)d.D);
  a.scale_log2 = (float)((double)sm * 1.4426950408889634);
  a.sm_scale = sm;
  a.qkm = v->qkm;
  a.s_q = v->s_q;
  a.s_k = v->s_k;
  a.s_v = v->s_v;
  a.dS = p->smooth_q ? v->dS : nullptr;
  a.out_fp16 = p->dtype == SAGE_FP16;
  set_out_strides(&a, p, d);
  a.two_level = p->pv_accum == SAGE_PV_TWO_LEVEL;
  return a;
}

sage_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA; }

// ---------------------------------------------------------------- NVFP4 layout
struct LayoutF4 {
  size_t q4, k4, v4t, sfq, sfk, sfv, km, ksum, kv_sync, kv_sync_end, qbar, dS, total;
};

LayoutF4 make_layout_f4(const sage_params* p, const Dims& d) {
  LayoutF4 L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, kAlign);
    return o;
  };
  const size_t tiles = (size_t)(d.Np / kTile);
  L.q4 = take((size_t)(d.B * d.Hq * d.Np * d.D / 2));
  L.k4 = take((size_t)(d.B * d.Hkv * d.Np * d.D / 2));
  L.v4t = take((size_t)(d.B * d.Hkv * d.D * d.Np / 2));
  L.sfq = take((size_t)(d.B * d.Hq) * tiles * 1024);
  L.sfk = take((size_t)(d.B * d.Hkv) * tiles * 1024);
  L.sfv = take((size_t)(d.B * d.Hkv) * tiles * 1024);
  L.km = take(4 * (size_t)(d.B * d.Hkv * d.D));
  // ksum, kv_sync consecutive: the one-read K kernel zeroes them with one memset
  L.ksum = take(8 * (size_t)(d.B * d.Hkv * d.D));
  L.kv_sync = take(4 * (size_t)(1 + d.B * d.Hkv));
  L.kv_sync_end = L.kv_sync + 4 * (size_t)(1 + d.B * d.Hkv);
  if (p->smooth_q) {
    L.qbar = take(4 * (size_t)(d.B * d.Hq * d.Tm * d.D));
    L.dS = take(4 * (size_t)(d.B * d.Hq * d.Tm * d.Np));
  }
  L.total = off;
  return L;
}

sage_status check_params_f4(const sage_params* p, Dims* d) {
  const sage_status s = check_params(p, d);
  if (s != SAGE_OK) return s;
  if (p->bq == 32) return SAGE_ERR_INVALID_ARG;  // the NVFP4 smooth-Q block is 64 or 128 rows
  return d->D == 128 ? SAGE_OK : SAGE_ERR_UNSUPPORTED_HEADDIM;
}

void fill_view_f4(const sage_params* p, const Dims& d, void* ws, sage_nvfp4_view* v) {
  const LayoutF4 L = make_layout_f4(p, d);
  uint8_t* base = static_cast<uint8_t*>(ws);
  v->q4 = base + L.q4;
  v->k4 = base + L.k4;
  v->v4t = base + L.v4t;
  v->sfq = base + L.sfq;
  v->sfk = base + L.sfk;
  v->sfv = base + L.sfv;
  v->km = reinterpret_cast<float*>(base + L.km);
  v->qbar = p->smooth_q ? reinterpret_cast<float*>(base + L.qbar) : nullptr;
  v->dS = p->smooth_q ? reinterpret_cast<float*>(base + L.dS) : nullptr;
  v->Np = d.Np;
}

// Q / K: rows of 64 bytes (128 E2M1 codes); V^T: rows of Np/2 bytes.  Boxes
// of 64 bytes x 128 rows, 64-byte swizzle (the MMA's K-major SW64 layout).
sage_status make_maps_f4(const sage_nvfp4_view* v, const Dims& d, CUtensorMap* mQ, CUtensorMap* mK,
                         CUtensorMap* mV) {
  const CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_64B;
  if (!map_2d_u8(mQ, v->q4, 64, (uint64_t)(d.B * d.Hq * d.Np), 64, kTile, swz)) return SAGE_ERR_CUDA;
  if (!map_2d_u8(mK, v->k4, 64, (uint64_t)(d.B * d.Hkv * d.Np), 64, kTile, swz)) return SAGE_ERR_CUDA;
  if (mV && !map_2d_u8(mV, v->v4t, (uint64_t)(d.Np / 2), (uint64_t)(d.B * d.Hkv * d.D), 64, kTile, swz))
    return SAGE_ERR_CUDA;
  return SAGE_OK;
}

AttnArgs attn_args_f4(const sage_nvfp4_view* v, const sage_params* p, const Dims& d) {
  AttnArgs a{};
  a.B = (int)d.B;
  a.Hq = (int)d.Hq;
  a.Hkv = (int)d.Hkv;
  a.N = (int)d.N;
  a.D = (int)d.D;
  a.Np = d.Np;
  a.Tm = (int)d.Tm;
  a.Tn = (int)d.Tn;
  a.bq = p->bq;
  a.bk = p->bk;
  a.causal = p->causal;
  a.n_qtiles = (int)(d.Np / kTile);
  const float sm = p->sm_scale > 0.0f ? p->sm_scale : 1.0f / std::sqrt((float)d.D);
  a.scale_log2 = (float)((double)sm * 1.4426950408889634);
  a.dS = p->smooth_q ? v->dS : nullptr;
  a.out_fp16 = p->dtype == SAGE_FP16;
  set_out_strides(&a, p, d);
  a.sfq = v->sfq;
  a.sfk = v->sfk;
  a.sfv = v->sfv;
  return a;
}



}  // namespace

extern "C" {

size_t sage_workspace_bytes(const sage_params* p) {
  Dims d;
  if (check_params(p, &d) != SAGE_OK) return 0;
  return make_layout(p, d).total;
}

sage_status sage_quant_qkv(const void* q, const void* k, const void* v, const sage_params* p, void* workspace,
                           size_t workspace_bytes, sage_quant_view* view, void* stream) {
  Dims d;
  sage_status s = check_params(p, &d);
  if (s != SAGE_OK) return s;
  if (!q || !k || !v || !workspace || !view) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SAGE_ERR_MISALIGNED;
  const Layout L = make_layout(p, d);
  if (workspace_bytes < L.total) return SAGE_ERR_WORKSPACE_TOO_SMALL;
  if ((s = check_arch()) != SAGE_OK) return s;
  fill_view(p, d, workspace, view);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  QuantArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.B = (int)d.B;
  a.Hq = (int)d.Hq;
  a.Hkv = (int)d.Hkv;
  a.N = (int)d.N;
  a.D = (int)d.D;
  a.Np = d.Np;
  a.Tm = (int)d.Tm;
  a.Tn = (int)d.Tn;
  a.bq = p->bq;
  a.bk = p->bk;
  a.smooth_k = p->smooth_k;
  a.smooth_q = p->smooth_q;
  a.nhd = p->layout;
  a.q8 = view->q8;
  a.k8 = view->k8;
  a.v8t = view->v8t;
  a.s_q = view->s_q;
  a.s_k = view->s_k;
  a.s_v = view->s_v;
  a.km = view->km;
  a.qbar = view->qbar;
  a.dS = view->dS;
  a.qkm = view->qkm;
  a.ksum = reinterpret_cast<double*>(base + L.ksum);
  a.vamax = reinterpret_cast<unsigned*>(base + L.vamax);
  a.kv_sync = g_kv_two_pass == 1 ? nullptr : reinterpret_cast<int*>(base + L.kv_sync);
  a.force_one_read = g_kv_two_pass == 2;
  a.kv_zero_bytes = L.kv_sync_end - L.ksum;
  QuantMaps m;
  if (!map_2d_u8(&m.vt, view->v8t, (uint64_t)d.Np, (uint64_t)(d.B * d.Hkv * d.D), kTile, (uint32_t)d.D,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map_input(&m.q, q, (uint64_t)d.D, (uint64_t)d.N, (uint64_t)d.Hq, (uint64_t)d.B, p->layout) ||
      !map_input(&m.k, k, (uint64_t)d.D, (uint64_t)d.N, (uint64_t)d.Hkv, (uint64_t)d.B, p->layout) ||
      !map_input(&m.v, v, (uint64_t)d.D, (uint64_t)d.N, (uint64_t)d.Hkv, (uint64_t)d.B, p->layout))
    return SAGE_ERR_CUDA;
  return from_cuda(launch_quant(a, m, p->dtype == SAGE_FP16, static_cast<cudaStream_t>(stream)));
}

sage_status sage_attn_fwd_quantized(const sage_quant_view* view, void* o, const sage_params* p, void* stream) {
  return sage_attn_fwd_quantized_lse(view, o, nullptr, p, stream);
}

sage_status sage_attn_fwd_quantized_lse(const sage_quant_view* view, void* o, float* lse, const sage_params* p,
                                        void* stream) {
  Dims d;
  sage_status s = check_params(p, &d);
  if (s != SAGE_OK) return s;
  if (!view || !o || !view->q8 || !view->k8 || !view->v8t || !view->s_q || !view->s_k || !view->s_v)
    return SAGE_ERR_INVALID_ARG;
  if (p->smooth_q && !view->dS) return SAGE_ERR_INVALID_ARG;
  if (view->Np != d.Np) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(view->q8) || !aligned16(view->k8) || !aligned16(view->v8t))
    return SAGE_ERR_MISALIGNED;
  if ((s = check_arch()) != SAGE_OK) return s;
  CUtensorMap mQ, mK, mV;
  if ((s = make_maps(view, d, &mQ, &mK, &mV)) != SAGE_OK) return s;
  if (lse && (!view->qkm || (reinterpret_cast<uintptr_t>(lse) & 3u))) return SAGE_ERR_INVALID_ARG;
  AttnArgs a = attn_args(view, p, d);
  a.o = o;
  a.lse = lse;
  CUtensorMap mO;
  if (!map_output(&mO, o, a)) return SAGE_ERR_CUDA;
  return from_cuda(launch_attn_i8f8(a, mQ, mK, mV, mO, static_cast<cudaStream_t>(stream)));
}

sage_status sage_attn_fwd(const void* q, const void* k, const void* v, void* o, const sage_params* p,
                          void* workspace, size_t workspace_bytes, void* stream) {
  return sage_attn_fwd_lse(q, k, v, o, nullptr, p, workspace, workspace_bytes, stream);
}

sage_status sage_attn_fwd_lse(const void* q, const void* k, const void* v, void* o, float* lse,
                              const sage_params* p, void* workspace, size_t workspace_bytes, void* stream) {
  if (!p) return SAGE_ERR_INVALID_ARG;
  sage_params pl = *p;
  pl.return_lse = lse ? 1 : 0;
  sage_quant_view view;
  sage_status s = sage_quant_qkv(q, k, v, &pl, workspace, workspace_bytes, &view, stream);
  if (s != SAGE_OK) return s;
  return sage_attn_fwd_quantized_lse(&view, o, lse, &pl, stream);
}

sage_status sage_debug_qk_int32(const sage_quant_view* view, const sage_params* p, int32_t b, int32_t h,
                                int32_t qtile, int32_t ktile, int32_t* out, void* stream) {
  Dims d;
  sage_status s = check_params(p, &d);
  if (s != SAGE_OK) return s;
  if (!view || !out || !view->q8 || !view->k8) return SAGE_ERR_INVALID_ARG;
  if (b < 0 || b >= d.B || h < 0 || h >= d.Hq || qtile < 0 || ktile < 0 || qtile >= d.Np / kTile ||
      ktile >= d.Np / kTile)
    return SAGE_ERR_INVALID_ARG;
  if ((s = check_arch()) != SAGE_OK) return s;
  CUtensorMap mQ, mK;
  if ((s = make_maps(view, d, &mQ, &mK, nullptr)) != SAGE_OK) return s;
  AttnArgs a = attn_args(view, p, d);
  a.probe_b = b;
  a.probe_h = h;
  a.probe_qtile = qtile;
  a.probe_ktile = ktile;
  a.probe_out = out;
  return from_cuda(launch_qk_probe(a, mQ, mK, static_cast<cudaStream_t>(stream)));
}

size_t sage_nvfp4_workspace_bytes(const sage_params* p) {
  Dims d;
  if (check_params_f4(p, &d) != SAGE_OK) return 0;
  return make_layout_f4(p, d).total;
}

sage_status sage_quant_nvfp4(const void* q, const void* k, const void* v, const sage_params* p, void* workspace,
                             size_t workspace_bytes, sage_nvfp4_view* view, void* stream) {
  Dims d;
  sage_status s = check_params_f4(p, &d);
  if (s != SAGE_OK) return s;
  if (!q || !k || !v || !workspace || !view) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SAGE_ERR_MISALIGNED;
  const LayoutF4 L = make_layout_f4(p, d);
  if (workspace_bytes < L.total) return SAGE_ERR_WORKSPACE_TOO_SMALL;
  if ((s = check_arch()) != SAGE_OK) return s;
  fill_view_f4(p, d, workspace, view);
  QuantArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.B = (int)d.B;
  a.Hq = (int)d.Hq;
  a.Hkv = (int)d.Hkv;
  a.N = (int)d.N;
  a.D = (int)d.D;
  a.Np = d.Np;
  a.Tm = (int)d.Tm;
  a.Tn = (int)d.Tn;
  a.bq = p->bq;
  a.bk = p->bk;
  a.smooth_k = p->smooth_k;
  a.smooth_q = p->smooth_q;
  a.nhd = p->layout;
  a.km = view->km;
  a.qbar = view->qbar;
  a.dS = view->dS;
  a.ksum = reinterpret_cast<double*>(static_cast<uint8_t*>(workspace) + L.ksum);
  a.q4 = view->q4;
  a.k4 = view->k4;
  a.v4t = view->v4t;
  a.sfq = view->sfq;
  a.sfk = view->sfk;
  a.sfv = view->sfv;
  a.kv_sync = g_kv_two_pass == 1 ? nullptr : reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + L.kv_sync);
  a.force_one_read = g_kv_two_pass == 2;
  a.kv_zero_bytes = L.kv_sync_end - L.ksum;
  QuantMaps m;
  if (!map_input(&m.q, q, (uint64_t)d.D, (uint64_t)d.N, (uint64_t)d.Hq, (uint64_t)d.B, p->layout) ||
      !map_input(&m.k, k, (uint64_t)d.D, (uint64_t)d.N, (uint64_t)d.Hkv, (uint64_t)d.B, p->layout) ||
      !map_input(&m.v, v, (uint64_t)d.D, (uint64_t)d.N, (uint64_t)d.Hkv, (uint64_t)d.B, p->layout))
    return SAGE_ERR_CUDA;
  m.vt = m.v;  // unused on this path
  return from_cuda(launch_quant_nvfp4(a, m, p->dtype == SAGE_FP16, static_cast<cudaStream_t>(stream)));
}

sage_status sage_attn_fwd_nvfp4_quantized(const sage_nvfp4_view* view, void* o, const sage_params* p,
                                          void* stream) {
  Dims d;
  sage_status s = check_params_f4(p, &d);
  if (s != SAGE_OK) return s;
  if (!view || !o || !view->q4 || !view->k4 || !view->v4t || !view->sfq || !view->sfk || !view->sfv)
    return SAGE_ERR_INVALID_ARG;
  if (p->smooth_q && !view->dS) return SAGE_ERR_INVALID_ARG;
  if (view->Np != d.Np) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(view->q4) || !aligned16(view->k4) || !aligned16(view->v4t) ||
      !aligned16(view->sfq) || !aligned16(view->sfk) || !aligned16(view->sfv))
    return SAGE_ERR_MISALIGNED;
  if ((s = check_arch()) != SAGE_OK) return s;
  CUtensorMap mQ, mK, mV;
  if ((s = make_maps_f4(view, d, &mQ, &mK, &mV)) != SAGE_OK) return s;
  AttnArgs a = attn_args_f4(view, p, d);
  a.o = o;
  return from_cuda(launch_attn_nvfp4(a, mQ, mK, mV, static_cast<cudaStream_t>(stream)));
}

sage_status sage_attn_fwd_nvfp4(const void* q, const void* k, const void* v, void* o, const sage_params* p,
                                void* workspace, size_t workspace_bytes, void* stream) {
  sage_nvfp4_view view;
  sage_status s = sage_quant_nvfp4(q, k, v, p, workspace, workspace_bytes, &view, stream);
  if (s != SAGE_OK) return s;
  return sage_attn_fwd_nvfp4_quantized(&view, o, p, stream);
}

sage_status sage_debug_qk_nvfp4(const sage_nvfp4_view* view, const sage_params* p, int32_t b, int32_t h,
                                int32_t qtile, int32_t ktile, float* out, void* stream) {
  Dims d;
  sage_status s = check_params_f4(p, &d);
  if (s != SAGE_OK) return s;
  if (!view || !out || !view->q4 || !view->k4 || !view->sfq || !view->sfk) return SAGE_ERR_INVALID_ARG;
  if (b < 0 || b >= d.B || h < 0 || h >= d.Hq || qtile < 0 || ktile < 0 || qtile >= d.Np / kTile ||
      ktile >= d.Np / kTile)
    return SAGE_ERR_INVALID_ARG;
  if ((s = check_arch()) != SAGE_OK) return s;
  CUtensorMap mQ, mK;
  if ((s = make_maps_f4(view, d, &mQ, &mK, nullptr)) != SAGE_OK) return s;
  AttnArgs a = attn_args_f4(view, p, d);
  a.probe_b = b;
  a.probe_h = h;
  a.probe_qtile = qtile;
  a.probe_ktile = ktile;
  return from_cuda(launch_qk_probe_nvfp4(a, mQ, mK, out, static_cast<cudaStream_t>(stream)));
}

sage_status sage_last_device_error(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int err = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&err, sage::g_device_error, sizeof(err), 0, cudaMemcpyDeviceToHost, st) !=
      cudaSuccess)
    return SAGE_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(sage::g_device_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st) !=
      cudaSuccess)
    return SAGE_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SAGE_ERR_CUDA;
  return err == 0 ? SAGE_OK : SAGE_ERR_TIMEOUT;
}

sage_status sage_debug_bounded_wait(uint32_t timeout_us, void* stream) {
  sage_status s = check_arch();
  if (s != SAGE_OK) return s;
  if (timeout_us == 0 || timeout_us > 10u * 1000u * 1000u) return SAGE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const unsigned long long limit = 1000ull * timeout_us, deflt = 4000000000ull;
  if (cudaMemcpyToSymbolAsync(sage::g_wait_limit_ns, &limit, sizeof(limit), 0, cudaMemcpyHostToDevice, st) !=
      cudaSuccess)
    return SAGE_ERR_CUDA;
  if (launch_bounded_wait_probe(st) != cudaSuccess) return SAGE_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(sage::g_wait_limit_ns, &deflt, sizeof(deflt), 0, cudaMemcpyHostToDevice, st) !=
      cudaSuccess)
    return SAGE_ERR_CUDA;
  return sage_last_device_error(stream);
}

sage_status sage_quant_kernel_count(const sage_params* p, int32_t* n) {
  Dims d;
  sage_status s = check_params(p, &d);
  if (s != SAGE_OK) return s;
  if (!n) return SAGE_ERR_INVALID_ARG;
  if ((s = check_arch()) != SAGE_OK) return s;
  QuantArgs a{};
  a.B = (int)d.B;
  a.Hq = (int)d.Hq;
  a.Hkv = (int)d.Hkv;
  a.N = (int)d.N;
  a.D = (int)d.D;
  a.Np = d.Np;
  a.Tm = (int)d.Tm;
  a.Tn = (int)d.Tn;
  a.bq = p->bq;
  a.bk = p->bk;
  a.smooth_k = p->smooth_k;
  a.smooth_q = p->smooth_q;
  a.force_one_read = g_kv_two_pass == 2;
  *n = quant_kernel_count(a, p->dtype == SAGE_FP16, g_kv_two_pass != 1);
  return SAGE_OK;
}

sage_status sage_quant_nvfp4_kernel_count(const sage_params* p, int32_t* n) {
  Dims d;
  sage_status s = check_params_f4(p, &d);
  if (s != SAGE_OK) return s;
  if (!n) return SAGE_ERR_INVALID_ARG;
  if ((s = check_arch()) != SAGE_OK) return s;
  QuantArgs a{};
  a.B = (int)d.B;
  a.Hq = (int)d.Hq;
  a.Hkv = (int)d.Hkv;
  a.N = (int)d.N;
  a.D = (int)d.D;
  a.Np = d.Np;
  a.Tm = (int)d.Tm;
  a.Tn = (int)d.Tn;
  a.bq = p->bq;
  a.bk = p->bk;
  a.smooth_k = p->smooth_k;
  a.smooth_q = p->smooth_q;
  a.force_one_read = g_kv_two_pass == 2;
  *n = quant_nvfp4_kernel_count(a, p->dtype == SAGE_FP16, g_kv_two_pass != 1);
  return SAGE_OK;
}

sage_status sage_debug_kv_quant_two_pass(int32_t on) {
  if (on < 0 || on > 2) return SAGE_ERR_INVALID_ARG;
  g_kv_two_pass = on;
  return SAGE_OK;
}

sage_status sage_debug_wait_limit(uint32_t timeout_us, void* stream) {
  if (timeout_us > 10u * 1000u * 1000u) return SAGE_ERR_INVALID_ARG;
  sage_status s = check_arch();
  if (s != SAGE_OK) return s;
  const unsigned long long limit = timeout_us ? 1000ull * timeout_us : 4000000000ull;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyToSymbolAsync(sage::g_wait_limit_ns, &limit, sizeof(limit), 0, cudaMemcpyHostToDevice, st) !=
      cudaSuccess)
    return SAGE_ERR_CUDA;
  return cudaStreamSynchronize(st) == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

sage_status sage_debug_exp2_poly(const float* x, float* y, int32_t n, void* stream) {
  if (!x || !y || n < 0) return SAGE_ERR_INVALID_ARG;
  if (n == 0) return SAGE_OK;
  sage_status s = check_arch();
  if (s != SAGE_OK) return s;
  return from_cuda(launch_exp2_poly_probe(x, y, n, static_cast<cudaStream_t>(stream)));
}

sage_status sage_debug_f8_accum_probe(float* out8, void* stream) {
  if (!out8 || !aligned16(out8)) return SAGE_ERR_INVALID_ARG;
  sage_status s = check_arch();
  if (s != SAGE_OK) return s;
  return from_cuda(launch_f8_accum_probe(out8, static_cast<cudaStream_t>(stream)));
}

sage_status sage_debug_mma_rate(int32_t kind, int32_t n, int32_t iters, int32_t ctas, double* ops, void* stream) {
  if (!ops || iters < 1 || iters > 2000000 || ctas < 0 || ctas > 4096) return SAGE_ERR_INVALID_ARG;
  if (mma_rate_ops(kind, n, 1, 1) == 0.0) return SAGE_ERR_INVALID_ARG;
  sage_status s = check_arch();
  if (s != SAGE_OK) return s;
  if (ctas == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&ctas, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return SAGE_ERR_CUDA;
  }
  *ops = mma_rate_ops(kind, n, iters, ctas);
  return from_cuda(launch_mma_rate(kind, n, iters, ctas, static_cast<cudaStream_t>(stream)));
}

const char* sage_status_string(sage_status s) {
  switch (s) {
    case SAGE_OK: return "SAGE_OK";
    case SAGE_ERR_INVALID_ARG: return "SAGE_ERR_INVALID_ARG";
    case SAGE_ERR_UNSUPPORTED_HEADDIM: return "SAGE_ERR_UNSUPPORTED_HEADDIM";
    case SAGE_ERR_UNSUPPORTED_DTYPE: return "SAGE_ERR_UNSUPPORTED_DTYPE";
    case SAGE_ERR_UNSUPPORTED_ARCH: return "SAGE_ERR_UNSUPPORTED_ARCH";
    case SAGE_ERR_WORKSPACE_TOO_SMALL: return "SAGE_ERR_WORKSPACE_TOO_SMALL";
    case SAGE_ERR_CUDA: return "SAGE_ERR_CUDA";
    case SAGE_ERR_TIMEOUT: return "SAGE_ERR_TIMEOUT";
    case SAGE_ERR_MISALIGNED: return "SAGE_ERR_MISALIGNED";
  }
  return "SAGE_ERR_UNKNOWN";
}

}  // extern "C"
