// libsage.cu -- single translation unit for the library (the device-side
// error word and wait limit are shared by all kernels without relocatable
// device code).
#include "quant.cu"
#include "attn_i8f8.cu"
#include "quant_nvfp4.cu"
#include "attn_nvfp4.cu"
#include "peak.cu"
#include "api.cu"
#include "noalloc.cu"
