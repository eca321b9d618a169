// Single translation unit of the CUDA library: the device-side error record
// (g_device_error) is one object shared by every kernel.
#include "quant.cu"
#include "lora_shrink.cu"
#include "gemm_sm100.cu"
#include "decode.cu"
#include "alpha_error.cu"
#include "api.cu"
#include "noalloc.cu"
