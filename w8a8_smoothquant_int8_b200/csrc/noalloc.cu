// sq_linear_lora_noalloc: sq_linear_lora for callers that cannot allocate
// device memory.  Its scratch (the LoRA T planes and tile masks, or the
// small-M shrink partials) lives in one file-scope device array that every
// GPU loading this library holds until the process exits.
#include "common.cuh"

namespace sq {

// Scratch of sq_linear_lora_noalloc; SQ_NOALLOC_SCRATCH_BYTES (16 MiB).
static __device__ __align__(256) unsigned char g_noalloc_scratch[SQ_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on each device, looked up on the first
// call made with that device current.  In host code the array's name is only
// a host-side stand-in, never a device address.
static void *g_noalloc_scratch_addr[64] = {nullptr};

static int noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SQ_ERR_CUDA;
  if (dev < 0 || dev >= 64) return SQ_ERR_UNSUPPORTED_DEVICE;
  if (!g_noalloc_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return SQ_ERR_CUDA;
    g_noalloc_scratch_addr[dev] = p;
  }
  *out = g_noalloc_scratch_addr[dev];
  return SQ_OK;
}

}  // namespace sq

extern "C" int sq_linear_lora_noalloc(const int8_t *Xq, const float *x_scale, const int8_t *Wq,
                                      const float *w_scale, int64_t M, int64_t N, int64_t K,
                                      const uint16_t *A_pack, const uint16_t *B_pack,
                                      const int32_t *lora_offset, const int32_t *lora_rank,
                                      int n_adapters, int64_t R, const int32_t *seg_offsets,
                                      const int32_t *seg_adapter, int64_t S, uint16_t *Y,
                                      void *stream) {
  if (M < 0 || R < 0) return SQ_ERR_INVALID_ARG;
  if (sq_linear_lora_workspace_size(M, R) > SQ_NOALLOC_SCRATCH_BYTES) return SQ_ERR_WORKSPACE;
  int st = sq_device_supported_current();
  if (st) return st;
  void *scratch = nullptr;
  if ((st = sq::noalloc_scratch(&scratch))) return st;
  // every byte the kernels read from the scratch is written earlier in the
  // same call (the tile masks are cleared by the launch sequence itself)
  return sq_linear_lora(Xq, x_scale, Wq, w_scale, M, N, K, A_pack, B_pack, lora_offset, lora_rank,
                        n_adapters, R, seg_offsets, seg_adapter, S, Y, scratch,
                        SQ_NOALLOC_SCRATCH_BYTES, stream);
}
