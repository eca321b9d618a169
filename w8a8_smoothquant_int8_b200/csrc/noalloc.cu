// sq_linear_lora_noalloc: sq_linear_lora for callers that cannot allocate
// device memory.  Its scratch (the LoRA T planes and tile masks, or the
// small-M shrink partials) lives in one file-scope device array that every
// GPU loading this library holds until the process exits.
#include "common.cuh"

namespace sq {

// Scratch of sq_linear_lora_noalloc; SQ_NOALLOC_SCRATCH_BYTES (16 MiB).
static __device__ __align__(256) unsigned char g_noalloc_scratch[SQ_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on each device, looked up on the first
// call made with that device current (std::atomic: host threads may call
// concurrently; two that find the slot empty store the same address).  In
// host code the array's name is only a host-side stand-in, never a device
// address.  After cudaDeviceReset of a device the cached address is stale:
// the library must not be used on that device again.
static std::atomic<void *> g_noalloc_scratch_addr[kMaxDevices];

static int noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SQ_ERR_UNSUPPORTED_DEVICE;
  void *p = g_noalloc_scratch_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return SQ_ERR_CUDA;
    g_noalloc_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
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
  // the scratch's address needs the library's module on this device
  int st = sq_device_supported_current();
  if (st) return st;
  void *scratch = nullptr;
  if ((st = sq::noalloc_scratch(&scratch))) return st;
  // sq_linear_lora checks everything else, the scratch's size as it checks a
  // caller's workspace (after the shapes, and only when an adapter is in
  // play).  Every byte the kernels read from the scratch is written earlier
  // in the same call (the tile masks are cleared by the launch sequence).
  return sq_linear_lora(Xq, x_scale, Wq, w_scale, M, N, K, A_pack, B_pack, lora_offset, lora_rank,
                        n_adapters, R, seg_offsets, seg_adapter, S, Y, scratch,
                        SQ_NOALLOC_SCRATCH_BYTES, stream);
}
