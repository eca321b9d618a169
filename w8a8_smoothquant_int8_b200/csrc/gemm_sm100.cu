// W8A8 GEMM with fused dequantization and multi-adapter LoRA delta, sm_100a.
//
// Computes, for a tile of 128 tokens x 256 output channels ("SmoothQuant"
// explainer, Step 7; "[Feature]: LoRA support for W8A8 SmoothQuant", Pitch):
//   acc   = Xq Wq^T                       int8 x int8 -> int32, tensor cores
//   delta = T_hi Bp^T + T_lo Bp^T         bf16 x bf16 -> fp32, tensor cores
//   Y     = bf16(f32(acc) * x_scale_i * w_scale_n + delta)
// with T = (x_scale * Xq) A_pack^T from the shrink kernel, stored as two bf16
// planes that are zero outside each token's adapter columns, so all adapters
// present in a tile are handled by dense MMAs over the packed width.
//
// Structure: persistent, one CTA per SM, 6 warps.
//   warp 0     TMA producer: Xq/Wq k-blocks (and LoRA chunks) into a ring of
//              shared-memory stages, 128-byte swizzled.
//   warp 1     owns TMEM (512 columns) and issues tcgen05.mma:
//              columns [0,256) int32 accumulator, [256,512) fp32 LoRA delta.
//   warps 2-5  epilogue: tcgen05.ld -> dequant + delta -> bf16 -> global.
// Every wait is bounded (see mbar_wait); a wait that runs out makes all roles
// stop, drain the copies and MMAs already issued, free TMEM and record
// SQ_ERR_DEVICE_TIMEOUT.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx_sm100.cuh"

namespace sq {

constexpr int BM = 128;              // tokens per tile (MMA M)
constexpr int BN = 256;              // output channels per tile (MMA N)
constexpr int BK = 128;              // int8 K elements per stage (128 bytes)
constexpr int kStages = 4;
constexpr int kABytes = BM * BK;     // 16 KB
constexpr int kBBytes = BN * BK;     // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kLoraChunk = 64;       // bf16 columns of the LoRA width per stage
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemAcc = 0;
constexpr uint32_t kTmemLora = 256;
// Bound of the final waits for this CTA's own copies and MMAs, independent of
// the (possibly tiny) user wait bound: those always complete.
constexpr uint64_t kDrainNs = 1000000000ull;

enum EpiMode : int { kEpiY = 0, kEpiAcc = 1, kEpiDelta = 2 };

struct GemmArgs {
  int64_t M, N, K;
  int mode;
  const float *x_scale;
  const float *w_scale;
  void *out;
  const unsigned long long *lora_mask;  // [num_mb] 16-column group masks, or null
  int num_mb, num_nb, num_tiles, group_m;
  uint64_t timeout_ns;
};

struct SharedCtl {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemBytes = static_cast<size_t>(kStages) * kStageBytes + sizeof(SharedCtl) + 1024;

__device__ __forceinline__ void tile_coords(int tile, const GemmArgs &a, int &mb, int &nb) {
  // groups of group_m token tiles walk the output-channel tiles together, so
  // the CTAs running at the same time share Xq rows and Wq columns in L2
  const int per_group = a.group_m * a.num_nb;
  const int g = tile / per_group;
  const int first = g * a.group_m;
  const int gm = min(a.num_mb - first, a.group_m);
  const int local = tile - g * per_group;
  mb = first + local % gm;
  nb = local / gm;
}

__device__ __forceinline__ void signal_abort(SharedCtl *ctl) {
  *reinterpret_cast<volatile int *>(&ctl->abort) = 1;
  record_device_error(SQ_ERR_DEVICE_TIMEOUT);
}

__global__ void __launch_bounds__(kThreads, 1)
    w8a8_lora_gemm_kernel(const __grid_constant__ CUtensorMap tm_xq,
                          const __grid_constant__ CUtensorMap tm_wq,
                          const __grid_constant__ CUtensorMap tm_thi,
                          const __grid_constant__ CUtensorMap tm_tlo,
                          const __grid_constant__ CUtensorMap tm_bp, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  SharedCtl *ctl = reinterpret_cast<SharedCtl *>(smem + kStages * kStageBytes);
  volatile int *abort_flag = &ctl->abort;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool use_lora = args.lora_mask != nullptr;
  // the LoRA-only epilogue needs no int8 contraction
  const int nk = (args.mode == kEpiDelta) ? 0 : static_cast<int>((args.K + BK - 1) / BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    mbar_init(&ctl->acc_full, 1);
    mbar_init(&ctl->acc_empty, 4 * 32);
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_xq);
    prefetch_tmap(&tm_wq);
    if (use_lora) {
      prefetch_tmap(&tm_thi);
      prefetch_tmap(&tm_tlo);
      prefetch_tmap(&tm_bp);
    }
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_parity = 0;  // per-stage bit sets
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < args.num_tiles; tile += gridDim.x) {
        int mb, nb;
        tile_coords(tile, args, mb, nb);
        const unsigned long long mask = use_lora ? args.lora_mask[mb] : 0ull;
        for (int c = 0; ok && c < SQ_MAX_LORA_COLS / kLoraChunk; ++c) {
          if (((mask >> (4 * c)) & 0xFull) == 0) continue;
          for (int part = 0; part < 2; ++part) {
            if (!(ok = mbar_wait(&ctl->empty[stage], phase ^ 1u, args.timeout_ns, abort_flag)))
              break;
            uint8_t *a_dst = smem + stage * kStageBytes;
            mbar_arrive_expect_tx(&ctl->full[stage], kStageBytes);
            tma_load_2d(a_dst, part ? &tm_tlo : &tm_thi, &ctl->full[stage], c * kLoraChunk,
                        mb * BM);
            tma_load_2d(a_dst + kABytes, &tm_bp, &ctl->full[stage], c * kLoraChunk, nb * BN);
            issued |= 1u << stage;
            issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
            if (++stage == kStages) { stage = 0; phase ^= 1u; }
          }
        }
        for (int kb = 0; ok && kb < nk; ++kb) {
          if (!(ok = mbar_wait(&ctl->empty[stage], phase ^ 1u, args.timeout_ns, abort_flag)))
            break;
          uint8_t *a_dst = smem + stage * kStageBytes;
          mbar_arrive_expect_tx(&ctl->full[stage], kStageBytes);
          tma_load_2d(a_dst, &tm_xq, &ctl->full[stage], kb * BK, mb * BM);
          tma_load_2d(a_dst + kABytes, &tm_wq, &ctl->full[stage], kb * BK, nb * BN);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) signal_abort(ctl);
      // every issued copy must land before the CTA exits
      volatile int never = 0;
      for (int s = 0; s < kStages; ++s)
        if (issued & (1u << s))
          mbar_wait(&ctl->full[s], (issued_parity >> s) & 1u, kDrainNs, &never);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t idesc8 = idesc_i8_s32(BM, BN);
      const uint32_t idesc16 = idesc_bf16_f32(BM, BN);
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < args.num_tiles; tile += gridDim.x) {
        int mb, nb;
        tile_coords(tile, args, mb, nb);
        const unsigned long long mask = use_lora ? args.lora_mask[mb] : 0ull;
        if (!(ok = mbar_wait(&ctl->acc_empty, acc_phase ^ 1u, args.timeout_ns, abort_flag))) break;
        tc_fence_after();
        uint32_t lora_acc = 0;
        for (int c = 0; ok && c < SQ_MAX_LORA_COLS / kLoraChunk; ++c) {
          const unsigned groups = static_cast<unsigned>((mask >> (4 * c)) & 0xFull);
          if (groups == 0) continue;
          for (int part = 0; part < 2; ++part) {
            if (!(ok = mbar_wait(&ctl->full[stage], phase, args.timeout_ns, abort_flag))) break;
            tc_fence_after();
            const uint32_t a_base = smem_u32(smem + stage * kStageBytes);
            const uint32_t b_base = a_base + kABytes;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              if (groups & (1u << g)) {
                mma_f16(tmem + kTmemLora, sdesc_kmajor_sw128(a_base + 32 * g),
                        sdesc_kmajor_sw128(b_base + 32 * g), idesc16, lora_acc);
                lora_acc = 1;
              }
            }
            mma_commit(&ctl->empty[stage]);
            if (++stage == kStages) { stage = 0; phase ^= 1u; }
          }
        }
        for (int kb = 0; ok && kb < nk; ++kb) {
          if (!(ok = mbar_wait(&ctl->full[stage], phase, args.timeout_ns, abort_flag))) break;
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + stage * kStageBytes);
          const uint32_t b_base = a_base + kABytes;
#pragma unroll
          for (int j = 0; j < BK / 32; ++j)
            mma_i8(tmem + kTmemAcc, sdesc_kmajor_sw128(a_base + 32 * j),
                   sdesc_kmajor_sw128(b_base + 32 * j), idesc8, (kb | j) ? 1u : 0u);
          mma_commit(&ctl->empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (ok) mma_commit(&ctl->acc_full);
        acc_phase ^= 1u;
      }
      if (!ok) signal_abort(ctl);
      // all MMAs issued by this thread must finish before TMEM is freed
      mma_commit(&ctl->drain);
      volatile int never = 0;
      mbar_wait(&ctl->drain, 0, kDrainNs, &never);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter+32)
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < args.num_tiles; tile += gridDim.x) {
      int mb, nb;
      tile_coords(tile, args, mb, nb);
      const bool has_lora = use_lora && args.lora_mask[mb] != 0ull;
      if (!(ok = mbar_wait(&ctl->acc_full, acc_phase, args.timeout_ns, abort_flag))) break;
      tc_fence_after();
      const int64_t row = static_cast<int64_t>(mb) * BM + row_in_tile;
      const bool row_ok = row < args.M;
      const float xs = (row_ok && args.mode == kEpiY) ? args.x_scale[row] : 0.f;
      for (int c = 0; c < BN / 32; ++c) {
        const int64_t col0 = static_cast<int64_t>(nb) * BN + c * 32;
        if (col0 >= args.N) break;
        const int nvalid = (col0 + 32 <= args.N) ? 32 : static_cast<int>(args.N - col0);
        uint32_t acc[32], dl[32];
        if (args.mode != kEpiDelta) tmem_ld_32x32b_x32(tmem + kTmemAcc + lane_addr + c * 32, acc);
        if (has_lora) tmem_ld_32x32b_x32(tmem + kTmemLora + lane_addr + c * 32, dl);
        tmem_ld_wait();
        if (!row_ok) continue;
        if (args.mode == kEpiY) {
          const float *ws = args.w_scale + col0;
          uint32_t packed[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            float v0 = 0.f, v1 = 0.f;
            if (j < nvalid) {
              v0 = __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(acc[j])), xs), __ldg(ws + j));
              v1 = __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(acc[j + 1])), xs),
                             __ldg(ws + j + 1));
              if (has_lora) {
                v0 = __fadd_rn(v0, __uint_as_float(dl[j]));
                v1 = __fadd_rn(v1, __uint_as_float(dl[j + 1]));
              }
            }
            __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
            packed[j / 2] = *reinterpret_cast<uint32_t *>(&h);
          }
          uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(args.out) + row * args.N + col0);
#pragma unroll
          for (int t = 0; t < 4; ++t)
            if (t * 8 < nvalid)
              dst[t] = make_uint4(packed[4 * t], packed[4 * t + 1], packed[4 * t + 2], packed[4 * t + 3]);
        } else if (args.mode == kEpiAcc) {
          uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint32_t *>(args.out) + row * args.N + col0);
#pragma unroll
          for (int t = 0; t < 8; ++t)
            if (t * 4 < nvalid)
              dst[t] = make_uint4(acc[4 * t], acc[4 * t + 1], acc[4 * t + 2], acc[4 * t + 3]);
        } else {
          uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint32_t *>(args.out) + row * args.N + col0);
#pragma unroll
          for (int t = 0; t < 8; ++t)
            if (t * 4 < nvalid)
              dst[t] = has_lora ? make_uint4(dl[4 * t], dl[4 * t + 1], dl[4 * t + 2], dl[4 * t + 3])
                                : make_uint4(0, 0, 0, 0);
        }
      }
      tc_fence_before();
      mbar_arrive(&ctl->acc_empty);
      acc_phase ^= 1u;
    }
    if (!ok) signal_abort(ctl);
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2D row-major tensor [outer, inner] of `esize`-byte elements, 128B swizzle.
static bool make_tmap(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int esize,
                      uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * static_cast<uint64_t>(esize)};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int sm_count_of_current_device() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 148;
  }
  return cached[dev];
}

// Launch the fused GEMM.  `lora` may be null (plain W8A8 / raw int32).
cudaError_t launch_w8a8_gemm(const int8_t *Xq, const int8_t *Wq, const float *x_scale,
                             const float *w_scale, int64_t M, int64_t N, int64_t K, int mode,
                             void *out, const LoraOperands *lora, cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  CUtensorMap tm_xq, tm_wq, tm_thi, tm_tlo, tm_bp;
  memset(&tm_thi, 0, sizeof tm_thi);
  memset(&tm_tlo, 0, sizeof tm_tlo);
  memset(&tm_bp, 0, sizeof tm_bp);
  if (!make_tmap(&tm_xq, Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, M, BK, BM))
    return cudaErrorInvalidValue;
  if (mode == kEpiDelta)
    tm_wq = tm_xq;  // never loaded: the LoRA-only epilogue skips the int8 mainloop
  else if (!make_tmap(&tm_wq, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, N, BK, BN))
    return cudaErrorInvalidValue;
  GemmArgs a;
  a.M = M;
  a.N = N;
  a.K = K;
  a.mode = mode;
  a.x_scale = x_scale;
  a.w_scale = w_scale;
  a.out = out;
  a.lora_mask = nullptr;
  if (lora && lora->R > 0) {
    if (!make_tmap(&tm_thi, lora->T_hi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, lora->R, M,
                   kLoraChunk, BM) ||
        !make_tmap(&tm_tlo, lora->T_lo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, lora->R, M,
                   kLoraChunk, BM) ||
        !make_tmap(&tm_bp, lora->B_pack, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, lora->R, N,
                   kLoraChunk, BN))
      return cudaErrorInvalidValue;
    a.lora_mask = lora->mask;
  }
  a.num_mb = static_cast<int>((M + BM - 1) / BM);
  a.num_nb = static_cast<int>((N + BN - 1) / BN);
  a.num_tiles = a.num_mb * a.num_nb;
  a.group_m = 8;
  a.timeout_ns = wait_timeout_ns();
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(w8a8_lora_gemm_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int grid = min(a.num_tiles, sm_count_of_current_device());
  w8a8_lora_gemm_kernel<<<grid, kThreads, kSmemBytes, st>>>(tm_xq, tm_wq, tm_thi, tm_tlo, tm_bp, a);
  return cudaGetLastError();
}

}  // namespace sq
