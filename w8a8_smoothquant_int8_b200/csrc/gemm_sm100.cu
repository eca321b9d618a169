// W8A8 GEMM with fused dequantization and multi-adapter LoRA delta, sm_100a.
//
// Computes, for a tile of 256 tokens x 256 output channels ("SmoothQuant"
// explainer, Step 7; "[Feature]: LoRA support for W8A8 SmoothQuant", Pitch):
//   acc   = Xq Wq^T                       int8 x int8 -> int32, tensor cores
//   base  = f32(acc) * x_scale_i * w_scale_n
//   Y     = bf16(base + T_hi Bp^T + T_lo Bp^T)   bf16 x bf16 -> fp32 on top
// with T = (x_scale * Xq) A_pack^T from the shrink kernel, stored as two bf16
// planes that are zero outside each token's adapter columns, so all adapters
// of a tile are applied by dense MMAs over the packed LoRA width.
//
// Structure: a pair of CTAs (a cluster of two, one per SM) shares each
// 256x256 tile through tcgen05.mma.cta_group::2: each CTA stages 128 token
// rows of Xq and 128 output-channel rows of Wq per K block, and each keeps the
// accumulator of its 128 token rows in its own tensor memory.  Persistent:
// one pair per two SMs walks the tiles.  Per CTA, 6 warps:
//   warp 0     TMA producer: Xq/Wq K blocks and LoRA chunks into a ring of
//              128-byte-swizzled shared-memory stages.  Completion of both
//              CTAs' copies is counted on the first CTA's barrier.
//   warp 1     allocates TMEM (two 256-column accumulator buffers); in the
//              first CTA of the pair its lane 0 issues every MMA of the pair.
//   warps 2-9  epilogue (two warps per TMEM lane quarter, 128 columns each).
//              A tile with LoRA rows is finished in two passes:
//              int32 -> base (fp32) rewritten in place in TMEM, then, after
//              the LoRA MMAs have accumulated onto it, fp32 -> bf16 -> global.
// The LoRA MMAs of tile i are issued half way through tile i+1, after the
// epilogue has converted tile i, so the tensor pipe does not wait for it.
// Every wait is bounded (mbar_wait); when one runs out, all roles stop,
// record SQ_ERR_DEVICE_TIMEOUT, wait for their own copies and MMAs, free
// TMEM and return.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx_sm100.cuh"
#include "tmap.cuh"

namespace sq {

constexpr int BM = 256;              // tokens per tile (pair MMA M; 128 per CTA)
constexpr int BN = 256;              // output channels per tile (MMA N; 128 staged per CTA)
constexpr int BK = 128;              // int8 K elements per stage (128 bytes)
constexpr int kHalf = 128;           // rows each CTA stages / owns
constexpr int kStages = 6;
constexpr int kABytes = kHalf * BK;  // 16 KB
constexpr int kBBytes = kHalf * BK;  // 16 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kLoraChunk = 64;       // bf16 columns of the LoRA width per stage
constexpr int kThreads = 320;        // producer warp, MMA warp, 8 epilogue warps
constexpr int kEpiWarps = 8;         // two per TMEM lane quarter, each owning 128 columns
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;  // two 256-column accumulator buffers
// Output staging of the bf16 epilogue: per epilogue warp two buffers of 32
// rows x 32 columns (64-byte swizzle), written to global by TMA stores.
constexpr int kEpiBufBytes = 32 * 32 * 2;
constexpr int kEpiSmem = kEpiWarps * 2 * kEpiBufBytes;  // 32 KB
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
  const unsigned long long *lora_mask;  // [ceil(M/16)] 16-column group masks, or null
  int num_mb, num_nb, num_tiles, group_m, num_pairs;
  // 0: groups of group_m token tiles walk the output-channel tiles; 1: groups
  // of group_m output-channel tiles walk the token tiles
  int raster_n;
  // operand kept in L2 across the walk (loaded with the evict-last policy):
  // 0 none, 2 Xq
  int keep;
  uint64_t timeout_ns;
};

struct SharedCtl {
  uint64_t full[kStages];    // first CTA: both CTAs' copies of a stage landed
  uint64_t empty[kStages];   // each CTA: the MMAs reading a stage finished
  uint64_t acc_full[2];      // each CTA: the int8 MMAs of a buffer finished
  uint64_t acc_empty[2];     // first CTA: both epilogues released a buffer
  uint64_t base_ready[2];    // first CTA: both epilogues rewrote a buffer as fp32
  uint64_t lora_done[2];     // each CTA: the LoRA MMAs of a buffer finished
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  uint32_t issued;           // stages this CTA's producer issued
  uint32_t peer_issued;      // first CTA: stages the second CTA's producer issued
};

static_assert(sizeof(SharedCtl) <= 1024, "control block fits its 1 KB slot");
// stages | control block (1 KB slot) | output staging | alignment slack
constexpr size_t kSmemBytes = static_cast<size_t>(kStages) * kStageBytes + 1024 + kEpiSmem + 1024;

__device__ __forceinline__ void tile_coords(int tile, const GemmArgs &a, int &mb, int &nb) {
  // groups of group_m tiles of one dimension walk the other dimension
  // together, so the pairs running at the same time share Xq rows and Wq
  // columns in L2; the walked operand is the one kept in L2 when it fits
  const int inner = a.raster_n ? a.num_mb : a.num_nb;
  const int outer = a.raster_n ? a.num_nb : a.num_mb;
  const int per_group = a.group_m * inner;
  const int g = tile / per_group;
  const int first = g * a.group_m;
  const int gsz = min(outer - first, a.group_m);
  const int local = tile - g * per_group;
  const int o = first + local % gsz, i = local / gsz;
  mb = a.raster_n ? i : o;
  nb = a.raster_n ? o : i;
}

// The 16-column groups of R that the tile's tokens use: the OR of the words
// of its groups of 16 tokens.
__device__ __forceinline__ unsigned long long tile_lora_mask(const GemmArgs &a, int mb) {
  if (a.lora_mask == nullptr || a.mode == kEpiAcc) return 0ull;
  const int g0 = mb * (BM / 16);
  const int ng = static_cast<int>((a.M + 15) / 16);
  unsigned long long m = 0ull;
#pragma unroll
  for (int g = 0; g < BM / 16; ++g)
    if (g0 + g < ng) m |= __ldg(a.lora_mask + g0 + g);
  return m;
}

// Scales of the columns col0 .. col0+31, the same in every lane (warp-uniform
// 16-byte loads; the columns past N read as 0).
__device__ __forceinline__ void load_wscale32(const float *__restrict__ w, int64_t col0, int64_t N,
                                              float (&ws)[32]) {
  if (col0 + 32 <= N) {
    const float4 *p = reinterpret_cast<const float4 *>(w + col0);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 t = __ldg(p + q);
      ws[4 * q] = t.x; ws[4 * q + 1] = t.y; ws[4 * q + 2] = t.z; ws[4 * q + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) ws[j] = (col0 + j < N) ? __ldg(w + col0 + j) : 0.f;
  }
}

// Dequantized values of 32 accumulators: RN(RN(float(acc) * xs) * w_j).
__device__ __forceinline__ void dequant32(uint32_t (&v)[32], float xs, const float (&ws)[32]) {
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    const float2 f = make_float2(__int2float_rn(static_cast<int>(v[j])),
                                 __int2float_rn(static_cast<int>(v[j + 1])));
    const float2 y = __fmul2_rn(__fmul2_rn(f, make_float2(xs, xs)), make_float2(ws[j], ws[j + 1]));
    v[j] = __float_as_uint(y.x);
    v[j + 1] = __float_as_uint(y.y);
  }
}

__device__ __forceinline__ void signal_abort(SharedCtl *ctl) {
  *reinterpret_cast<volatile int *>(&ctl->abort) = 1;
  record_device_error(SQ_ERR_DEVICE_TIMEOUT);
}

// The sequence of ring stages a pair consumes, identical for both producers
// and the MMA issuer:  for tile i = 0, 1, ...:
//   MAIN(i, kb) for kb < split;  LORA(i-1) chunks;  MAIN(i, kb) for kb >= split;
// and LORA(last) at the end, with split = nk/2 (the epilogue rewrites tile
// i-1 as fp32 during the first half of tile i; the LoRA MMAs follow).  LORA(t) = for every 64-column
// chunk of the LoRA width the tile uses, a T_hi stage and a T_lo stage.
// `f(kind, i, tile, a, b, first, last)` returns false to stop the walk.
enum ItemKind : int { kMain = 0, kLora = 1, kNoMain = 2 };

template <class F>
__device__ __forceinline__ bool walk_items(const GemmArgs &args, int pair, int nk, F &&f) {
  int i = 0, prev_tile = -1;
  auto lora_items = [&](int ti, int tile) -> bool {
    int mb, nb;
    tile_coords(tile, args, mb, nb);
    const unsigned long long mask = tile_lora_mask(args, mb);
    if (mask == 0ull) return true;
    int last_c = 0;
    for (int c = 0; c < SQ_MAX_LORA_COLS / kLoraChunk; ++c)
      if ((mask >> (4 * c)) & 0xFull) last_c = c;
    bool first = true;
    for (int c = 0; c < SQ_MAX_LORA_COLS / kLoraChunk; ++c) {
      if (((mask >> (4 * c)) & 0xFull) == 0) continue;
      for (int part = 0; part < 2; ++part) {
        if (!f(kLora, ti, tile, c, part, first, c == last_c && part == 1)) return false;
        first = false;
      }
    }
    return true;
  };
  for (int tile = pair; tile < args.num_tiles; tile += args.num_pairs, ++i) {
    const int split = (nk + 1) / 2;
    if (nk == 0 && !f(kNoMain, i, tile, 0, 0, true, true)) return false;
    for (int kb = 0; kb < split; ++kb)
      if (!f(kMain, i, tile, kb, 0, kb == 0, kb == nk - 1)) return false;
    if (prev_tile >= 0 && !lora_items(i - 1, prev_tile)) return false;
    for (int kb = split; kb < nk; ++kb)
      if (!f(kMain, i, tile, kb, 0, kb == 0, kb == nk - 1)) return false;
    prev_tile = tile;
  }
  if (prev_tile >= 0 && !lora_items(i - 1, prev_tile)) return false;
  return true;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    w8a8_lora_gemm_kernel(const __grid_constant__ CUtensorMap tm_xq,
                          const __grid_constant__ CUtensorMap tm_wq,
                          const __grid_constant__ CUtensorMap tm_thi,
                          const __grid_constant__ CUtensorMap tm_tlo,
                          const __grid_constant__ CUtensorMap tm_bp,
                          const __grid_constant__ CUtensorMap tm_y, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  SharedCtl *ctl = reinterpret_cast<SharedCtl *>(smem + kStages * kStageBytes);
  uint8_t *epi_smem = smem + kStages * kStageBytes + 1024;
  volatile int *abort_flag = &ctl->abort;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs of the pair
  const int pair = blockIdx.x >> 1;
  const bool use_lora = args.lora_mask != nullptr && args.mode != kEpiAcc;
  // the LoRA-only epilogue needs no int8 contraction
  const int nk = (args.mode == kEpiDelta) ? 0 : static_cast<int>((args.K + BK - 1) / BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->acc_full[b], 1);
      mbar_init(&ctl->acc_empty[b], 2 * kEpiThreads);
      mbar_init(&ctl->base_ready[b], 2 * kEpiThreads);
      mbar_init(&ctl->lora_done[b], 1);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    ctl->issued = 0;
    ctl->peer_issued = 0;
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
    tmem_alloc_pair(&ctl->tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive or copy
  tc_fence_after();
  // inputs written by the preceding kernels are read only from here on
  // (programmatic dependent launch: the set-up above may overlap their tail)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const uint32_t tmem = ctl->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const int row_off = static_cast<int>(rank) * kHalf;
      const uint64_t pol_keep = l2_policy_evict_last();
      bool ok = walk_items(args, pair, nk, [&](int kind, int, int tile, int a, int part, bool,
                                               bool) -> bool {
        if (kind == kNoMain) return true;
        if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, args.timeout_ns, abort_flag)) return false;
        int mb, nb;
        tile_coords(tile, args, mb, nb);
        uint8_t *a_dst = smem + stage * kStageBytes;
        uint64_t *full_local = &ctl->full[stage];
        const uint32_t full_pair = map_to_rank(smem_u32(full_local), 0);
        if (rank == 0) mbar_arrive_expect_tx(full_local, 2 * kStageBytes);
        if (kind == kMain) {
          if (args.keep == 2)
            tma_load_2d_pair_hint(a_dst, &tm_xq, full_pair, a * BK, mb * BM + row_off, pol_keep);
          else
            tma_load_2d_pair(a_dst, &tm_xq, full_pair, a * BK, mb * BM + row_off);
          tma_load_2d_pair(a_dst + kABytes, &tm_wq, full_pair, a * BK, nb * BN + row_off);
        } else {
          tma_load_2d_pair(a_dst, part ? &tm_tlo : &tm_thi, full_pair, a * kLoraChunk,
                           mb * BM + row_off);
          tma_load_2d_pair(a_dst + kABytes, &tm_bp, full_pair, a * kLoraChunk, nb * BN + row_off);
        }
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
        ++ctl->issued;
        return true;
      });
      if (!ok) signal_abort(ctl);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (rank == 0 && lane == 0) {
      const uint32_t idesc8 = idesc_i8_s32(BM, BN);
      const uint32_t idesc16 = idesc_bf16_f32(BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t lora_uses[2] = {0, 0};
      bool ok = walk_items(args, pair, nk, [&](int kind, int i, int tile, int a, int, bool first,
                                               bool last) -> bool {
        const int b = i & 1;
        const uint32_t dbuf = tmem + static_cast<uint32_t>(b) * 256u;
        if (kind != kLora && first) {
          // the buffer is free once both epilogues finished tile i-2
          if (!mbar_wait_cluster(&ctl->acc_empty[b], ((i >> 1) & 1) ^ 1u, args.timeout_ns,
                                 abort_flag))
            return false;
          tc_fence_after();
        }
        if (kind == kNoMain) {
          mma_commit_pair(&ctl->acc_full[b], 0x3);
          return true;
        }
        if (kind == kLora && first) {
          // the epilogues have rewritten the accumulator as fp32 base values
          if (!mbar_wait_cluster(&ctl->base_ready[b], lora_uses[b] & 1u, args.timeout_ns,
                                 abort_flag))
            return false;
          tc_fence_after();
        }
        if (!mbar_wait(&ctl->full[stage], phase, args.timeout_ns, abort_flag)) return false;
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + stage * kStageBytes);
        const uint32_t b_base = a_base + kABytes;
        if (kind == kMain) {
#pragma unroll
          for (int j = 0; j < BK / 32; ++j)
            mma_i8_pair(dbuf, sdesc_kmajor_sw128(a_base + 32 * j),
                        sdesc_kmajor_sw128(b_base + 32 * j), idesc8, (a | j) ? 1u : 0u);
        } else {
          int mb, nb;
          tile_coords(tile, args, mb, nb);
          const unsigned groups =
              static_cast<unsigned>((tile_lora_mask(args, mb) >> (4 * a)) & 0xFull);
#pragma unroll
          for (int g = 0; g < 4; ++g)
            if (groups & (1u << g))
              mma_f16_pair(dbuf, sdesc_kmajor_sw128(a_base + 32 * g),
                           sdesc_kmajor_sw128(b_base + 32 * g), idesc16, 1u);
        }
        mma_commit_pair(&ctl->empty[stage], 0x3);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
        if (kind == kMain && last) mma_commit_pair(&ctl->acc_full[b], 0x3);
        if (kind == kLora && last) {
          mma_commit_pair(&ctl->lora_done[b], 0x3);
          ++lora_uses[b];
        }
        return true;
      });
      if (!ok) signal_abort(ctl);
      // all MMAs issued by this thread must finish before TMEM is freed
      mma_commit(&ctl->drain);
      volatile int never = 0;
      mbar_wait(&ctl->drain, 0, kDrainNs, &never);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;               // epilogue warp 0..7
    const int quarter = warp & 3;          // TMEM lanes [32*quarter, 32*quarter+32)
    const int col_half = ew >> 2;          // columns [128*col_half, 128*col_half+128)
    const int row_in_tile = static_cast<int>(rank) * kHalf + quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t acc_empty_pair = map_to_rank(smem_u32(&ctl->acc_empty[0]), 0);
    const uint32_t base_ready_pair = map_to_rank(smem_u32(&ctl->base_ready[0]), 0);
    uint32_t lora_uses[2] = {0, 0};
    bool ok = true;
    int i = 0;
    int sbuf = 0;  // output staging buffer of this warp
    for (int tile = pair; tile < args.num_tiles; tile += args.num_pairs, ++i) {
      const int b = i & 1;
      const uint32_t dbuf = tmem + static_cast<uint32_t>(b) * 256u + lane_addr;
      int mb, nb;
      tile_coords(tile, args, mb, nb);
      const bool has_lora = use_lora && tile_lora_mask(args, mb) != 0ull;
      // the warp leaves together: the collective TMEM loads below need all lanes
      if (!(ok = __all_sync(0xffffffffu,
                            mbar_wait(&ctl->acc_full[b], (i >> 1) & 1, args.timeout_ns, abort_flag))))
        break;
      tc_fence_after();
      const int64_t row = static_cast<int64_t>(mb) * BM + row_in_tile;
      const bool row_ok = row < args.M;
      const float xs = (row_ok && args.mode == kEpiY) ? args.x_scale[row] : 0.f;
      if (has_lora) {
        // pass 1: base values rewritten in place as fp32
        for (int cc = 0; cc < 4; ++cc) {
          const int c = col_half * 4 + cc;
          uint32_t v[32];
          if (args.mode == kEpiY) {
            const int64_t col0 = static_cast<int64_t>(nb) * BN + c * 32;
            float ws[32];
            load_wscale32(args.w_scale, col0, args.N, ws);
            tmem_ld_32x32b_x32(dbuf + c * 32, v);
            tmem_ld_wait();
            dequant32(v, xs, ws);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0u;
          }
          tmem_st_32x32b_x32(dbuf + c * 32, v);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive_cluster(base_ready_pair + 8u * b);
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&ctl->lora_done[b], lora_uses[b] & 1u,
                                                      args.timeout_ns, abort_flag))))
          break;
        ++lora_uses[b];
        tc_fence_after();
      }
      // final pass: TMEM -> global
      for (int cc = 0; cc < 4; ++cc) {
        const int c = col_half * 4 + cc;
        const int64_t col0 = static_cast<int64_t>(nb) * BN + c * 32;
        if (col0 >= args.N) break;
        const int nvalid = (col0 + 32 <= args.N) ? 32 : static_cast<int>(args.N - col0);
        uint32_t v[32];
        const bool zero = (args.mode == kEpiDelta) && !has_lora;
        if (!zero) {
          tmem_ld_32x32b_x32(dbuf + c * 32, v);
          tmem_ld_wait();
        }
        if (args.mode == kEpiY) {
          if (!has_lora) {
            float ws[32];
            load_wscale32(args.w_scale, col0, args.N, ws);
            dequant32(v, xs, ws);
          }
          uint32_t packed[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(v[j]), __uint_as_float(v[j + 1]));
            packed[j / 2] = *reinterpret_cast<uint32_t *>(&h);
          }
          // stage the warp's 32 rows x 32 columns, then one TMA store (rows
          // past M and columns past N are clipped by the store)
          uint8_t *sb = epi_smem + (ew * 2 + sbuf) * kEpiBufBytes;
          if (lane == 0) bulk_wait_group_read<1>();  // this buffer's previous store has read it
          __syncwarp();
#pragma unroll
          for (int t = 0; t < 4; ++t)
            *reinterpret_cast<uint4 *>(sb + lane * 64 + ((t ^ ((lane >> 1) & 3)) * 16)) =
                make_uint4(packed[4 * t], packed[4 * t + 1], packed[4 * t + 2], packed[4 * t + 3]);
          fence_proxy_async_shared();
          __syncwarp();
          const int64_t row_base = static_cast<int64_t>(mb) * BM + rank * kHalf + quarter * 32;
          if (lane == 0 && row_base < args.M) {
            tma_store_2d(&tm_y, sb, static_cast<int32_t>(col0), static_cast<int32_t>(row_base));
            bulk_commit_group();
          }
          sbuf ^= 1;
        } else {
          if (!row_ok) continue;
          uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint32_t *>(args.out) + row * args.N + col0);
#pragma unroll
          for (int t = 0; t < 8; ++t)
            if (t * 4 < nvalid)
              dst[t] = zero ? make_uint4(0, 0, 0, 0)
                            : make_uint4(v[4 * t], v[4 * t + 1], v[4 * t + 2], v[4 * t + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive_cluster(acc_empty_pair + 8u * b);
    }
    if (!ok) signal_abort(ctl);
    if (lane == 0) bulk_wait_group<0>();  // this warp's output stores are complete
  }

  // Copies of both CTAs complete on the first CTA's `full` barriers, which
  // only that CTA can wait on.  After a wait that ran out the two producers
  // may have stopped at different stages (at most a ring apart): the first
  // CTA settles each stage that only one of them issued (complete-tx for the
  // copy that was announced but never made; expect-tx for a copy the second
  // CTA made unannounced) and then waits, bounded, for the last phase of every
  // slot, so that no copy is still in flight when either CTA leaves.  In a
  // run without a timeout the two counts agree and every wait returns at once.
  if (warp == 0 && lane == 0 && rank == 1)
    st_cluster_u32(map_to_rank(smem_u32(&ctl->peer_issued), 0), ctl->issued);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both producers have stopped; the second one's count is posted
  if (warp == 0 && lane == 0 && rank == 0) {
    const uint32_t mine = ctl->issued, theirs = ctl->peer_issued;
    const uint32_t hi = mine > theirs ? mine : theirs;
    const uint32_t lo = hi > static_cast<uint32_t>(kStages) ? hi - kStages : 0u;
    volatile int never = 0;
    for (uint32_t q = lo; q < hi; ++q) {
      uint64_t *bar = &ctl->full[q % kStages];
      const uint32_t par = (q / kStages) & 1u;
      if (q >= theirs) mbar_complete_tx(bar, kStageBytes);               // second CTA's share
      if (q >= mine) mbar_arrive_expect_tx(bar, kStageBytes);            // only its copy
      mbar_wait(bar, par, kDrainNs, &never);
    }
  }
  __syncthreads();
  cluster_sync();  // neither CTA leaves while its peer may still touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
// Launch the fused GEMM.  `lora` may be null (plain W8A8 / raw int32).
cudaError_t launch_w8a8_gemm(const int8_t *Xq, const int8_t *Wq, const float *x_scale,
                             const float *w_scale, int64_t M, int64_t N, int64_t K, int mode,
                             void *out, const LoraOperands *lora, cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  CUtensorMap tm_xq, tm_wq, tm_thi, tm_tlo, tm_bp, tm_y;
  memset(&tm_y, 0, sizeof tm_y);
  if (mode == kEpiY && !make_tmap(&tm_y, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, M, 32, 32,
                                  CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  memset(&tm_thi, 0, sizeof tm_thi);
  memset(&tm_tlo, 0, sizeof tm_tlo);
  memset(&tm_bp, 0, sizeof tm_bp);
  if (!make_tmap(&tm_xq, Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, M, BK, kHalf))
    return cudaErrorInvalidValue;
  if (mode == kEpiDelta)
    tm_wq = tm_xq;  // never loaded: the LoRA-only epilogue skips the int8 mainloop
  else if (!make_tmap(&tm_wq, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, N, BK, kHalf))
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
  if (lora && lora->R > 0 && mode != kEpiAcc) {
    if (!make_tmap(&tm_thi, lora->T_hi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, lora->R, M,
                   kLoraChunk, kHalf) ||
        !make_tmap(&tm_tlo, lora->T_lo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, lora->R, M,
                   kLoraChunk, kHalf) ||
        !make_tmap(&tm_bp, lora->B_pack, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, lora->R, N,
                   kLoraChunk, kHalf))
      return cudaErrorInvalidValue;
    a.lora_mask = lora->mask;
  }
  a.num_mb = static_cast<int>((M + BM - 1) / BM);
  a.num_nb = static_cast<int>((N + BN - 1) / BN);
  a.num_tiles = a.num_mb * a.num_nb;
  a.group_m = 4;
  // When all of Xq fits half the L2 and Wq does not, groups of
  // output-channel tiles walk all the token tiles and Xq is loaded with the
  // evict-last policy: Xq stays, Wq streams through once (measured at
  // 8192x4096x28672: DRAM reads 1085 -> 361 MB per launch, same time).
  // Otherwise groups of token tiles walk all output-channel tiles.  (Keeping
  // Wq the same way at 16384x14336x4096, or walking it in slabs of a
  // quarter of the L2, did not cut its re-reads and made the kernel slower.)
  {
    const double xq_bytes = static_cast<double>(M) * static_cast<double>(K);
    const double wq_bytes = static_cast<double>(N) * static_cast<double>(K);
    const double budget = 64.0 * 1024.0 * 1024.0;
    a.raster_n = 0;
    a.keep = 0;
    if (xq_bytes <= budget && wq_bytes > budget) {
      a.raster_n = 1;
      a.keep = 2;
    }
  }
  a.num_pairs = min(a.num_tiles, sm_count_of_current_device() / 2);
  a.timeout_ns = wait_timeout_ns();
  static std::atomic<int> attr_set[kMaxDevices];
  const cudaError_t e = ensure_smem_optin(w8a8_lora_gemm_kernel, static_cast<int>(kSmemBytes), attr_set);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * a.num_pairs, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, w8a8_lora_gemm_kernel, tm_xq, tm_wq, tm_thi, tm_tlo, tm_bp, tm_y, a);
}

}  // namespace sq
