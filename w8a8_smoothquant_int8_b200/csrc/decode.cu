// Small-M (decode) form of the W8A8 + LoRA linear ("SmoothQuant" explainer,
// Step 7 and "Limitations": smaller gain at small batches, memory-bound;
// "[Feature]: LoRA support for W8A8 SmoothQuant", Pitch and Motivation: one
// adapter per request).  With a few dozen tokens the layer is bound by
// streaming Wq and the adapters from HBM, so the aim is to keep every SM
// pulling bytes from the first to the last microsecond:
//   kernel 1 (shrink)   one block per (token, K slice): the partial sums of
//                       T[i,:] = Xq[i,:] A_a^T over the slice, every A' row of
//                       the adapter requested at once; it lets the GEMM grid
//                       launch at once, so both stream side by side;
//   kernel 2 (GEMM + expand), CTA pairs (thread-block clusters of two): each
//                       pair owns a tile of up to 64 output channels and each
//                       CTA of the pair one half of K, so a CTA streams its
//                       half of the Wq tile and the matching half of Xq
//                       through a TMA ring once; acc = Xq Wq^T with int8
//                       tensor-core MMAs (m16n8k32, exact int32); the two
//                       halves are added through distributed shared memory;
//                       the B' rows of the CTA's output channels are
//                       bulk-copied into shared memory while the weights
//                       stream; after the shrink grid has completed
//                       (programmatic dependent launch), T = x_scale * (sum of
//                       the partials in a fixed order) and
//                       Y = bf16(acc*xs*ws + T B_a^T).
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx_sm100.cuh"
#include "tmap.cuh"

namespace sq {

constexpr int kDecMaxM = 64;            // token rows handled by this form
constexpr int kDecMaxRank = 256;        // largest adapter rank (the library-wide limit)
constexpr int kDecTable = 256;          // adapter table entries staged in shared memory
constexpr int kDecShrinkThreads = 256;
constexpr int kDecShrinkSplitMax = 8;   // K slices of the shrink, at most
constexpr int kDecShrinkSpan = 2048;    // K elements a shrink block covers per pass

__device__ __forceinline__ void group_bar(int id, int nthr) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthr) : "memory");
}

// ---------------------------------------------------------------------------
// Adapter of each token.  Token i belongs to the first segment s with
// seg_offsets[s] <= i < seg_offsets[s+1] and takes adapter seg_adapter[s]
// (-1: none).  Every segment is examined by one thread of the group, all in
// one round of loads, and the smallest covering s wins through a
// shared-memory minimum over (s, adapter) keys; the adapters' column offsets
// and ranks are staged in the same round when there are at most kDecTable of
// them.  Results for tokens [t0, t0 + nt): off[k], rank[k] (rank 0: no
// adapter; an index or an offset/rank out of range is recorded as
// SQ_ERR_BAD_SEGMENTS and the token gets no adapter).  `bar_id` names a
// barrier over the group's `nthr` threads.
// ---------------------------------------------------------------------------
struct DecodeTables {
  unsigned long long best[kDecMaxM];
  int ad_off[kDecTable];
  int ad_rank[kDecTable];
};

__device__ void decode_lookup(const int32_t *__restrict__ seg_offsets,
                              const int32_t *__restrict__ seg_adapter, int64_t S,
                              const int32_t *__restrict__ lora_offset,
                              const int32_t *__restrict__ lora_rank, int n_adapters, int64_t R,
                              int64_t t0, int nt, int tid, int nthr, int bar_id, DecodeTables &tb,
                              int *off_out, int *rank_out) {
  for (int k = tid; k < nt; k += nthr) tb.best[k] = ~0ull;
  const bool staged = n_adapters <= kDecTable;
  // the first pass of segments is loaded with the adapter tables, in one
  // round; more segments than threads take further rounds
  int32_t so0 = 0, so1 = 0, sa0 = 0;
  if (tid < S) {
    so0 = __ldg(seg_offsets + tid);
    so1 = __ldg(seg_offsets + tid + 1);
    sa0 = __ldg(seg_adapter + tid);
  }
  if (staged) {
    for (int a = tid; a < n_adapters; a += nthr) {
      tb.ad_off[a] = __ldg(lora_offset + a);
      tb.ad_rank[a] = __ldg(lora_rank + a);
    }
  }
  group_bar(bar_id, nthr);
  for (int64_t s = tid; s < S; s += nthr) {
    if (s != tid) {
      so0 = __ldg(seg_offsets + s);
      so1 = __ldg(seg_offsets + s + 1);
      sa0 = __ldg(seg_adapter + s);
    }
    const int64_t lo = max(static_cast<int64_t>(so0), t0);
    const int64_t hi = min(static_cast<int64_t>(so1), t0 + nt);
    if (lo < hi) {
      const unsigned long long key =
          (static_cast<unsigned long long>(s) << 32) | static_cast<uint32_t>(sa0);
      for (int64_t i = lo; i < hi; ++i) atomicMin(&tb.best[i - t0], key);
    }
  }
  group_bar(bar_id, nthr);
  for (int k = tid; k < nt; k += nthr) {
    const unsigned long long key = tb.best[k];
    int off = 0, r = 0;
    if (key != ~0ull) {
      const int a = static_cast<int>(static_cast<uint32_t>(key));
      if (a < -1 || a >= n_adapters) {
        record_device_error(SQ_ERR_BAD_SEGMENTS);
      } else if (a >= 0) {
        off = staged ? tb.ad_off[a] : __ldg(lora_offset + a);
        r = staged ? tb.ad_rank[a] : __ldg(lora_rank + a);
        if (off < 0 || (off & 15) || r <= 0 || r > kDecMaxRank || off + ((r + 15) & ~15) > R) {
          record_device_error(SQ_ERR_BAD_SEGMENTS);
          off = 0;
          r = 0;
        }
      }
    }
    off_out[k] = off;
    rank_out[k] = r;
  }
  group_bar(bar_id, nthr);
}

// ---------------------------------------------------------------------------
// kernel 1: shrink partials.  Block (i, ks) writes
//   part[(ks * M + i) * kDecMaxRank + j] = sum over its K slice of Xq[i,k] A'[off+j, k]
// for j < r (no x_scale: the GEMM applies it to the sum of the slices).
// Thread t covers 8 consecutive K elements per pass and loads the 16 A' rows
// of a rank group together (all of the block's 16 x 4 KB at once).
// ---------------------------------------------------------------------------
// At most 104 registers a thread: an SM's registers are split between its
// four sub-partitions (16K each) and a block's warps are dealt to them in
// turn, so a GEMM CTA (9 warps of 96 registers: 3 on one sub-partition) fits
// beside a shrink block (2 warps on each) only while 3*96 + 2*r <= 512.
__global__ void __maxnreg__(104) decode_shrink_kernel(
    const int8_t *__restrict__ Xq, int64_t M, int64_t K, int ksplit,
    const uint16_t *__restrict__ A_pack, const int32_t *__restrict__ lora_offset,
    const int32_t *__restrict__ lora_rank, int n_adapters, int64_t R,
    const int32_t *__restrict__ seg_offsets, const int32_t *__restrict__ seg_adapter, int64_t S,
    float *__restrict__ part) {
  // the dependent GEMM grid may launch at once: its weight stream needs
  // nothing from here, and it waits for this grid to complete before it
  // reads the partial sums
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ DecodeTables tb;
  __shared__ int s_off, s_rank;
  __shared__ float red[kDecShrinkThreads / 32][16];
  const int64_t i = blockIdx.x / ksplit;
  const int ks = static_cast<int>(blockIdx.x % ksplit);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  decode_lookup(seg_offsets, seg_adapter, S, lora_offset, lora_rank, n_adapters, R, i, 1, tid,
                kDecShrinkThreads, 1, tb, &s_off, &s_rank);
  const int off = s_off, r = s_rank;
  if (r == 0) return;  // block-uniform
  // the codes come from the quantizer (a no-op unless this grid is launched
  // as its programmatic dependent)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t span = ((K + ksplit - 1) / ksplit + 7) / 8 * 8;
  const int64_t k0 = ks * span, k1 = min(K, k0 + span);
  const int8_t *xrow = Xq + i * K;
  float *out = part + (static_cast<int64_t>(ks) * M + i) * kDecMaxRank;
  for (int j0 = 0; j0 < r; j0 += 16) {
    float acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.f;
    for (int64_t k = k0 + 8 * tid; k < k1; k += 8 * kDecShrinkThreads) {
      // rows off+j0 .. off+j0+15 exist (the pack pads every adapter to 16 rows)
      const uint2 xv = __ldg(reinterpret_cast<const uint2 *>(xrow + k));
      uint4 av[16];
#pragma unroll
      for (int j = 0; j < 16; ++j)
        av[j] = __ldg(reinterpret_cast<const uint4 *>(A_pack + (off + j0 + j) * K + k));
      float xf[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const uint32_t w = (t < 4) ? xv.x : xv.y;
        xf[t] = static_cast<float>(static_cast<int8_t>((w >> (8 * (t & 3))) & 0xff));
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint32_t a8[4] = {av[j].x, av[j].y, av[j].z, av[j].w};
        float s = acc[j];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          s = fmaf(xf[2 * t], __uint_as_float(a8[t] << 16), s);
          s = fmaf(xf[2 * t + 1], __uint_as_float(a8[t] & 0xffff0000u), s);
        }
        acc[j] = s;
      }
    }
    // sum over the warp by halving exchanges (a fixed order): after the
    // steps over lane bits 4..1 lane l holds rank (l >> 1) of the group
#pragma unroll
    for (int o = 16, n = 8; o >= 2; o >>= 1, n >>= 1) {
      const bool up = (lane & o) != 0;
#pragma unroll
      for (int m = 0; m < n; ++m) {
        const float send = up ? acc[m] : acc[m + n];
        const float keep = up ? acc[m + n] : acc[m];
        acc[m] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], 1);
    if ((lane & 1) == 0) red[warp][lane >> 1] = acc[0];
    __syncthreads();
    if (tid < 16 && j0 + tid < r) {
      float t = 0.f;
#pragma unroll
      for (int w = 0; w < kDecShrinkThreads / 32; ++w) t += red[w][tid];
      out[j0 + tid] = t;
    }
    __syncthreads();
  }
}


// ---------------------------------------------------------------------------
// kernel 2: int8 GEMM + LoRA expand on CTA pairs.
// A tile is `tile_units` groups of 8 output channels (at most 64 channels);
// tiles are dealt to the pairs in turn.  Per CTA and tile:
//   warp 8 (producer) streams the CTA's K half in stages of two 128-byte K
//     blocks: one TMA copy of the tile's Wq rows and one of the 64 Xq rows,
//     each a 3D box over the K blocks (two boxes per operand per stage when
//     K is not a multiple of 128), lanes 0 and 1 issuing together.  A copy
//     costs a few hundred ns to issue whatever its size, so the copies are
//     made large.  Before its first tile it also bulk-copies the B' rows of
//     the CTA's output channels when the tokens use at least half of the
//     pack's columns;
//   warps 0-7 (compute): warp w owns tokens [16(w&3), +16) and channel groups
//     [4(w>>2), +4) of the tile; the K loop's int32 partials go to shared
//     memory, the pair adds them through distributed shared memory (CTA c
//     keeps channels [c*half, (c+1)*half) of the tile), then the epilogue.
// Loads that the tail depends on (peer partials, the shrink's partial sums,
// w_scale) are all issued before any of them is used.  Every spin-wait is
// bounded; all threads of both CTAs pass the same barriers in the same order,
// also after a wait that ran out.
// ---------------------------------------------------------------------------
constexpr int kDecTileUnits = 8;                     // 8-channel groups per tile, at most
constexpr int kDecRowsMax = 8 * kDecTileUnits;       // 64 output channels
constexpr int kDecKbStage = 2;                       // 128-byte K blocks per stage
constexpr int kDecStages = 4;
constexpr int kDecWBytes = kDecKbStage * kDecRowsMax * 128;  // Wq slabs of a stage (16 KB)
constexpr int kDecXBytes = kDecKbStage * kDecMaxM * 128;     // Xq slabs of a stage (16 KB)
constexpr int kDecStageBytes = kDecWBytes + kDecXBytes;
constexpr int kDecBBytes = (kDecRowsMax / 2) * SQ_MAX_LORA_COLS * 2;  // 64 KB
constexpr int kDecComputeWarps = 8;
constexpr int kDecComputeThreads = 32 * kDecComputeWarps;
constexpr int kDecGemmThreads = kDecComputeThreads + 32;
// named barriers: 1 compute warps; 2 all warps after the token lookup;
// 3 all warps after a tile's K loop; 4 all warps after a tile's epilogue
constexpr int kBarCompute = 1, kBarLookup = 2, kBarRingFree = 3, kBarTileEnd = 4;

struct DecodeCtl {
  uint64_t full[kDecStages];
  uint64_t empty[kDecStages];
  uint64_t bfull;                  // B' rows landed
  int tok_off[kDecMaxM];           // adapter column offset per token
  int tok_rank[kDecMaxM];          // adapter rank per token (0: none)
  float xs[kDecMaxM];              // x_scale per token
  DecodeTables tb;
  int abort;
  int bdense;                      // B' rows staged in shared memory (first tile)
  int rmax;                        // largest rank among the tokens
};
// after the K loop the ring holds the int32 partials [64][64] and then T [64][256] fp32
// (row strides padded so that the epilogue's lanes, which walk tokens, hit
// distinct shared-memory banks)
constexpr int kDecPStride = kDecRowsMax + 2;         // int32 per partial row
constexpr int kDecTStride = kDecMaxRank + 4;         // fp32 per T row
constexpr int kDecPartBytes = (kDecMaxM * kDecPStride * 4 + 15) / 16 * 16;
static_assert(kDecPartBytes + kDecMaxM * kDecTStride * 4 <= kDecStages * kDecStageBytes,
              "partials and T must fit the ring");

constexpr size_t kDecSmemBytes =
    static_cast<size_t>(kDecStages) * kDecStageBytes + kDecBBytes + sizeof(DecodeCtl) + 1024;

__device__ __forceinline__ void mma_s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 8 bf16 (one 16-byte word) times 8 fp32 values, added to d
__device__ __forceinline__ float dot8_bf16(const uint4 &w, const float4 &t0, const float4 &t1,
                                           float d) {
  d = fmaf(t0.x, __uint_as_float(w.x << 16), d);
  d = fmaf(t0.y, __uint_as_float(w.x & 0xffff0000u), d);
  d = fmaf(t0.z, __uint_as_float(w.y << 16), d);
  d = fmaf(t0.w, __uint_as_float(w.y & 0xffff0000u), d);
  d = fmaf(t1.x, __uint_as_float(w.z << 16), d);
  d = fmaf(t1.y, __uint_as_float(w.z & 0xffff0000u), d);
  d = fmaf(t1.z, __uint_as_float(w.w << 16), d);
  d = fmaf(t1.w, __uint_as_float(w.w & 0xffff0000u), d);
  return d;
}

// (at most 112 registers a thread: a block of the shrink fits beside it on an SM)
__global__ void __launch_bounds__(kDecGemmThreads, 2) decode_gemm_kernel(
    const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
    int view3d, const float *__restrict__ x_scale, const float *__restrict__ w_scale, int64_t M,
    int64_t N, int64_t K, int mode, const uint16_t *__restrict__ B_pack,
    const int32_t *__restrict__ lora_offset, const int32_t *__restrict__ lora_rank,
    int n_adapters, int64_t R, const int32_t *__restrict__ seg_offsets,
    const int32_t *__restrict__ seg_adapter, int64_t S, const float *part, int ksplit,
    int tile_units, int tiles, void *__restrict__ out, uint64_t timeout_ns) {
  extern __shared__ uint8_t dsm_raw[];
  uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint16_t *bsm = reinterpret_cast<uint16_t *>(ring + kDecStages * kDecStageBytes);
  DecodeCtl &ctl = *reinterpret_cast<DecodeCtl *>(ring + kDecStages * kDecStageBytes + kDecBBytes);
  int *P = reinterpret_cast<int *>(ring);                          // [64][kDecPStride] int32
  float *Tm = reinterpret_cast<float *>(ring + kDecPartBytes);     // [64][kDecTStride] fp32
  volatile int *abort_flag = &ctl.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const int pair = static_cast<int>(blockIdx.x >> 1), npairs = static_cast<int>(gridDim.x >> 1);
  const bool lora = (part != nullptr);
  const int tile_rows = 8 * tile_units, half = 4 * tile_units;
  const int slab_w = tile_rows * 128;  // bytes of one K block of the Wq tile
  const int nk = (mode == 2) ? 0 : static_cast<int>((K + 127) / 128);
  const int nk_half = (nk + 1) / 2;
  const int kb0 = static_cast<int>(crank) * nk_half;
  const int my_nk = max(0, min(nk, kb0 + nk_half) - kb0);
  const int nstage = (my_nk + kDecKbStage - 1) / kDecKbStage;
  // the pairs start their K walk at different stages, so that few CTAs read
  // the same Xq lines of L2 at once
  const int rot = nstage > 0 ? pair % nstage : 0;
  const int mt = static_cast<int>(min(M, static_cast<int64_t>(kDecMaxM)));

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(&ctl.full[s], 1);
      mbar_init(&ctl.empty[s], kDecComputeWarps);
    }
    mbar_init(&ctl.bfull, 1);
    ctl.abort = 0;
    ctl.bdense = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kDecComputeWarps) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tmap(&tm_w);
      prefetch_tmap(&tm_x);
    }
    int q = 0;  // stages issued so far (all tiles)
    bool looked_up = false, b_issued = false, stop = false;
    auto after_lookup = [&](int first_tile) {
      // B' rows of this CTA's channels in the first tile, when the tokens use
      // at least half of the pack's columns (else the epilogue reads the used
      // columns from global memory)
      group_bar(kBarLookup, kDecGemmThreads);
      looked_up = true;
      if (!lora || first_tile >= tiles || lane != 0 || R <= 0) return;
      unsigned long long used = 0;  // 16-column groups (R <= 1024)
      for (int i = 0; i < mt; ++i) {
        const int r = ctl.tok_rank[i];
        if (r > 0) {
          const int g0 = ctl.tok_off[i] >> 4, g1 = (ctl.tok_off[i] + r + 15) >> 4;
          for (int g = g0; g < g1; ++g) used |= 1ull << g;
        }
      }
      if (2 * 16 * __popcll(used) < R) return;
      const int64_t c0 = static_cast<int64_t>(first_tile) * tile_rows + crank * half;
      const int64_t rows = max(static_cast<int64_t>(0), min(static_cast<int64_t>(half), N - c0));
      if (rows <= 0) return;
      const uint32_t bytes = static_cast<uint32_t>(rows * R * 2);
      ctl.bdense = 1;
      mbar_arrive_expect_tx(&ctl.bfull, bytes);
      bulk_load(bsm, B_pack + c0 * R, bytes, &ctl.bfull);
      b_issued = true;
    };
    for (int tile = pair; tile < tiles; tile += npairs) {
      const int32_t n0 = tile * tile_rows;
      for (int si = 0; si < nstage; ++si) {
        const int slot = q % kDecStages;
        const uint32_t ph = static_cast<uint32_t>(q / kDecStages) & 1u;
        const int sj = si + rot < nstage ? si + rot : si + rot - nstage;
        const int kbs = kb0 + sj * kDecKbStage;                       // first K block
        const int nkb = min(kDecKbStage, kb0 + my_nk - kbs);          // this CTA's blocks
        const int boxes = view3d ? kDecKbStage : nkb;                 // K blocks copied
        bool got = true;
        if (lane == 0 && !stop) {
          // nothing more is issued once any wait has run out: a slot whose
          // copy nobody waited for may still be written to
          got = !*abort_flag && mbar_wait(&ctl.empty[slot], ph ^ 1u, timeout_ns, abort_flag) &&
                !*abort_flag;
          if (got)
            mbar_arrive_expect_tx(&ctl.full[slot],
                                  static_cast<uint32_t>(boxes * (slab_w + kDecMaxM * 128)));
        }
        got = __shfl_sync(0xffffffffu, got && !stop, 0);
        if (!got) {
          if (lane == 0 && !stop) {
            *reinterpret_cast<volatile int *>(abort_flag) = 1;
            record_device_error(SQ_ERR_DEVICE_TIMEOUT);
          }
          stop = true;
        } else {
          uint8_t *st = ring + slot * kDecStageBytes;
          if (view3d) {
            if (lane == 0) tma_load_3d(st, &tm_w, &ctl.full[slot], 0, n0, kbs);
            if (lane == 1) tma_load_3d(st + kDecWBytes, &tm_x, &ctl.full[slot], 0, 0, kbs);
          } else if (lane < 2 * nkb) {
            const int kb = lane >> 1;
            if ((lane & 1) == 0)
              tma_load_2d(st + kb * slab_w, &tm_w, &ctl.full[slot], (kbs + kb) * 128, n0);
            else
              tma_load_2d(st + kDecWBytes + kb * kDecMaxM * 128, &tm_x, &ctl.full[slot],
                          (kbs + kb) * 128, 0);
          }
          ++q;
        }
        if (!looked_up && (q == kDecStages || si == nstage - 1)) after_lookup(pair);
      }
      if (!looked_up) after_lookup(pair);
      // every copy of this tile must land before the ring is reused (also
      // after a wait that ran out: wait for the last use of each slot)
      if (lane == 0) {
        volatile int never = 0;
        const int issued = q;
        for (int k = 0; k < kDecStages && k < issued; ++k) {
          const int last = issued - 1 - ((issued - 1 - k) % kDecStages);
          mbar_wait(&ctl.full[last % kDecStages], static_cast<uint32_t>(last / kDecStages) & 1u,
                    1000000000ull, &never);
        }
      }
      __syncwarp();
      group_bar(kBarRingFree, kDecGemmThreads);
      cluster_sync();  // partials written by both CTAs
      cluster_sync();  // partials read by both CTAs
      group_bar(kBarTileEnd, kDecGemmThreads);
    }
    if (!looked_up) after_lookup(pair);
    if (lane == 0 && b_issued) {
      volatile int never = 0;
      mbar_wait(&ctl.bfull, 0, 1000000000ull, &never);
    }
    return;
  }

  // ----------------------------------------------------------- compute
  const int tid = threadIdx.x;
  const int g = lane >> 2, tig = lane & 3;
  if (lora)
    decode_lookup(seg_offsets, seg_adapter, S, lora_offset, lora_rank, n_adapters, R, 0, mt, tid,
                  kDecComputeThreads, kBarCompute, ctl.tb, ctl.tok_off, ctl.tok_rank);
  else
    for (int i = tid; i < kDecMaxM; i += kDecComputeThreads) ctl.tok_rank[i] = 0;
  for (int i = tid; i < kDecMaxM; i += kDecComputeThreads)
    ctl.xs[i] = (mode != 1 && i < M) ? __ldg(x_scale + i) : 0.f;
  if (warp == 0) {  // (the lookup ended with a barrier of the compute warps)
    int r = max(lane < mt ? ctl.tok_rank[lane] : 0, lane + 32 < mt ? ctl.tok_rank[lane + 32] : 0);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) r = max(r, __shfl_xor_sync(0xffffffffu, r, o));
    if (lane == 0) ctl.rmax = r;
  }
  group_bar(kBarLookup, kDecGemmThreads);

  const int mtile = warp & 3, ng = warp >> 2;
  const int ra = mtile * 16 + g, rb = ra + 8;  // token rows of this lane's A fragments
  int q = 0;
  bool first = true;
  for (int tile = pair; tile < tiles; tile += npairs) {
    const int64_t n0 = static_cast<int64_t>(tile) * tile_rows;
    const int64_t c0 = n0 + static_cast<int64_t>(crank) * half;  // this CTA's first channel
    // epilogue: token tok = tid % 64 and channel pairs p = tid/64 + 4m of this
    // CTA's half of the tile (a warp's lanes walk 32 tokens)
    const int tok = tid & 63;
    const int npairs_out = half / 2;
    // w_scale of this thread's epilogue channels, loaded ahead of every wait
    float wsv[4][2];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int p = (tid >> 6) + 4 * m;
      const int64_t n = c0 + 2 * p;
      const bool ok_n = mode == 0 && p < npairs_out && n < N;
      wsv[m][0] = ok_n ? __ldg(w_scale + n) : 0.f;
      wsv[m][1] = ok_n ? __ldg(w_scale + n + 1) : 0.f;
    }
    int acc[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[u][e] = 0;
    bool ok = true;
    for (int si = 0; si < nstage; ++si, ++q) {
      const int slot = q % kDecStages;
      const uint32_t ph = static_cast<uint32_t>(q / kDecStages) & 1u;
      // the warp leaves together: the mma.sync below needs all lanes.  A warp
      // whose wait ran out raises the abort flag at once and hands no more
      // stages back (the producer then issues nothing more)
      if (ok) {
        ok = __all_sync(0xffffffffu, mbar_wait(&ctl.full[slot], ph, timeout_ns, abort_flag));
        if (!ok && lane == 0) *reinterpret_cast<volatile int *>(abort_flag) = 1;
      }
      if (!ok) continue;
      const int sj = si + rot < nstage ? si + rot : si + rot - nstage;
      const int nkb = min(kDecKbStage, my_nk - sj * kDecKbStage);
      for (int kb = 0; kb < nkb; ++kb) {
        const uint8_t *wt = ring + slot * kDecStageBytes + kb * slab_w;
        const uint8_t *xt = ring + slot * kDecStageBytes + kDecWBytes + kb * kDecMaxM * 128;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // 16 contiguous K bytes (chunk 4h + tig of the 128-byte row, stored
          // 128B-swizzled) of each operand row; the K order inside the 64
          // bytes is a permutation that A and B share
          const uint4 xa = *reinterpret_cast<const uint4 *>(xt + ra * 128 + (((4 * h + tig) ^ (ra & 7)) * 16));
          const uint4 xb = *reinterpret_cast<const uint4 *>(xt + rb * 128 + (((4 * h + tig) ^ (rb & 7)) * 16));
          const uint32_t fa0[4] = {xa.x, xb.x, xa.y, xb.y};
          const uint32_t fa1[4] = {xa.z, xb.z, xa.w, xb.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (ng * 4 + u >= tile_units) continue;  // warp-uniform
            const int row = (ng * 4 + u) * 8 + g;
            const uint4 bw = *reinterpret_cast<const uint4 *>(wt + row * 128 + (((4 * h + tig) ^ (row & 7)) * 16));
            mma_s8_16832(acc[u], fa0, bw.x, bw.y);
            mma_s8_16832(acc[u], fa1, bw.z, bw.w);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.empty[slot]);
    }
    if (!ok) {
      *reinterpret_cast<volatile int *>(abort_flag) = 1;
      record_device_error(SQ_ERR_DEVICE_TIMEOUT);
    }
    // every copy into the ring has landed (the producer waited): the
    // partials go where the stages were
    group_bar(kBarRingFree, kDecGemmThreads);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = (ng * 4 + u) * 8 + 2 * tig;
      *reinterpret_cast<int2 *>(P + ra * kDecPStride + c) = make_int2(acc[u][0], acc[u][1]);
      *reinterpret_cast<int2 *>(P + rb * kDecPStride + c) = make_int2(acc[u][2], acc[u][3]);
    }
    cluster_sync();
    // this CTA keeps channels [crank*half, (crank+1)*half) of the tile: its
    // own partial plus the peer's, every load issued before the first add
    const uint32_t peer = crank ^ 1u;
    int2 own[4], oth[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int p = (tid >> 6) + 4 * m;
      own[m] = make_int2(0, 0);
      oth[m] = make_int2(0, 0);
      if (p < npairs_out) {
        const int c = static_cast<int>(crank) * half + 2 * p;
        own[m] = *reinterpret_cast<const int2 *>(P + tok * kDecPStride + c);
        oth[m] = ld_cluster_i2(map_to_rank(smem_u32(P + tok * kDecPStride + c), peer));
      }
    }
    int2 accv[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) accv[m] = make_int2(own[m].x + oth[m].x, own[m].y + oth[m].y);
    cluster_sync();
    // ---- LoRA: T = x_scale * (sum of the shrink's slices in order), after
    //      the shrink grid has completed; each thread takes four (token, rank)
    //      entries of a 16-rank group and loads all their slices at once
    const int r_i = (tok < mt) ? ctl.tok_rank[tok] : 0;
    const int off_i = (tok < mt) ? ctl.tok_off[tok] : 0;
    const bool any_lora = lora && mode != 1;
    if (any_lora) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      const int rmax = ctl.rmax;
      for (int jb = 0; jb < rmax; jb += 16) {
        const int j = jb + (tid & 15);
        float pv[4][kDecShrinkSplitMax];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int t = (tid >> 4) + 16 * u;
          const int r = (t < mt) ? ctl.tok_rank[t] : 0;
#pragma unroll
          for (int ks = 0; ks < kDecShrinkSplitMax; ++ks)
            pv[u][ks] = (j < r && ks < ksplit)
                            ? part[(static_cast<int64_t>(ks) * M + t) * kDecMaxRank + j]
                            : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int t = (tid >> 4) + 16 * u;
          const int r = (t < mt) ? ctl.tok_rank[t] : 0;
          if (t < mt && j < ((r + 15) & ~15)) {
            float sacc = 0.f;  // zero in the padding columns
#pragma unroll
            for (int ks = 0; ks < kDecShrinkSplitMax; ++ks) sacc += pv[u][ks];
            Tm[t * kDecTStride + j] = __fmul_rn(ctl.xs[t], sacc);
          }
        }
      }
      group_bar(kBarCompute, kDecComputeThreads);
    }
    const bool use_bsm = first && ctl.bdense;
    if (use_bsm && !mbar_wait(&ctl.bfull, 0, timeout_ns, abort_flag)) {
      *reinterpret_cast<volatile int *>(abort_flag) = 1;
      record_device_error(SQ_ERR_DEVICE_TIMEOUT);
    }
    const bool aborted = *abort_flag != 0;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int p = (tid >> 6) + 4 * m;
      const int64_t n = c0 + 2 * p;
      if (p >= npairs_out || tok >= mt || n >= N || aborted) continue;
      float d0 = 0.f, d1 = 0.f;
      if (any_lora && r_i > 0) {
        const float *Ti = Tm + tok * kDecTStride;
        for (int j = 0; j < r_i; j += 8) {
          const float4 t0 = *reinterpret_cast<const float4 *>(Ti + j);
          const float4 t1 = *reinterpret_cast<const float4 *>(Ti + j + 4);
          uint4 w0, w1;
          if (use_bsm) {
            w0 = *reinterpret_cast<const uint4 *>(bsm + (n - c0) * R + off_i + j);
            w1 = *reinterpret_cast<const uint4 *>(bsm + (n + 1 - c0) * R + off_i + j);
          } else {
            w0 = __ldg(reinterpret_cast<const uint4 *>(B_pack + n * R + off_i + j));
            w1 = __ldg(reinterpret_cast<const uint4 *>(B_pack + (n + 1) * R + off_i + j));
          }
          d0 = dot8_bf16(w0, t0, t1, d0);
          d1 = dot8_bf16(w1, t0, t1, d1);
        }
      }
      if (mode == 0) {
        const float xs = ctl.xs[tok];
        const float y0 = __fadd_rn(__fmul_rn(__fmul_rn(__int2float_rn(accv[m].x), xs), wsv[m][0]), d0);
        const float y1 = __fadd_rn(__fmul_rn(__fmul_rn(__int2float_rn(accv[m].y), xs), wsv[m][1]), d1);
        __nv_bfloat162 hh = __floats2bfloat162_rn(y0, y1);
        *reinterpret_cast<uint32_t *>(static_cast<uint16_t *>(out) + tok * N + n) =
            *reinterpret_cast<uint32_t *>(&hh);
      } else if (mode == 1) {
        *reinterpret_cast<int2 *>(static_cast<int32_t *>(out) + tok * N + n) = accv[m];
      } else {
        *reinterpret_cast<float2 *>(static_cast<float *>(out) + tok * N + n) = make_float2(d0, d1);
      }
    }
    first = false;
    group_bar(kBarTileEnd, kDecGemmThreads);
  }
}

size_t decode_workspace_bytes(int64_t M) {
  return static_cast<size_t>(kDecShrinkSplitMax) * static_cast<size_t>(M) * kDecMaxRank *
         sizeof(float);
}

bool decode_applicable(int64_t M) { return M > 0 && M <= kDecMaxM; }

// CTA pairs of decode_gemm_kernel that fit on the current device at once
// (cached per device).  On first use per device the kernels' shared-memory
// settings are made: the GEMM's opt-in, and the shrink's preference for the
// largest shared-memory carveout, so that an SM running shrink blocks keeps
// room for a GEMM CTA beside them (a block pins its SM's carveout, and an SM
// split for a small-shared-memory kernel cannot host the GEMM until it empties).
static cudaError_t decode_pairs(int *pairs) {
  static std::atomic<int> attr_set[kMaxDevices];
  static std::atomic<int> cached[kMaxDevices];
  const int dev = current_device_index();
  if (dev < 0) return cudaErrorInvalidDevice;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    cudaError_t e = ensure_smem_optin(decode_gemm_kernel, static_cast<int>(kDecSmemBytes), attr_set);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(decode_shrink_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(kDecGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = kDecSmemBytes;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    e = cudaOccupancyMaxActiveClusters(&n, decode_gemm_kernel, &cfg);
    if (e != cudaSuccess) return e;
    n = n > 0 ? n : sm_count_of_current_device() / 2;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  *pairs = n;
  return cudaSuccess;
}

// mode: 0 = Y bf16, 1 = int32 accumulators, 2 = LoRA delta fp32.
// `part` (scratch, decode_workspace_bytes(M)) may be null when there is no LoRA.
cudaError_t launch_decode(const int8_t *Xq, const float *x_scale, const int8_t *Wq,
                          const float *w_scale, int64_t M, int64_t N, int64_t K, int mode,
                          const uint16_t *A_pack, const uint16_t *B_pack,
                          const int32_t *lora_offset, const int32_t *lora_rank, int n_adapters,
                          int64_t R, const int32_t *seg_offsets, const int32_t *seg_adapter,
                          int64_t S, float *part, void *out, cudaStream_t st) {
  const bool lora = part != nullptr && mode != 1;
  int max_pairs = 0;
  cudaError_t e = decode_pairs(&max_pairs);
  if (e != cudaSuccess) return e;
  int ksplit = static_cast<int>((K + kDecShrinkSpan - 1) / kDecShrinkSpan);
  ksplit = ksplit < 1 ? 1 : (ksplit > kDecShrinkSplitMax ? kDecShrinkSplitMax : ksplit);
  if (lora) {
    decode_shrink_kernel<<<static_cast<unsigned>(M * ksplit), kDecShrinkThreads, 0, st>>>(
        Xq, M, K, ksplit, A_pack, lora_offset, lora_rank, n_adapters, R, seg_offsets, seg_adapter,
        S, part);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // tiles of up to 8 groups of 8 channels, sized so that the pairs that fit
  // on the device get one tile each where N allows
  const int64_t units = N / 8;
  const int64_t per = (units + max_pairs - 1) / max_pairs;
  const int tile_units = static_cast<int>(per < 1 ? 1 : (per > kDecTileUnits ? kDecTileUnits : per));
  const int64_t tiles = (units + tile_units - 1) / tile_units;
  const int pairs = static_cast<int>(tiles < max_pairs ? tiles : max_pairs);
  CUtensorMap tm_w, tm_x;
  memset(&tm_w, 0, sizeof tm_w);
  memset(&tm_x, 0, sizeof tm_x);
  // K a multiple of 128: one 3D box per operand and stage; otherwise one 2D
  // box per K block (the last block's tail is filled with zeros)
  const int view3d = (K % 128 == 0) ? 1 : 0;
  if (mode != 2) {
    const bool made =
        view3d ? (make_tmap_kblocks(&tm_w, Wq, K, N, 8 * tile_units, kDecKbStage) &&
                  make_tmap_kblocks(&tm_x, Xq, K, M, kDecMaxM, kDecKbStage))
               : (make_tmap(&tm_w, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, N, 128, 8 * tile_units) &&
                  make_tmap(&tm_x, Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, M, 128, kDecMaxM));
    if (!made) return cudaErrorInvalidValue;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
  cfg.blockDim = dim3(kDecGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = kDecSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = 2;
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = lora ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, decode_gemm_kernel, tm_w, tm_x, view3d, x_scale, w_scale, M, N,
                            K, mode, B_pack, lora_offset, lora_rank, n_adapters, R, seg_offsets,
                            seg_adapter, S, lora ? static_cast<const float *>(part) : nullptr,
                            ksplit, tile_units, static_cast<int>(tiles), out, wait_timeout_ns());
}

}  // namespace sq
