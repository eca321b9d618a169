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
//                       CTA of the pair one half of K; the Wq tile streams in
//                       through cp.async on the load/store path (a 2D TMA box
//                       of short rows from HBM is issued too slowly to keep
//                       an SM's share of the bandwidth) beside one TMA box of
//                       Xq per stage, and acc = Xq Wq^T runs on the tensor
//                       cores (tcgen05, exact int32 in tensor memory); the
//                       pair adds its halves with one bulk copy from shared
//                       memory to the peer's; after the shrink grid has
//                       completed (programmatic dependent launch),
//                       T = x_scale * (sum of the partials in a fixed order)
//                       and Y = bf16(acc*xs*ws + T B_a^T).
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
// At most 96 registers a thread: an SM's registers are split between its
// four sub-partitions (16K each) and a block's warps are dealt to them in
// turn, so a GEMM CTA (12 warps of 96 registers: 3 on each sub-partition)
// fits beside a shrink block (2 warps on each) only while 3*96 + 2*r <= 512.
__global__ void __maxnreg__(96) decode_shrink_kernel(
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
// A tile is `tile_units` groups of 8 output channels (at most 64); tiles are
// dealt to the pairs in turn and each CTA of a pair takes one half of K.
// Per CTA and tile:
//   warps 3-11 (loaders) stream the CTA's K half in stages of two 128-byte K
//     blocks: the tile's Wq rows by 16-byte cp.async copies (256 contiguous
//     bytes of a row per stage, stored in the 128-byte swizzled layout the
//     tensor core reads; a warp keeps only a few dozen copies in flight, so
//     nine warps share them), and the 64 Xq rows by one TMA box of warp 11's
//     lane 0 (every CTA reads the same Xq, so it comes from L2);
//   warp 0, lane 0 issues the tensor-core MMAs of each stage as it lands:
//     D[ch, tok] += Wq[ch, k] Xq[tok, k] with M = 128 channel rows (rows past
//     the tile read bytes of the next slab; their results are never used),
//     N = 64 tokens, exact int32 accumulators in tensor memory;
//   warps 1-2 meanwhile find each token's adapter and, once the shrink grid
//     has completed, form T = x_scale * (sum of the shrink's slices), each
//     in one round of loads (a load issued while the SM streams waits behind
//     the copies in flight; for ranks above 64 T is formed after the K loop
//     where the stages were);
//   the B' rows of the channels this CTA keeps are bulk-copied into a region
//     of their own during the K loop when the tokens read most of each row
//     (else each thread's B' words are copied after it);
//   then warps 0-1 move D to shared memory, the channels the peer finishes
//     go to the peer in one bulk copy counted on its mbarrier, and warps 0-7
//     finish the channels this CTA keeps, one channel per lane and 8 tokens
//     per warp: acc = own + peer partial, delta = T B_a^T,
//     Y = bf16(acc*xs*ws + delta).
// Every wait on another thread is bounded; all threads of both CTAs pass the
// same barriers in the same order, also after a wait that ran out, and no
// CTA exits while a copy into its shared memory or a tensor-core operation
// may still be in flight.
// ---------------------------------------------------------------------------
constexpr int kDecTileUnits = 8;                     // 8-channel groups per tile, at most
constexpr int kDecRowsMax = 8 * kDecTileUnits;       // 64 output channels
constexpr int kDecKbStage = 2;                       // 128-byte K blocks per stage
constexpr int kDecStages = 4;
constexpr int kDecWBytes = kDecKbStage * kDecRowsMax * 128;  // Wq slabs of a stage (16 KB)
constexpr int kDecXBytes = kDecKbStage * kDecMaxM * 128;     // Xq slabs of a stage (16 KB)
constexpr int kDecStageBytes = kDecWBytes + kDecXBytes;
constexpr int kDecRingBytes = kDecStages * kDecStageBytes;
constexpr int kDecKeepMax = kDecRowsMax / 2;                 // channels a CTA finishes
constexpr int kDecTEarlyCols = 64;                           // T has its own region up to this rank
constexpr int kDecTEarlyBytes = kDecMaxM * kDecTEarlyCols * 4;
constexpr int kDecRecvBytes = kDecMaxM * kDecKeepMax * 4;    // the peer's partials
constexpr int kDecEpiWarps = 8;
constexpr int kDecEpiThreads = 32 * kDecEpiWarps;
constexpr int kDecGemmThreads = kDecEpiThreads + 128;       // warps 8-11 only load
constexpr int kDecLookupThreads = 64;                        // warps 1-2
constexpr int kDecFirstLoader = 3;                           // warps 3-11 load Wq
constexpr int kDecLoaderThreads = kDecGemmThreads - 32 * kDecFirstLoader;
constexpr int kDecXWarp = kDecGemmThreads / 32 - 1;          // warp 11 also loads Xq
constexpr uint32_t kDecTmemCols = 64;
constexpr uint32_t kDecIdesc = idesc_i8_s32(128, kDecMaxM);
// full barrier of a stage: one cp.async arrival per loader thread; the Xq
// box of the stage is counted on a barrier of its own (xfull)
// after the K loop the ring holds the partials sent to the peer [64][peer
// channels], this CTA's own partials [64][32] and T [64][rank padded to 16]
// when it has no room of its own
constexpr int kDecSendOff = 0, kDecOwnOff = 8192, kDecTOff = 16384;
static_assert(kDecTOff + kDecMaxM * kDecMaxRank * 4 <= kDecRingBytes, "T must fit the ring");
// the epilogue's B' words have a region of their own: either the kept
// channels' whole B' rows (copied during the K loop; row stride 2R + 16
// bytes, so that lanes on consecutive rows hit distinct banks) or 16 words of
// 16 bytes per thread, stored [word][thread]
constexpr int kDecBBytes = kDecKeepMax * (2 * SQ_MAX_LORA_COLS + 16);
static_assert(16 * kDecEpiThreads * 16 <= kDecBBytes, "the per-thread B' words fit the region");
// the MMA of K block 1 reads 128 rows from its slab: still inside the stage
static_assert((kDecKbStage - 1) * kDecRowsMax * 128 + 128 * 128 <= kDecStageBytes,
              "the channel rows an MMA reads must stay inside its stage");
// named barriers: 1 warps 1-2 (token lookup); 2 warps 0-7; 3 all warps at a tile's end
constexpr int kBarLookup = 1, kBarEpi = 2, kBarTileEnd = 3;

struct DecodeCtl {
  uint64_t full[kDecStages];       // Wq bytes of the stage landed
  uint64_t xfull[kDecStages];      // Xq bytes of the stage landed
  uint64_t empty[kDecStages];      // the stage's MMAs have read it
  uint64_t accfull;                // the tile's MMAs have completed
  uint64_t rbar;                   // the peer's partials have landed
  uint64_t bbar;                   // the kept channels' B' rows have landed
  uint32_t tmem_base;
  int tok_off[kDecMaxM];           // adapter column offset per token
  int tok_rank[kDecMaxM];          // adapter rank per token (0: none)
  float xs[kDecMaxM];              // x_scale per token
  DecodeTables tb;
  int abort;
  int rmax;                        // largest rank among the tokens
  int b_dense;                     // the tokens use at least half of the B' columns
  int t_early;                     // T formed during the K loop, in its own region
};

constexpr size_t kDecSmemBytes = static_cast<size_t>(kDecRingBytes) + kDecRecvBytes +
                                 kDecTEarlyBytes + kDecBBytes + sizeof(DecodeCtl) + 1024;

// 8 bf16 (one 16-byte word) times 8 fp32 values, added to d in order
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

// T[t][j] = x_scale[t] * (sum over the shrink's K slices, in order, of its
// partial sums) for tokens t < mt and j < tstride (zero for j >= rank_t).
// Work goes by quads of four consecutive j (tstride is a multiple of 16 and
// a partial-sum row holds kDecMaxRank values, so a quad never leaves its
// row; values past the rank are read but not used).  Each thread takes kB
// quads at a time and loads two slices of each per round (one round when K
// is at most two slices).
template <int kB>
__device__ void decode_form_t(float *T, int tstride, const float *part, int64_t M, int ksplit,
                              int mt, const DecodeCtl &ctl, int tid, int nthr) {
  const int qrow = tstride >> 2;
  const int nq = mt * qrow;
  for (int q0 = tid; q0 < nq; q0 += kB * nthr) {
    float4 sacc[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) sacc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int ks0 = 0; ks0 < ksplit; ks0 += 2) {
      float4 v[kB][2];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int qq = q0 + u * nthr;
        const int t = qq < nq ? qq / qrow : 0, j = 4 * (qq - t * qrow);
        const bool use = qq < nq && j < ctl.tok_rank[t];
#pragma unroll
        for (int h = 0; h < 2; ++h)
          v[u][h] = (use && ks0 + h < ksplit)
                        ? *reinterpret_cast<const float4 *>(
                              part + (static_cast<int64_t>(ks0 + h) * M + t) * kDecMaxRank + j)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kB; ++u) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          sacc[u].x += v[u][h].x;
          sacc[u].y += v[u][h].y;
          sacc[u].z += v[u][h].z;
          sacc[u].w += v[u][h].w;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const int qq = q0 + u * nthr;
      if (qq < nq) {
        const int t = qq / qrow, j = 4 * (qq - t * qrow);
        const int r = ctl.tok_rank[t];
        const float xs = ctl.xs[t];
        float4 o;
        o.x = j + 0 < r ? __fmul_rn(xs, sacc[u].x) : 0.f;
        o.y = j + 1 < r ? __fmul_rn(xs, sacc[u].y) : 0.f;
        o.z = j + 2 < r ? __fmul_rn(xs, sacc[u].z) : 0.f;
        o.w = j + 3 < r ? __fmul_rn(xs, sacc[u].w) : 0.f;
        *reinterpret_cast<float4 *>(T + t * tstride + j) = o;
      }
    }
  }
}

// B' words [jb, jb + 16) of channel row `brow` for the thread's tokens
// tk0 .. tk0 + 7 into its slots of `bst` (slot 2u + h of token tk0 + u holds
// columns jb + 8h .. jb + 8h + 7); words past a token's rank are not copied
__device__ __forceinline__ void decode_stage_b(uint8_t *bst, int etid, const uint16_t *brow,
                                               int tk0, int jb, int mt, const DecodeCtl &ctl) {
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int tok = tk0 + u;
    const int r = tok < mt ? ctl.tok_rank[tok] : 0;
    const uint16_t *bp = brow + (tok < mt ? ctl.tok_off[tok] : 0) + jb;
#pragma unroll
    for (int h = 0; h < 2; ++h)
      if (jb + 8 * h < r) cp_async_16(bst + ((2 * u + h) * kDecEpiThreads + etid) * 16, bp + 8 * h);
  }
}

// (at most 96 registers a thread: a block of the shrink fits beside it on an SM)
__global__ void __maxnreg__(96) decode_gemm_kernel(
    const __grid_constant__ CUtensorMap tm_x, int view3d, const int8_t *__restrict__ Wq,
    const float *__restrict__ x_scale, const float *__restrict__ w_scale, int64_t M, int64_t N,
    int64_t K, int mode, const uint16_t *__restrict__ B_pack,
    const int32_t *__restrict__ lora_offset, const int32_t *__restrict__ lora_rank,
    int n_adapters, int64_t R, const int32_t *__restrict__ seg_offsets,
    const int32_t *__restrict__ seg_adapter, int64_t S, const float *part, int ksplit,
    int tile_units, int tiles, void *__restrict__ out, uint64_t timeout_ns) {
  extern __shared__ uint8_t dsm_raw[];
  uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  int *recv = reinterpret_cast<int *>(ring + kDecRingBytes);
  float *t_own = reinterpret_cast<float *>(ring + kDecRingBytes + kDecRecvBytes);
  uint8_t *bst = ring + kDecRingBytes + kDecRecvBytes + kDecTEarlyBytes;  // the B' region
  DecodeCtl &ctl = *reinterpret_cast<DecodeCtl *>(ring + kDecRingBytes + kDecRecvBytes +
                                                  kDecTEarlyBytes + kDecBBytes);
  int *sendp = reinterpret_cast<int *>(ring + kDecSendOff);
  int *own = reinterpret_cast<int *>(ring + kDecOwnOff);
  volatile int *abort_flag = &ctl.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank(), peer = crank ^ 1u;
  const int pair = static_cast<int>(blockIdx.x >> 1), npairs = static_cast<int>(gridDim.x >> 1);
  const bool lora = (part != nullptr) && mode != 1;
  const int tile_rows = 8 * tile_units;
  // channels [keep_lo, keep_lo + keep_cols) of a tile are finished here, the
  // others by the peer
  const int lo_units = (tile_units + 1) / 2;
  const int keep_lo = crank == 0 ? 0 : 8 * lo_units;
  const int keep_cols = crank == 0 ? 8 * lo_units : 8 * (tile_units - lo_units);
  const int peer_lo = crank == 0 ? 8 * lo_units : 0;
  const int peer_cols = tile_rows - keep_cols;
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
      mbar_init(&ctl.full[s], kDecLoaderThreads);
      mbar_init(&ctl.xfull[s], 1);
      mbar_init(&ctl.empty[s], 1);
    }
    mbar_init(&ctl.accfull, 1);
    mbar_init(&ctl.rbar, 1);
    mbar_init(&ctl.bbar, 1);
    ctl.abort = 0;
    ctl.rmax = 0;
    ctl.b_dense = 0;
    ctl.t_early = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&ctl.tmem_base, kDecTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;
  // the peer pushes its partials only after this arrival: the receive
  // barrier exists by then
  cluster_arrive();

  // ---------------------------------------------------------- loaders
  // (warps 3-7 then join the epilogue; warps 8-11 only load)
  int q = 0;  // stages issued so far by this warp (all tiles)
  bool stop = false;
  auto load_tile = [&](int64_t n0) {
    const int ltid = static_cast<int>(threadIdx.x) - 32 * kDecFirstLoader;
    const int rows = static_cast<int>(min(static_cast<int64_t>(tile_rows), N - n0));
    const int8_t *wtile = Wq + n0 * K;
    for (int si = 0; si < nstage && !stop; ++si) {
      const int slot = q % kDecStages;
      const uint32_t ph = static_cast<uint32_t>(q / kDecStages) & 1u;
      const int sj = si + rot < nstage ? si + rot : si + rot - nstage;
      const int kbs = kb0 + sj * kDecKbStage;               // first K block
      const int nkb = min(kDecKbStage, kb0 + my_nk - kbs);  // this CTA's blocks
      bool got = false;
      if (lane == 0) {
        // nothing more is issued once any wait has run out: a slot whose
        // copy nobody waited for may still be written to
        got = !*abort_flag && mbar_wait(&ctl.empty[slot], ph ^ 1u, timeout_ns, abort_flag) &&
              !*abort_flag;
        if (!got) {
          *reinterpret_cast<volatile int *>(abort_flag) = 1;
          record_device_error(SQ_ERR_DEVICE_TIMEOUT);
        }
      }
      if (!__shfl_sync(0xffffffffu, got, 0)) {
        stop = true;
        break;
      }
      uint8_t *st = ring + slot * kDecStageBytes;
      // Wq: rows x nkb K blocks x 8 chunks of 16 bytes; consecutive threads
      // take consecutive chunks of a row.  Chunks past K are not copied (the
      // Xq box is zero there).
      const int cshift = nkb == 2 ? 4 : 3;
      const int total = rows << cshift;
      const int8_t *src0 = wtile + static_cast<int64_t>(kbs) * 128;
      const int64_t kleft = K - static_cast<int64_t>(kbs) * 128;  // bytes of K from kbs on
      for (int idx = ltid; idx < total; idx += kDecLoaderThreads) {
        const int row = idx >> cshift, cc = idx & ((1 << cshift) - 1);
        if (cc * 16 < kleft) {
          const int kb = cc >> 3, c = cc & 7;
          cp_async_16(st + kb * slab_w + row * 128 + ((c ^ (row & 7)) << 4),
                      src0 + static_cast<int64_t>(row) * K + cc * 16);
        }
      }
      cp_async_mbar_arrive_noinc(&ctl.full[slot]);
      if (warp == kDecXWarp && lane == 0) {
        if (view3d) {
          mbar_arrive_expect_tx(&ctl.xfull[slot], static_cast<uint32_t>(kDecXBytes));
          tma_load_3d(st + kDecWBytes, &tm_x, &ctl.xfull[slot], 0, 0, kbs);
        } else {
          mbar_arrive_expect_tx(&ctl.xfull[slot], static_cast<uint32_t>(nkb * kDecMaxM * 128));
          for (int kb = 0; kb < nkb; ++kb)
            tma_load_2d(st + kDecWBytes + kb * kDecMaxM * 128, &tm_x, &ctl.xfull[slot],
                        (kbs + kb) * 128, 0);
        }
      }
      ++q;
    }
  };
  // every copy into shared memory has landed before the CTA exits (also
  // after a wait that ran out: cp.async by each thread, the Xq boxes by the
  // last use of each slot's barrier)
  auto drain_loads = [&]() {
    cp_async_wait_all();
    if (warp == kDecXWarp && lane == 0) {
      volatile int never = 0;
      for (int k = 0; k < kDecStages && k < q; ++k) {
        const int last = q - 1 - ((q - 1 - k) % kDecStages);
        mbar_wait(&ctl.xfull[last % kDecStages], static_cast<uint32_t>(last / kDecStages) & 1u,
                  1000000000ull, &never);
      }
    }
    __syncwarp();
  };
  if (warp >= kDecEpiWarps) {
    if (warp == kDecXWarp && lane == 0) prefetch_tmap(&tm_x);
    for (int tile = pair; tile < tiles; tile += npairs) {
      load_tile(static_cast<int64_t>(tile) * tile_rows);
      // the ring is reused for this tile's partials: the next tile's copies
      // start after its epilogue
      cluster_wait();
      group_bar(kBarTileEnd, kDecGemmThreads);
      cluster_arrive();
    }
    drain_loads();
    cluster_wait();
    return;
  }

  // ------------------------------------------------ MMA, lookup, epilogue
  // the B' rows of a tile's kept channels into their region, while the K
  // loop runs, when the tokens read most of each row (issued by warp 1,
  // lane 0; the region is free: the previous tile's epilogue has ended)
  const uint32_t brow_stride = static_cast<uint32_t>(R * 2 + 16);
  auto load_b_rows = [&](int64_t n0) {
    const int64_t c0 = n0 + keep_lo;
    const int rows = static_cast<int>(
        max(static_cast<int64_t>(0), min(static_cast<int64_t>(keep_cols), N - c0)));
    if (!(lora && ctl.b_dense) || rows <= 0) return;
    mbar_arrive_expect_tx(&ctl.bbar, static_cast<uint32_t>(rows * R * 2));
    for (int i = 0; i < rows; ++i)
      bulk_load(bst + i * brow_stride, B_pack + (c0 + i) * R, static_cast<uint32_t>(R * 2),
                &ctl.bbar);
  };
  const int etid = threadIdx.x;  // 0..255
  int mq = 0;                    // stages consumed by the MMA thread (all tiles)
  bool mma_ok = true;
  int it = 0;
  for (int tile = pair; tile < tiles; tile += npairs, ++it) {
    const int64_t n0 = static_cast<int64_t>(tile) * tile_rows;
    // this thread's epilogue channel; its w_scale is loaded long before use
    const int64_t n = n0 + keep_lo + lane;
    const float ws_n = (mode == 0 && lane < keep_cols && n < N) ? __ldg(w_scale + n) : 0.f;
    if (warp == 0) {
      if (lane == 0) {
        bool any = false;
        for (int si = 0; si < nstage; ++si, ++mq) {
          const int slot = mq % kDecStages;
          const uint32_t ph = static_cast<uint32_t>(mq / kDecStages) & 1u;
          if (mma_ok) {
            mma_ok = mbar_wait(&ctl.full[slot], ph, timeout_ns, abort_flag) &&
                     mbar_wait(&ctl.xfull[slot], ph, timeout_ns, abort_flag);
            if (!mma_ok) {
              *reinterpret_cast<volatile int *>(abort_flag) = 1;
              record_device_error(SQ_ERR_DEVICE_TIMEOUT);
            }
          }
          if (!mma_ok) continue;
          // the Wq bytes were written by cp.async (generic proxy)
          fence_proxy_async_shared();
          tc_fence_after();
          const int sj = si + rot < nstage ? si + rot : si + rot - nstage;
          const int nkb = min(kDecKbStage, my_nk - sj * kDecKbStage);
          const uint32_t wa = smem_u32(ring + slot * kDecStageBytes);
          const uint32_t xa = wa + kDecWBytes;
          for (int kb = 0; kb < nkb; ++kb) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              mma_i8(tmem, sdesc_kmajor_sw128(wa + kb * slab_w + 32 * k),
                     sdesc_kmajor_sw128(xa + kb * kDecMaxM * 128 + 32 * k), kDecIdesc,
                     any ? 1u : 0u);
              any = true;
            }
          }
          mma_commit(&ctl.empty[slot]);
        }
        if (any)
          mma_commit(&ctl.accfull);
        else
          mbar_arrive(&ctl.accfull);
      }
      __syncwarp();
    } else if (warp >= kDecFirstLoader) {
      load_tile(n0);
    } else if (it == 0) {
      // token lookup and x_scale in one round of loads, then the largest rank
      // and whether the tokens read most of the B' columns
      const int ltid = etid - 32;
      static_assert(kDecMaxM == kDecLookupThreads, "one token a lookup thread");
      const float xsv = (mode != 1 && ltid < M) ? __ldg(x_scale + ltid) : 0.f;
      if (lora) {
        decode_lookup(seg_offsets, seg_adapter, S, lora_offset, lora_rank, n_adapters, R, 0, mt,
                      ltid, kDecLookupThreads, kBarLookup, ctl.tb, ctl.tok_off, ctl.tok_rank);
      } else {
        ctl.tok_rank[ltid] = 0;
        ctl.tok_off[ltid] = 0;
      }
      ctl.xs[ltid] = xsv;
      group_bar(kBarLookup, kDecLookupThreads);
      if (warp == 1) {
        // lane l takes tokens l and l + 32; 16-column groups of the pack the
        // tokens use (R <= 1024)
        int r = 0;
        uint32_t used_lo = 0, used_hi = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int i = lane + 32 * h;
          const int ri = i < mt ? ctl.tok_rank[i] : 0;
          r = max(r, ri);
          if (ri > 0) {
            const int g0 = ctl.tok_off[i] >> 4, g1 = (ctl.tok_off[i] + ri + 15) >> 4;
            for (int g = g0; g < g1; ++g) {
              if (g < 32)
                used_lo |= 1u << g;
              else
                used_hi |= 1u << (g - 32);
            }
          }
        }
        r = __reduce_max_sync(0xffffffffu, r);
        used_lo = __reduce_or_sync(0xffffffffu, used_lo);
        used_hi = __reduce_or_sync(0xffffffffu, used_hi);
        if (lane == 0) {
          ctl.rmax = r;
          ctl.b_dense = lora && r > 0 && 2 * 16 * (__popc(used_lo) + __popc(used_hi)) >= R;
          ctl.t_early = ((r + 15) & ~15) <= kDecTEarlyCols;
          load_b_rows(n0);
        }
      }
      group_bar(kBarLookup, kDecLookupThreads);
      if (lora && ctl.rmax > 0 && ctl.t_early) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        decode_form_t<4>(t_own, (ctl.rmax + 15) & ~15, part, M, ksplit, mt, ctl, ltid,
                          kDecLookupThreads);
      }
    }
    if (warp == 1 && lane == 0 && it > 0) load_b_rows(n0);
    group_bar(kBarEpi, kDecEpiThreads);
    const int rmax = ctl.rmax;
    const int tstride = (rmax + 15) & ~15;
    // ---- D -> shared memory (warps 0-1, thread = channel 32*warp + lane)
    if (warp < 2) {
      const bool acc_ok =
          __all_sync(0xffffffffu, mbar_wait(&ctl.accfull, static_cast<uint32_t>(it) & 1u,
                                             timeout_ns, abort_flag));
      if (!acc_ok && lane == 0) {
        *reinterpret_cast<volatile int *>(abort_flag) = 1;
        record_device_error(SQ_ERR_DEVICE_TIMEOUT);
      }
      tc_fence_after();
      const bool have = acc_ok && my_nk > 0;  // warp-uniform
      const int c = 32 * warp + lane;
      const bool mine = c >= keep_lo && c < keep_lo + keep_cols;
      int *dst = mine ? own + (c - keep_lo) : sendp + (c - peer_lo);
      const int stride = mine ? kDecKeepMax : peer_cols;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t v[32];
        if (have) {
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + 32 * h, v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int t = 0; t < 32; ++t) v[t] = 0;
        }
        if (c < tile_rows) {
#pragma unroll
          for (int t = 0; t < 32; ++t) dst[(32 * h + t) * stride] = static_cast<int>(v[t]);
        }
      }
      // the send buffer is read by the bulk copy (async proxy)
      fence_proxy_async_shared();
    }
    // the peer has finished with its receive buffer (previous tile)
    cluster_wait();
    group_bar(kBarEpi, kDecEpiThreads);
    if (etid == 0 && peer_cols > 0) {
      bulk_copy_to_cta(map_to_rank(smem_u32(recv), peer), sendp,
                       static_cast<uint32_t>(kDecMaxM * peer_cols * 4),
                       map_to_rank(smem_u32(&ctl.rbar), peer));
      bulk_commit_group();
    }
    if (etid == 32) mbar_arrive_expect_tx(&ctl.rbar, static_cast<uint32_t>(kDecMaxM * keep_cols * 4));
    // ---- epilogue: channel keep_lo + lane, tokens [8*warp, 8*warp + 8)
    const bool live = lane < keep_cols && n < N;
    const uint16_t *brow = B_pack + (live ? n : 0) * R;
    float *T = t_own;
    if (lora && rmax > 0 && !ctl.t_early) {
      // T had no room of its own: it goes where the stages were
      T = reinterpret_cast<float *>(ring + kDecTOff);
      asm volatile("griddepcontrol.wait;" ::: "memory");
      decode_form_t<2>(T, tstride, part, M, ksplit, mt, ctl, etid, kDecEpiThreads);
      group_bar(kBarEpi, kDecEpiThreads);
    }
    // the B' words go out before the peer's partials are awaited: whole
    // rows by bulk copies when the tokens read most of them, else each
    // thread's words by cp.async
    const bool b_rows = lora && ctl.b_dense;
    const int b_nrows =
        static_cast<int>(max(static_cast<int64_t>(0),
                             min(static_cast<int64_t>(keep_cols), N - (n0 + keep_lo))));
    const bool b_staged = lora && !b_rows && rmax <= 16;
    if (live && b_staged) decode_stage_b(bst, etid, brow, 8 * warp, 0, mt, ctl);
    if (!mbar_wait(&ctl.rbar, static_cast<uint32_t>(it) & 1u, timeout_ns, abort_flag)) {
      *reinterpret_cast<volatile int *>(abort_flag) = 1;
      record_device_error(SQ_ERR_DEVICE_TIMEOUT);
    }
    if (b_rows && b_nrows > 0 &&
        !mbar_wait(&ctl.bbar, static_cast<uint32_t>(it) & 1u, timeout_ns, abort_flag)) {
      *reinterpret_cast<volatile int *>(abort_flag) = 1;
      record_device_error(SQ_ERR_DEVICE_TIMEOUT);
    }
    if (b_staged) cp_async_wait_all();
    // one rolled loop over the thread's tokens: the epilogue runs once per
    // CTA, so its code is fetched cold and is kept short
    if (live && *abort_flag == 0) {
      const uint8_t *mine_row = bst + lane * brow_stride;
#pragma unroll 1
      for (int u = 0; u < 8; ++u) {
        const int tok = 8 * warp + u;
        if (tok >= mt) break;
        const int r = lora ? ctl.tok_rank[tok] : 0;
        const int off = ctl.tok_off[tok];
        float d = 0.f;
#pragma unroll 1
        for (int j = 0; j < r; j += 8) {
          // the 8 B' words [j, j + 8): from the kept rows, this thread's
          // staged words, or (a sparse pack with ranks above 16) global memory
          uint4 w;
          if (b_rows)
            w = *reinterpret_cast<const uint4 *>(mine_row + (off + j) * 2);
          else if (b_staged)
            w = *reinterpret_cast<const uint4 *>(
                bst + ((2 * u + (j >> 3)) * kDecEpiThreads + etid) * 16);
          else
            w = __ldg(reinterpret_cast<const uint4 *>(brow + off + j));
          const float *Ti = T + tok * tstride + j;
          d = dot8_bf16(w, *reinterpret_cast<const float4 *>(Ti),
                        *reinterpret_cast<const float4 *>(Ti + 4), d);
        }
        const int acc = own[tok * kDecKeepMax + lane] + recv[tok * keep_cols + lane];
        if (mode == 0) {
          const float y =
              __fadd_rn(__fmul_rn(__fmul_rn(__int2float_rn(acc), ctl.xs[tok]), ws_n), d);
          static_cast<__nv_bfloat16 *>(out)[tok * N + n] = __float2bfloat16_rn(y);
        } else if (mode == 1) {
          static_cast<int32_t *>(out)[tok * N + n] = acc;
        } else {
          static_cast<float *>(out)[tok * N + n] = d;
        }
      }
    }
    // (copies issued by a thread that then skipped the epilogue)
    cp_async_wait_all();
    // the send buffer has been read before the ring is reused
    if (etid == 0 && peer_cols > 0) bulk_wait_group_read<0>();
    tc_fence_before();
    group_bar(kBarTileEnd, kDecGemmThreads);
    cluster_arrive();
  }
  if (warp >= kDecFirstLoader) drain_loads();
  // before exit: the last tile's MMAs and the peer's copy into this CTA have
  // completed (also when a wait above ran out)
  if (etid == 0 && it > 0) {
    volatile int never = 0;
    mbar_wait(&ctl.accfull, static_cast<uint32_t>(it - 1) & 1u, 1000000000ull, &never);
    mbar_wait(&ctl.rbar, static_cast<uint32_t>(it - 1) & 1u, 1000000000ull, &never);
  }
  if (etid == 32 && it > 0 && lora && ctl.b_dense) {
    // the last tile's B' rows (issued by this thread whenever a row existed)
    volatile int never = 0;
    const int64_t nl = static_cast<int64_t>(pair + (it - 1) * npairs) * tile_rows + keep_lo;
    if (keep_cols > 0 && nl < N)
      mbar_wait(&ctl.bbar, static_cast<uint32_t>(it - 1) & 1u, 1000000000ull, &never);
  }
  cluster_wait();
  group_bar(kBarEpi, kDecEpiThreads);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kDecTmemCols);
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
  CUtensorMap tm_x;
  memset(&tm_x, 0, sizeof tm_x);
  // K a multiple of 128: one 3D Xq box per stage; otherwise one 2D box per K
  // block (the last block's tail is filled with zeros)
  const int view3d = (K % 128 == 0) ? 1 : 0;
  if (mode != 2) {
    const bool made = view3d ? make_tmap_kblocks(&tm_x, Xq, K, M, kDecMaxM, kDecKbStage)
                             : make_tmap(&tm_x, Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, M, 128,
                                         kDecMaxM);
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
  return cudaLaunchKernelEx(&cfg, decode_gemm_kernel, tm_x, view3d, Wq, x_scale, w_scale, M, N, K,
                            mode, B_pack, lora_offset, lora_rank, n_adapters, R, seg_offsets,
                            seg_adapter, S, lora ? static_cast<const float *>(part) : nullptr,
                            ksplit, tile_units, static_cast<int>(tiles), out, wait_timeout_ns());
}

}  // namespace sq
