// Small-M (decode) form of the W8A8 + LoRA linear ("SmoothQuant" explainer,
// Step 7 and "Smaller gain at small batches ... memory-bound"; "[Feature]:
// LoRA support for W8A8 SmoothQuant", Pitch and Motivation: one adapter per
// request).  With a few dozen tokens the layer is bound by streaming Wq and
// the adapters from HBM, so the work is spread over output-channel slices
// rather than 256x256 tiles:
//   kernel 1 (shrink)   one warp per (token, K slice): partial sums of
//                       T[i,:] = x_scale_i * Xq[i,:] A_a^T over the slice,
//                       written to a scratch table (no atomics: the sums are
//                       later added in a fixed order); it lets the GEMM grid
//                       launch at once, so the weight stream overlaps it;
//   kernel 2 (GEMM + expand), one block per 32 output channels:
//                       acc = Xq Wq^T with int8 tensor-core MMAs (m16n8k32,
//                       exact int32) from a TMA-fed ring of Wq tiles; then,
//                       after the shrink grid has completed (programmatic
//                       dependent launch: the weight stream starts before the
//                       shrink finishes), delta = T B_a^T in fp32 and
//                       Y = bf16(acc*xs*ws + delta).
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx_sm100.cuh"
#include "tmap.cuh"

namespace sq {

constexpr int kDecMaxM = 64;       // token rows handled by this form
constexpr int kDecMaxRank = 256;   // largest adapter rank (the library-wide limit)
constexpr int kDecKSplit = 16;     // K slices of the shrink
constexpr int kDecCols = 32;       // output channels per GEMM block
constexpr int kDecThreads = 256;

// ---------------------------------------------------------------------------
// kernel 1: shrink partials.  part[(i * kDecKSplit + ks) * kDecMaxRank + j]
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kDecThreads, 1) decode_shrink_kernel(
    const int8_t *__restrict__ Xq, const float *__restrict__ x_scale, int64_t M, int64_t K,
    const uint16_t *__restrict__ A_pack, const int32_t *__restrict__ lora_offset,
    const int32_t *__restrict__ lora_rank, int n_adapters, int64_t R,
    const int32_t *__restrict__ seg_offsets, const int32_t *__restrict__ seg_adapter, int64_t S,
    float *__restrict__ part) {
  // the dependent GEMM grid may launch at once: its weight stream needs
  // nothing from here, and it waits for this grid to complete before it
  // reads the partial sums
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.x * (kDecThreads / 32) + warp;  // (token, K slice)
  const int64_t i = unit / kDecKSplit;
  const int ks = unit % kDecKSplit;
  if (i >= M) return;
  int a = token_adapter(seg_offsets, seg_adapter, S, n_adapters, i);
  int off = 0, r = 0;
  if (a >= 0) {
    off = lora_offset[a];
    r = lora_rank[a];
    if (off < 0 || (off & 15) || r <= 0 || r > kDecMaxRank || off + ((r + 15) & ~15) > R) {
      if (lane == 0) record_device_error(SQ_ERR_BAD_SEGMENTS);
      r = 0;
    }
  }
  float *out = part + (i * kDecKSplit + ks) * kDecMaxRank;
  // K slice of this warp, in 16-element pieces (K % 16 == 0); lane = piece
  // (lane & 15) of each group of 16 pieces x half (lane >> 4) of each group
  // of 16 ranks, so that all lanes load at once
  const int64_t pieces = K / 16;
  const int64_t p0 = pieces * ks / kDecKSplit, p1 = pieces * (ks + 1) / kDecKSplit;
  const int pl = lane & 15, hf = lane >> 4;
  // the codes and scales come from the quantizer (a no-op unless this grid
  // is launched as its programmatic dependent)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const float xs = x_scale[i];
  for (int j0 = 0; j0 < r; j0 += 16) {
    const int jb = j0 + 8 * hf;  // this lane's 8 ranks (rows up to the padded rank exist)
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    for (int64_t p = p0 + pl; p < p1; p += 16) {
      // all loads of this piece first, then the products
      const uint4 xr = __ldg(reinterpret_cast<const uint4 *>(Xq + i * K + p * 16));
      uint4 av[8][2];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint16_t *ap = A_pack + static_cast<int64_t>(off + jb + j) * K + p * 16;
        av[j][0] = __ldg(reinterpret_cast<const uint4 *>(ap));
        av[j][1] = __ldg(reinterpret_cast<const uint4 *>(ap + 8));
      }
      const uint32_t w4[4] = {xr.x, xr.y, xr.z, xr.w};
      float xv[16];
#pragma unroll
      for (int t = 0; t < 16; ++t)
        xv[t] = static_cast<float>(static_cast<int8_t>((w4[t >> 2] >> (8 * (t & 3))) & 0xff));
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t a8[8] = {av[j][0].x, av[j][0].y, av[j][0].z, av[j][0].w,
                                av[j][1].x, av[j][1].y, av[j][1].z, av[j][1].w};
        float sacc = 0.f;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          sacc = fmaf(xv[2 * t], __uint_as_float(a8[t] << 16), sacc);
          sacc = fmaf(xv[2 * t + 1], __uint_as_float(a8[t] & 0xffff0000u), sacc);
        }
        acc[j] += sacc;
      }
    }
    // sum over the 16 piece lanes of each half, in a fixed order
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float v = acc[j];
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (pl == 0 && jb + j < r) out[jb + j] = xs * v;
    }
  }
}

// ---------------------------------------------------------------------------
// kernel 2: int8 GEMM over 32 output channels, then the LoRA expand.
// Warp 8 streams this block's 32 rows of Wq and the tokens' Xq through a ring
// of stages of 256 K-bytes, each two 128-byte-wide TMA tiles per operand
// (128-byte swizzle: the 8 rows an MMA fragment load touches sit in distinct
// banks); the four copies of a stage are issued by four lanes in one warp
// instruction, since one thread's copies are issued one after another.
// Compute warp w owns tokens [16*(w&3), +16) and channels [16*(w>>2), +16)
// over the whole K, so no cross-warp reduction is needed.
// ---------------------------------------------------------------------------
constexpr int kDecStages = 8;
constexpr int kDecKStage = 256;                   // K bytes per stage (two tiles)
constexpr int kDecWBytes = kDecCols * 128;        // Wq tile: 32 rows x 128 K-bytes
constexpr int kDecXBytes = kDecMaxM * 128;        // Xq tile: 64 rows x 128 K-bytes
constexpr int kDecStageBytes = 2 * (kDecWBytes + kDecXBytes);
constexpr int kDecComputeWarps = 8;
constexpr int kDecGemmThreads = 32 * (kDecComputeWarps + 1);

__device__ __forceinline__ void mma_s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

struct DecodeCtl {
  uint64_t full[kDecStages];
  uint64_t empty[kDecStages];
  int off[kDecMaxM];               // adapter column offset per token
  int rank[kDecMaxM];              // adapter rank per token (0: none)
  int abort;
};
// the LoRA intermediate T[kDecMaxM][kDecMaxRank] (fp32) reuses the ring once
// the K loop is over
static_assert(kDecStages * kDecStageBytes >= kDecMaxM * kDecMaxRank * 4, "T must fit the ring");
static_assert(32 * 8 == 4 * kDecMaxM, "four T threads per token");

constexpr size_t kDecSmemBytes = static_cast<size_t>(kDecStages) * kDecStageBytes + sizeof(DecodeCtl) + 1024;

__global__ void __launch_bounds__(kDecGemmThreads) decode_gemm_kernel(
    const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
    const float *__restrict__ x_scale, const float *__restrict__ w_scale, int64_t M, int64_t N,
    int64_t K, int mode, const uint16_t *__restrict__ B_pack,
    const int32_t *__restrict__ lora_offset, const int32_t *__restrict__ lora_rank,
    int n_adapters, int64_t R, const int32_t *__restrict__ seg_offsets,
    const int32_t *__restrict__ seg_adapter, int64_t S, const float *__restrict__ part,
    void *__restrict__ out, uint64_t timeout_ns) {
  extern __shared__ uint8_t dsm_raw[];
  uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  DecodeCtl &ctl = *reinterpret_cast<DecodeCtl *>(ring + kDecStages * kDecStageBytes);
  volatile int *abort_flag = &ctl.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kDecCols;
  const bool lora = (part != nullptr);
  const int nk = (mode == 2) ? 0 : static_cast<int>((K + kDecKStage - 1) / kDecKStage);
  const int kb_first = (nk > 0) ? static_cast<int>((blockIdx.x * 5u) % static_cast<unsigned>(nk)) : 0;

  if (threadIdx.x == 0) {
    for (int st = 0; st < kDecStages; ++st) {
      mbar_init(&ctl.full[st], 1);
      mbar_init(&ctl.empty[st], kDecComputeWarps);
    }
    ctl.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kDecComputeWarps) {
    // ---------------------------------------------------------- producer
    // lane 0 waits for a free stage and posts its bytes; lanes 0-3 then copy
    // Wq tile 0, Wq tile 1, Xq tile 0 and Xq tile 1 of the stage together
    int issued = 0;
    {
      if (lane == 0) {
        prefetch_tmap(&tm_w);
        prefetch_tmap(&tm_x);
      }
      uint32_t phase = 0;
      int st = 0;
      // blocks start their K walk at different stages so that they do not
      // all read the same Xq tile (from the same L2 lines) at once
      int kk = kb_first;
      for (int kb = 0; kb < nk; ++kb) {
        bool got = true;
        if (lane == 0) {
          got = mbar_wait(&ctl.empty[st], phase ^ 1u, timeout_ns, abort_flag);
          if (got) mbar_arrive_expect_tx(&ctl.full[st], kDecStageBytes);
        }
        if (!__shfl_sync(0xffffffffu, got, 0)) {
          if (lane == 0) {
            *reinterpret_cast<volatile int *>(abort_flag) = 1;
            record_device_error(SQ_ERR_DEVICE_TIMEOUT);
          }
          break;
        }
        if (lane < 4) {
          const int tile = lane & 1;  // K half of the stage
          const int32_t x = kk * kDecKStage + tile * 128;
          if (lane < 2)
            tma_load_2d(ring + st * kDecStageBytes + tile * kDecWBytes, &tm_w, &ctl.full[st], x,
                        static_cast<int32_t>(n0));
          else
            tma_load_2d(ring + st * kDecStageBytes + 2 * kDecWBytes + tile * kDecXBytes, &tm_x,
                        &ctl.full[st], x, 0);
        }
        ++issued;
        if (++kk == nk) kk = 0;
        if (++st == kDecStages) { st = 0; phase ^= 1u; }
      }
    }
    if (lane == 0) {
      // every issued copy must land before the block exits: wait for the
      // last use of each stage
      volatile int never = 0;
      for (int s2 = 0; s2 < kDecStages && s2 < issued; ++s2) {
        const int last_kb = issued - 1 - ((issued - 1 - s2) % kDecStages);
        const uint32_t par = static_cast<uint32_t>((last_kb / kDecStages) & 1);
        mbar_wait(&ctl.full[s2], par, 1000000000ull, &never);
      }
    }
  } else {
    // --------------------------------------------------------- compute
    const int mt = warp & 3, nh = warp >> 2;
    int acc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][e] = 0;
    const int ra = mt * 16 + g, rb = ra + 8;  // token rows of this lane's A fragments
    // adapter of each token (warps 0-3 cover the 64 tokens), looked up while
    // the first stages load; read by all compute warps after the K loop
    if (lora && nh == 0 && lane < 16) {
      const int i = mt * 16 + lane;
      int off = 0, r = 0;
      if (i < M) {
        const int a = token_adapter(seg_offsets, seg_adapter, S, n_adapters, i);
        if (a >= 0) {
          off = lora_offset[a];
          r = lora_rank[a];
          if (off < 0 || (off & 15) || r <= 0 || r > kDecMaxRank || off + ((r + 15) & ~15) > R)
            r = 0;
        }
      }
      ctl.off[i] = off;
      ctl.rank[i] = r;
    }
    uint32_t phase = 0;
    int st = 0;
    bool ok = true;
    for (int kb = 0; kb < nk; ++kb) {
      // the warp leaves together: the mma.sync below needs all lanes
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&ctl.full[st], phase, timeout_ns, abort_flag))))
        break;
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) {
        const int h = hh & 1;  // 64-byte half of a 128-byte tile row
        const uint8_t *wt = ring + st * kDecStageBytes + (hh >> 1) * kDecWBytes;
        const uint8_t *xt = ring + st * kDecStageBytes + 2 * kDecWBytes + (hh >> 1) * kDecXBytes;
        // 16 contiguous K bytes (chunk 4h + tig of the 128-byte row, stored
        // 128B-swizzled) of each operand row; the K order inside the 64 bytes
        // is a permutation that A and B share
        const uint4 xa = *reinterpret_cast<const uint4 *>(xt + ra * 128 + (((4 * h + tig) ^ (ra & 7)) * 16));
        const uint4 xb = *reinterpret_cast<const uint4 *>(xt + rb * 128 + (((4 * h + tig) ^ (rb & 7)) * 16));
        const uint32_t fa0[4] = {xa.x, xb.x, xa.y, xb.y};
        const uint32_t fa1[4] = {xa.z, xb.z, xa.w, xb.w};
        uint4 bw[2];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int row = nh * 16 + nt * 8 + g;
          bw[nt] = *reinterpret_cast<const uint4 *>(wt + row * 128 + (((4 * h + tig) ^ (row & 7)) * 16));
        }
        // independent accumulators back to back
        mma_s8_16832(acc[0], fa0, bw[0].x, bw[0].y);
        mma_s8_16832(acc[1], fa0, bw[1].x, bw[1].y);
        mma_s8_16832(acc[0], fa1, bw[0].z, bw[0].w);
        mma_s8_16832(acc[1], fa1, bw[1].z, bw[1].w);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.empty[st]);
      if (++st == kDecStages) { st = 0; phase ^= 1u; }
    }
    if (!ok) {
      *reinterpret_cast<volatile int *>(abort_flag) = 1;
      record_device_error(SQ_ERR_DEVICE_TIMEOUT);
    }
    // ---- LoRA: every compute warp has finished reading the ring (T may
    //      overwrite it) and the adapter table is complete; the B' columns of
    //      the first 16 ranks are loaded before the shrink's partial sums are
    //      waited for, then T = sum of the partials over the shrink's K slices.
    //      Every compute warp meets both barriers, also after a wait that ran out.
    float (*Tm)[kDecMaxRank] = reinterpret_cast<float (*)[kDecMaxRank]>(ring);
    asm volatile("bar.sync 1, %0;" ::"r"(32 * kDecComputeWarps) : "memory");
    // lane: rows ra, rb; channels n0 + 16nh + 8nt + 2tig + {0,1}
    float d[2][2][2];  // [half][nt][channel of the pair]
    int rr[2], oo[2];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int i = half ? rb : ra;
      rr[half] = (lora && i < M) ? ctl.rank[i] : 0;
      oo[half] = (lora && i < M) ? ctl.off[i] : 0;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) d[half][nt][0] = d[half][nt][1] = 0.f;
    }
    const int rmax = max(rr[0], rr[1]);
    auto load_b = [&](int j0, uint4 (&bv)[2][2][2]) {
#pragma unroll
      for (int half = 0; half < 2; ++half)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int64_t n = n0 + nh * 16 + nt * 8 + 2 * tig;
#pragma unroll
          for (int c = 0; c < 2; ++c)
            bv[half][nt][c] = (j0 < rr[half] && n + c < N)
                                  ? __ldg(reinterpret_cast<const uint4 *>(B_pack + (n + c) * R + oo[half] + j0))
                                  : make_uint4(0, 0, 0, 0);
        }
    };
    uint4 bpre[2][2][2][2];  // column groups 0 and 1 (ranks 0-15), loaded early
    load_b(0, bpre[0]);
    load_b(8, bpre[1]);
    if (lora) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      // four threads per token, each summing every fourth column; the 16
      // partials of four columns are loaded before any is added
      const int i = threadIdx.x >> 2, jq = threadIdx.x & 3;
      const int r = (i < M) ? ctl.rank[i] : 0;
      const int rpad = (r + 15) & ~15;
      for (int jb = 0; jb < rpad; jb += 16) {
        float pv[4][kDecKSplit];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int j = jb + jq + 4 * m;
#pragma unroll
          for (int ks = 0; ks < kDecKSplit; ++ks)
            pv[m][ks] = (j < r) ? part[(i * kDecKSplit + ks) * kDecMaxRank + j] : 0.f;
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          float t = 0.f;  // zero in the padding columns (the expand reads them)
#pragma unroll
          for (int ks = 0; ks < kDecKSplit; ++ks) t += pv[m][ks];
          Tm[i][jb + jq + 4 * m] = t;
        }
      }
      asm volatile("bar.sync 1, %0;" ::"r"(32 * kDecComputeWarps) : "memory");
    }
    for (int j0 = 0; j0 < rmax; j0 += 8) {
      uint4 bv[2][2][2];  // [half][nt][channel]
      if (j0 == 0) {
#pragma unroll
        for (int half = 0; half < 2; ++half)
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) bv[half][nt][c] = bpre[0][half][nt][c];
      } else if (j0 == 8) {
#pragma unroll
        for (int half = 0; half < 2; ++half)
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) bv[half][nt][c] = bpre[1][half][nt][c];
      } else {
        load_b(j0, bv);
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        if (j0 >= rr[half]) continue;
        const int i = half ? rb : ra;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const uint32_t w[4] = {bv[half][nt][c].x, bv[half][nt][c].y, bv[half][nt][c].z,
                                   bv[half][nt][c].w};
            float acc_d = d[half][nt][c];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              acc_d = fmaf(Tm[i][j0 + 2 * t], __uint_as_float(w[t] << 16), acc_d);
              acc_d = fmaf(Tm[i][j0 + 2 * t + 1], __uint_as_float(w[t] & 0xffff0000u), acc_d);
            }
            d[half][nt][c] = acc_d;
          }
      }
    }
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int64_t i = half ? rb : ra;
      if (i >= M) continue;
      const float xs = (mode == 0) ? x_scale[i] : 0.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int64_t n = n0 + nh * 16 + nt * 8 + 2 * tig;
        if (n >= N) continue;  // N % 16 == 0: both channels of the pair exist
        const int s0 = acc[nt][2 * half], s1 = acc[nt][2 * half + 1];
        const float d0 = d[half][nt][0], d1 = d[half][nt][1];
        if (mode == 0) {
          const float y0 = __fadd_rn(__fmul_rn(__fmul_rn(__int2float_rn(s0), xs), __ldg(w_scale + n)), d0);
          const float y1 = __fadd_rn(__fmul_rn(__fmul_rn(__int2float_rn(s1), xs), __ldg(w_scale + n + 1)), d1);
          __nv_bfloat162 hh = __floats2bfloat162_rn(y0, y1);
          *reinterpret_cast<uint32_t *>(static_cast<uint16_t *>(out) + i * N + n) =
              *reinterpret_cast<uint32_t *>(&hh);
        } else if (mode == 1) {
          *reinterpret_cast<int2 *>(static_cast<int32_t *>(out) + i * N + n) = make_int2(s0, s1);
        } else {
          *reinterpret_cast<float2 *>(static_cast<float *>(out) + i * N + n) = make_float2(d0, d1);
        }
      }
    }
  }
}

size_t decode_workspace_bytes(int64_t M) {
  return static_cast<size_t>(M) * kDecKSplit * kDecMaxRank * sizeof(float);
}

bool decode_applicable(int64_t M) { return M > 0 && M <= kDecMaxM; }

// mode: 0 = Y bf16, 1 = int32 accumulators, 2 = LoRA delta fp32.
// `part` (scratch, decode_workspace_bytes(M)) may be null when there is no LoRA.
cudaError_t launch_decode(const int8_t *Xq, const float *x_scale, const int8_t *Wq,
                          const float *w_scale, int64_t M, int64_t N, int64_t K, int mode,
                          const uint16_t *A_pack, const uint16_t *B_pack,
                          const int32_t *lora_offset, const int32_t *lora_rank, int n_adapters,
                          int64_t R, const int32_t *seg_offsets, const int32_t *seg_adapter,
                          int64_t S, float *part, void *out, cudaStream_t st) {
  const bool lora = part != nullptr && mode != 1;
  if (lora) {
    const int units = static_cast<int>(M) * kDecKSplit;
    const int blocks = (units + kDecThreads / 32 - 1) / (kDecThreads / 32);
    decode_shrink_kernel<<<blocks, kDecThreads, 0, st>>>(Xq, x_scale, M, K, A_pack, lora_offset,
                                                         lora_rank, n_adapters, R, seg_offsets,
                                                         seg_adapter, S, part);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  CUtensorMap tm_w, tm_x;
  memset(&tm_w, 0, sizeof tm_w);
  memset(&tm_x, 0, sizeof tm_x);
  if (mode != 2 &&
      (!make_tmap(&tm_w, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, N, 128, kDecCols) ||
       !make_tmap(&tm_x, Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, M, 128, kDecMaxM)))
    return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(decode_gemm_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kDecSmemBytes));
    if (e != cudaSuccess) return e;
    attr = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((N + kDecCols - 1) / kDecCols), 1, 1);
  cfg.blockDim = dim3(kDecGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = kDecSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = lora ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, decode_gemm_kernel, tm_w, tm_x, x_scale, w_scale, M, N, K, mode,
                            B_pack, lora_offset, lora_rank, n_adapters, R, seg_offsets,
                            seg_adapter, S, lora ? static_cast<const float *>(part) : nullptr, out,
                            wait_timeout_ns());
}

}  // namespace sq
