// Forward and backward of the NF4 frozen-base LoRA linear layer on sm_100a.
//
// Page "QLoRA：冻结的 4-bit 权重怎样参与一次微调":
//   §量化基座与可训练支路怎样相加      Z = X·A,  Y = X·Ŵ + c·Z·B
//   §冻结权重为什么仍然需要输入梯度    dZ = c·G·Bᵀ, dX = G·Ŵᵀ + dZ·Aᵀ,
//                                     dA = Xᵀ·dZ,  dB = c·Zᵀ·G
//
// Kernels in this file:
//   skinny_gemm_kernel   rank-r contractions (X·A, G·Bᵀ, Xᵀ·dZ, Gᵀ·Zc): TMA
//                        for both operands, tcgen05 MMA with N = 64, split-K
//                        into fp32 partials; the last split of each row
//                        tile adds them and writes the result.
//   fused_nf4_gemm_kernel  Y = X·Ŵ + Zc·B (forward) and dX = G·Ŵᵀ + dZ·Aᵀ
//                        (backward): persistent, warp-specialised; TMA brings
//                        activation tiles and packed-nibble tiles, decoder
//                        warps turn nibbles into bf16 operand tiles in shared
//                        memory, one thread issues tcgen05.mma into TMEM, and
//                        the rank-r LoRA term is one extra K-step of the same
//                        accumulator.
// The M <= 16 forward (a GEMV) is in gemv.cu.
#include <atomic>
#include <cfloat>
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "profile.cuh"
#include "tmap.cuh"

namespace qnf4 {

// code values of the two codebooks: [0, 16) NF4, [16, 32) uniform INT4
__constant__ float kNF4g[32] = {QNF4_TABLE_VALUES, QNF4_INT4_VALUES};

// ===========================================================================
// Skinny contraction:  D[m'][n'] = sum_k' A(m',k') * B(n',k'),  n' < 64.
// A tiles are 128 x 64 and B tiles 64 x 64 (bf16), each either K-major
// (rows of 64 contiguous k') or MN-major (rows of 64 contiguous m'/n'), all
// with the 128-byte swizzle.  blockIdx.x = 128-row tile, blockIdx.y = split.
// ===========================================================================
constexpr int kSkW = 2;                  // 64-wide k' boxes per stage
constexpr int kSkStages = 8 / kSkW;
constexpr int kSkA = 16384 * kSkW, kSkB = 8192 * kSkW;
constexpr int kSkThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr size_t kSkSmem = 1024 + kSkStages * (kSkA + kSkB) + 256;
static_assert(kSkStages * 8 * 3 + 16 <= 256, "skinny barriers and flags fit the tail");

struct SkinnyArgs {
  int Mp;            // rows of D
  int nk;            // number of k' blocks (64 * kSkW wide)
  int kb_per_split;  // k' blocks per split
  int splits;        // = cluster size along y (<= 8)
  int ncols;         // columns of D that are summed (the rank, or the padded rank)
  int nout;          // columns written to `out` (<= ncols)
  float scale;
  int mode;          // 0: bf16 out[Mp][ld]; 1: fp32 out[Mp][ld]; 2: fp32 out[nout][Mp]
  void* out;
  int ld;
  uint16_t* out2;    // mode 0 only, may be null: all ncols columns again, bf16 [Mp][ld2]
  int ld2;
  int32_t* d_status;
};

constexpr int kSkRedLd = 65;   // fp32 words per row of the split-sum buffer (bank spread)
constexpr int kSkMaxSplits = 8;  // portable cluster size

template <bool kAmn, bool kBmn>
__global__ void __launch_bounds__(kSkThreads, 1)
    skinny_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB, SkinnyArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kSkStages * kSkA;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kSkStages * kSkB);
  uint64_t* empty = full + kSkStages;
  uint64_t* done = empty + kSkStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_holder + 1);
  float* red = reinterpret_cast<float*>(sA);   // [128][kSkRedLd], after the last MMA

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128;
  const int kb0 = blockIdx.y * args.kb_per_split;
  const int kb1 = min(args.nk, kb0 + args.kb_per_split);
  const int nkb = kb1 - kb0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSkStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // Wait for the preceding kernel first and only then let the next one
  // launch: the fused kernel that follows a rank-r product then knows that
  // every kernel before this one has completed, and reads its activations
  // and weights at once, waiting only for this kernel's result.
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    for (int i = 0; i < nkb; ++i) {
      const int s = i % kSkStages;
      const uint32_t ph = (i / kSkStages) & 1;
      if (!mbar_wait(&empty[s], ph ^ 1)) { *abort_flag = 1; break; }
      const int kb = kb0 + i;
      mbar_arrive_expect_tx(&full[s], kSkA + kSkB);
#pragma unroll
      for (int w = 0; w < kSkW; ++w) {
        const int kx = (kb * kSkW + w) * 64;   // boxes past the end arrive as zero fill
        uint8_t* a = sA + s * kSkA + w * 16384;
        uint8_t* b = sB + s * kSkB + w * 8192;
        if (kAmn) {
          tma_load_2d(a, &tmA, &full[s], m0, kx);
          tma_load_2d(a + 8192, &tmA, &full[s], m0 + 64, kx);
        } else {
          tma_load_2d(a, &tmA, &full[s], kx, m0);
        }
        if (kBmn)
          tma_load_2d(b, &tmB, &full[s], 0, kx);
        else
          tma_load_2d(b, &tmB, &full[s], kx, 0);
      }
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(128, 64, kAmn ? 1 : 0, kBmn ? 1 : 0);
    bool ok = true;
    for (int i = 0; i < nkb; ++i) {
      const int s = i % kSkStages;
      const uint32_t ph = (i / kSkStages) & 1;
      if (!mbar_wait(&full[s], ph)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int w = 0; w < kSkW; ++w) {
        const uint32_t a0 = smem_u32(sA + s * kSkA + w * 16384), b0 = smem_u32(sB + s * kSkB + w * 8192);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t ad = kAmn ? smem_desc(a0 + j * 2048, 8192, 1024) : smem_desc(a0 + j * 32, 16, 1024);
          const uint64_t bd = kBmn ? smem_desc(b0 + j * 2048, 8192, 1024) : smem_desc(b0 + j * 32, 16, 1024);
          umma_bf16(tmem, ad, bd, idesc, (i > 0 || w > 0 || j > 0) ? 1u : 0u);
        }
      }
      umma_commit(&empty[s]);
    }
    if (!ok) *abort_flag = 1;
    umma_commit(done);  // also drains whatever was issued
  } else if (warp >= 2) {
    // Epilogue, part 1: this split's fp32 sums into shared memory (the A ring
    // is free once the last MMA has completed).
    const int q = warp & 3;
    const bool okd = mbar_wait(done, 0);
    tc_fence_after();
    if (!okd) *abort_flag = 1;
    const int row = q * 32 + lane;
    const int nc = args.ncols;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      if (c * 32 < nc) {
        uint32_t v[32];
        if (okd) {
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + c * 32, v);
          tmem_ld_wait();
        }
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (c * 32 + i < nc) red[row * kSkRedLd + c * 32 + i] = okd ? __uint_as_float(v[i]) : 0.0f;
      }
    }
  }
  // Part 2: the splits of a row tile are one thread-block cluster along y.
  // Each adds a share of the tile's rows over all splits, in split order,
  // reading the others' sums from distributed shared memory, and writes out.
  cluster_sync_all();
  if (warp >= 2) {
    const int S = args.splits;
    const int rank = static_cast<int>(blockIdx.y);   // cluster spans all of y
    const int rows_per = (128 + S - 1) / S;
    const int r0 = rank * rows_per;
    const int nrow = min(rows_per, 128 - r0);
    const int nc = args.ncols;
    const int total = nrow > 0 ? nrow * nc : 0;
    const uint32_t red_s = smem_u32(red);
    for (int e = threadIdx.x - 64; e < total; e += 128) {
      // mode 2 writes columns of out: let consecutive threads take consecutive rows
      const int rr = args.mode == 2 ? e % nrow : e / nc;
      const int cc = args.mode == 2 ? e / nrow : e % nc;
      const int lrow = r0 + rr, grow = m0 + lrow;
      // all S loads in flight first, then the sum in split order
      const uint32_t off = red_s + static_cast<uint32_t>((lrow * kSkRedLd + cc) * 4);
      float part[kSkMaxSplits];
#pragma unroll
      for (int sp = 0; sp < kSkMaxSplits; ++sp)
        part[sp] = sp < S ? ld_dsmem_f32(off, static_cast<uint32_t>(sp)) : 0.0f;
      float acc = 0.0f;
#pragma unroll
      for (int sp = 0; sp < kSkMaxSplits; ++sp)
        if (sp < S) acc += part[sp];
      acc *= args.scale;
      if (grow < args.Mp) {
        if (args.mode == 0) {
          const uint16_t v = static_cast<uint16_t>(pack_bf16x2(acc, 0.0f) & 0xFFFFu);
          if (cc < args.nout) static_cast<uint16_t*>(args.out)[static_cast<int64_t>(grow) * args.ld + cc] = v;
          if (args.out2 != nullptr) args.out2[static_cast<int64_t>(grow) * args.ld2 + cc] = v;
        } else if (cc < args.nout) {
          if (args.mode == 1)
            static_cast<float*>(args.out)[static_cast<int64_t>(grow) * args.ld + cc] = acc;
          else
            static_cast<float*>(args.out)[static_cast<int64_t>(cc) * args.Mp + grow] = acc;
        }
      }
    }
  }
  cluster_sync_all();   // no CTA leaves while another still reads its sums
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) raise_status(args.d_status, QLORA_ERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}


// ===========================================================================
// Rank-r product on a few SMs beside the fused GEMM:  D = scale * A B (the
// operand layouts and output modes of the split kernel above), the whole
// contraction per 128-row tile in one CTA (no split), tiles blockIdx.x,
// + gridDim.x, ...  The fused GEMM leaves these SMs free (its grid is sized
// to the fewest pairs that need no more waves of tiles): Zc (dZ) here lets
// it start at once and wait for the product only at its LoRA step, and dA,
// dB here run beside dX.  Same roles as above: warp 0 TMA, warp 1 MMA into
// one TMEM accumulator (128 x 64 fp32), warps 2..5 read it (released on
// `tempty` per tile), scale and store.
// ===========================================================================
template <bool kAmn, bool kBmn>
__global__ void __launch_bounds__(kSkThreads, 1)
    rank_rows_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB, SkinnyArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kSkStages * kSkA;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kSkStages * kSkB);
  uint64_t* empty = full + kSkStages;
  uint64_t* done = empty + kSkStages;
  uint64_t* tempty = done + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tempty + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = (args.Mp + 127) / 128;
  const int nkb = args.nk;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSkStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    mbar_init(tempty, 4);   // the four epilogue warps
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // wait for the preceding kernel, then let the fused GEMM launch
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    int g = 0;   // stage uses over all tiles
    bool ok = true;
    for (int t = blockIdx.x; t < m_tiles && ok; t += gridDim.x) {
      const int m0 = t * 128;
      for (int i = 0; i < nkb; ++i, ++g) {
        const int s = g % kSkStages;
        const uint32_t ph = (g / kSkStages) & 1;
        if (g >= kSkStages && !mbar_wait(&empty[s], ph ^ 1)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[s], kSkA + kSkB);
#pragma unroll
        for (int w = 0; w < kSkW; ++w) {
          const int kx = (i * kSkW + w) * 64;   // boxes past the end arrive as zero fill
          uint8_t* a = sA + s * kSkA + w * 16384;
          uint8_t* b = sB + s * kSkB + w * 8192;
          if (kAmn) {
            tma_load_2d(a, &tmA, &full[s], m0, kx);
            tma_load_2d(a + 8192, &tmA, &full[s], m0 + 64, kx);
          } else {
            tma_load_2d(a, &tmA, &full[s], kx, m0);
          }
          if (kBmn)
            tma_load_2d(b, &tmB, &full[s], 0, kx);
          else
            tma_load_2d(b, &tmB, &full[s], kx, 0);
        }
      }
    }
    if (!ok) *abort_flag = 1;
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(128, 64, kAmn ? 1 : 0, kBmn ? 1 : 0);
    int g = 0, it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < m_tiles && ok; t += gridDim.x, ++it) {
      // the epilogue has read the previous tile's accumulator
      if (it > 0 && !mbar_wait(tempty, (it - 1) & 1)) { ok = false; break; }
      tc_fence_after();
      for (int i = 0; i < nkb; ++i, ++g) {
        const int s = g % kSkStages;
        const uint32_t ph = (g / kSkStages) & 1;
        if (!mbar_wait(&full[s], ph)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int w = 0; w < kSkW; ++w) {
          const uint32_t a0 = smem_u32(sA + s * kSkA + w * 16384), b0 = smem_u32(sB + s * kSkB + w * 8192);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t ad = kAmn ? smem_desc(a0 + j * 2048, 8192, 1024) : smem_desc(a0 + j * 32, 16, 1024);
            const uint64_t bd = kBmn ? smem_desc(b0 + j * 2048, 8192, 1024) : smem_desc(b0 + j * 32, 16, 1024);
            umma_bf16(tmem, ad, bd, idesc, (i > 0 || w > 0 || j > 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty[s]);
      }
      umma_commit(done);   // one phase per tile (also drains an aborted tile)
    }
    if (!ok) *abort_flag = 1;
  } else if (warp >= 2) {
    const int q = warp & 3;   // TMEM lanes 32q .. 32q + 31
    const int nc = args.ncols;
    int it = 0;
    for (int t = blockIdx.x; t < m_tiles; t += gridDim.x, ++it) {
      const bool okd = mbar_wait(done, it & 1);
      tc_fence_after();
      if (!okd) { *abort_flag = 1; break; }
      const int grow = t * 128 + q * 32 + lane;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        if (c * 32 < nc) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + c * 32, v);
          tmem_ld_wait();
          if (grow < args.Mp && args.mode == 0) {
            uint16_t* o = static_cast<uint16_t*>(args.out) + static_cast<int64_t>(grow) * args.ld;
            uint16_t* o2 = args.out2 != nullptr ? args.out2 + static_cast<int64_t>(grow) * args.ld2 : nullptr;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int cc = c * 32 + i;
              if (cc < nc) {
                // (0 + v) * scale: the split kernel's sum and rounding for one split
                const uint16_t b = static_cast<uint16_t>(
                    pack_bf16x2((0.0f + __uint_as_float(v[i])) * args.scale, 0.0f) & 0xFFFFu);
                if (cc < args.nout) o[cc] = b;
                if (o2 != nullptr) o2[cc] = b;
              }
            }
          } else if (grow < args.Mp) {
            // fp32: mode 1 out[Mp][ld], mode 2 out[nout][Mp] (consecutive lanes, consecutive rows)
            float* o = static_cast<float*>(args.out);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int cc = c * 32 + i;
              if (cc < args.nout) {
                const float x = (0.0f + __uint_as_float(v[i])) * args.scale;
                if (args.mode == 1)
                  o[static_cast<int64_t>(grow) * args.ld + cc] = x;
                else
                  o[static_cast<int64_t>(cc) * args.Mp + grow] = x;
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) raise_status(args.d_status, QLORA_ERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

// ===========================================================================
// Fused NF4-decode GEMM (forward: kBwd = false, input gradient: kBwd = true)
//
// Persistent pairs of CTAs on neighbouring SMs (a 1 x 2 thread-block cluster)
// run CTA-pair tensor-core products (tcgen05.mma.cta_group::2, M = 256,
// N = 256, K = 16), issued by CTA rank 0 for both: the A operand is split by
// rows (128 per CTA) and the B operand by columns (128 per CTA), each half in
// its own CTA's shared memory, and each CTA's TMEM receives its 128 rows of D
// over all 256 columns.  So each CTA stages only half of each operand, and
// the tensor core reads 8 KB of shared memory per CTA and 16-wide K slice
// for a 128 x 256 x 16 product per SM.
//   forward   pair tile 512 rows x 256 columns; CTA q holds rows
//             m0 + 256q + [0, 256) (slices h = 0, 1 of 128 rows, the K-major
//             A operand of accumulator h) and decodes columns n0 + 128q + [0,
//             128) of every weight K-step (the MN-major B operand);
//   backward  transposed: pair tile 256 output columns x 512 dY rows; CTA q
//             decodes the weight rows n0 + 128q + [0, 128) (the K-major A
//             operand: its output columns) and holds dY rows m0 + 256h + 128q +
//             [0, 128) (its half of the B operand of accumulator h = 0, 1).
// TMEM: two accumulators of 128 lanes x 256 fp32 columns per CTA (all 512).
//
// Shared memory holds two rings per CTA.  Activation tiles (256 x 64 bf16,
// K-major, two TMA boxes of 128 rows) have 4 stages; TMA loads of both CTAs
// complete on CTA 0's barrier (the cta_group::2 form of the copy), which CTA
// 0's producer arms with both CTAs' bytes.  Decoded weight tiles have 4
// stages; decoder warps write them as 128 rows of 128 bytes, each row one NF4
// block of 64 consecutive weights (row R at R*128, 16-byte chunk c at
// (c ^ (R & 7))*16, the 128-byte swizzle pattern):
//   forward   row R = 64*nb + k: weights (k0+k, n0+128q+64nb .. +63) — an
//             MN-major operand (atoms of 8 k-rows x 64 n; 8 KB between
//             n-atoms);
//   backward  row R: weights (n0+128q+R, k0 .. k0+63) of W, i.e. row R of
//             Ŵᵀ's K-major operand.
// Each decoder thread owns one row and loads its 32 packed bytes and its
// block scale straight from global memory K-steps ahead; both CTAs' decoder
// warps arrive on CTA 0's barrier of the stage.  The MMA's commit releases
// the stages and signals the accumulators in both CTAs (multicast), and both
// CTAs' epilogue warps release an accumulator on CTA 0's barrier.
//
// After the last K-step of a tile, the LoRA step takes two activation stages:
// Zc (or dZ) as the activation tile and B (or A) as the weight tile, both by
// TMA with the rank padded to a multiple of 16 by TMA's zero fill; the decoder
// warps skip it.  The epilogue releases each accumulator as soon as it has
// read it, so the next tile's first MMAs overlap the drain of the last.  In
// the backward a warp's TMEM load gives each lane one output column over 32
// consecutive rows, so every store instruction writes 32 adjacent bf16 of one
// output row.
// ===========================================================================
constexpr int kFAStages = 4;          // activation tiles (TMA)
constexpr int kFBStages = 4;          // decoded weight tiles (decoder warps)
constexpr int kFBN = 128;             // decoded rows per CTA and K-step
constexpr int kFSlices = 2;           // 128-row activation slices per CTA = accumulators
constexpr int kFAccCols = 256;        // TMEM columns per accumulator (the pair MMA's N)
constexpr int kFPairRows = 512;       // activation rows of a pair tile
constexpr int kFPairCols = 256;       // output columns of a pair tile
constexpr int kFA = kFSlices * 128 * 128;   // 256 x 64 bf16
constexpr int kFB = kFBN * 128;             // 128 x 64 bf16
constexpr int kFDecWarps = kFBN / 32;       // one weight-tile row per decoder thread and K-step
// Decoder groups of kFDecWarps warps take turns by K-step (group g decodes the
// steps g, g + kFDecGroups, ...), so each warp has kFDecGroups K-steps of time
// per row and its loads reach further ahead.
constexpr int kFDecGroups = 2;
constexpr int kFDecAll = kFDecWarps * kFDecGroups;
constexpr int kFEpiWarps = 4;
constexpr int kFThreads = (2 + kFDecAll + kFEpiWarps) * 32;  // TMA, MMA, decoders, epilogue
constexpr size_t kFSmem = 1024 + kFAStages * kFA + kFBStages * kFB + 1024 + 512;
static_assert(kFSlices * kFAccCols == 512 && kFBN == 128, "accumulators fill TMEM");
static_assert(kFSmem <= 232448, "fused kernel shared memory");

struct FusedArgs {
  int M;          // rows of the activation / output
  int Nout;       // output columns (forward: N, backward: K)
  int Nw;         // row length of the weight (N); blocks per weight row = Nw/64
  int nk;         // K-steps over the contraction (forward: K/64, backward: N/64)
  int rsteps;     // MMAs of K=16 in the LoRA step (ceil(r/16))
  int m_tiles, n_tiles;
  ScaleView sv;
  const uint8_t* packed;
  uint16_t* out;  // bf16 [M][Nout]
  int32_t* d_status;
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// 8 packed nibbles (4 bytes, first weight in the high nibble of byte 0) ->
// 8 bf16 from the per-block table whose high and low bytes are split into
// H[0..3] and L[0..3] (entry j's byte in byte j%4 of H[j/4] / L[j/4]).
__device__ __forceinline__ uint4 decode8(uint32_t p, const uint32_t (&H)[4],
                                         const uint32_t (&L)[4]) {
  // selector nibbles: low 3 bits pick a byte within a plane pair, bit 3
  // (moved to the "+4" position) picks the pair
  const uint32_t s = p & 0x77777777u;
  const uint32_t b = ((p >> 1) & 0x44444444u) | 0x32103210u;
  uint4 o;
  {
    const uint32_t hF = prmt(prmt(H[0], H[1], s), prmt(H[2], H[3], s), b);
    const uint32_t lF = prmt(prmt(L[0], L[1], s), prmt(L[2], L[3], s), b);
    o.x = prmt(lF, hF, 0x4051u);
    o.y = prmt(lF, hF, 0x6273u);
  }
  {
    const uint32_t s2 = s >> 16, b2 = b >> 16;
    const uint32_t hF = prmt(prmt(H[0], H[1], s2), prmt(H[2], H[3], s2), b2);
    const uint32_t lF = prmt(prmt(L[0], L[1], s2), prmt(L[2], L[3], s2), b2);
    o.z = prmt(lF, hF, 0x4051u);
    o.w = prmt(lF, hF, 0x6273u);
  }
  return o;
}

// Per-block table: entry j = bf16(C_j * a) (fp32 product, then bf16).
__device__ __forceinline__ void build_lut(const float* C, float a, uint32_t (&H)[4], uint32_t (&L)[4]) {
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(C[2 * i] * a, C[2 * i + 1] * a);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    H[q] = prmt(w[2 * q], w[2 * q + 1], 0x7531u);
    L[q] = prmt(w[2 * q], w[2 * q + 1], 0x6420u);
  }
}

// What one decoder thread needs for one K-step, loaded ahead of use.
struct RowFetch {
  uint4 p0, p1;   // 32 packed bytes of the row's NF4 block
  float absv;     // absmax (no double quant)
  uint32_t q;     // scale code (double quant)
  float s2v;      // second-level scale (double quant)
  bool valid;     // row inside the weight; false also for LoRA steps
};

// Row Rg (0 .. kFPairCols-1) of the pair's decoded tile at K-step kk.
template <bool kBwd>
__device__ __forceinline__ RowFetch fetch_row(const FusedArgs& a, int tile, int kk, int Rg,
                                              int num_tiles) {
  RowFetch f;
  f.p0 = make_uint4(0, 0, 0, 0);
  f.p1 = f.p0;
  f.absv = 1.0f;
  f.q = 0;
  f.s2v = 1.0f;
  f.valid = false;
  if (tile >= num_tiles || kk >= a.nk) return f;
  const int n0 = (tile / a.m_tiles) * kFPairCols;
  const int64_t rowbytes = a.Nw / 2;
  const int64_t bpr = a.Nw / 64;
  int64_t blk;
  const uint8_t* src;
  if (!kBwd) {
    const int nb = Rg >> 6, kr = Rg & 63;
    if (n0 + nb * 64 >= a.Nout) return f;
    const int64_t k = static_cast<int64_t>(kk) * 64 + kr;
    src = a.packed + k * rowbytes + n0 / 2 + nb * 32;
    blk = k * bpr + n0 / 64 + nb;
  } else {
    if (n0 + Rg >= a.Nout) return f;
    const int64_t kw = n0 + Rg;
    src = a.packed + kw * rowbytes + kk * 32;
    blk = kw * bpr + kk;
  }
  f.valid = true;
  // volatile asm: the loads issue here, K-steps before their use, instead of
  // being moved down to it
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(f.p0.x), "=r"(f.p0.y), "=r"(f.p0.z), "=r"(f.p0.w) : "l"(src));
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(f.p1.x), "=r"(f.p1.y), "=r"(f.p1.z), "=r"(f.p1.w) : "l"(src + 16));
  if (a.sv.code8 == nullptr) {
    asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(f.absv) : "l"(a.sv.absmax + blk));
  } else {
    uint16_t qv;
    asm volatile("ld.global.nc.u8 %0, [%1];" : "=h"(qv) : "l"(a.sv.code8 + blk));
    f.q = qv;
    asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(f.s2v) : "l"(a.sv.s2 + (blk >> 8)));
  }
  return f;
}

// Advance an iteration cursor (tile, kk) by `n` steps of nsteps per tile;
// consecutive tiles of one pair are `stride` apart.
__device__ __forceinline__ void advance(int& tile, int& kk, int n, int nsteps, int stride) {
  kk += n;
  while (kk >= nsteps) {
    kk -= nsteps;
    tile += stride;
  }
}

template <bool kBwd>
__global__ void __launch_bounds__(kFThreads, 1)
    fused_nf4_gemm_kernel(const __grid_constant__ CUtensorMap tmAct,
                          const __grid_constant__ CUtensorMap tmLA,
                          const __grid_constant__ CUtensorMap tmLB, FusedArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kFAStages * kFA;
  float* t8 = reinterpret_cast<float*>(sB + kFBStages * kFB);
  uint64_t* full_a = reinterpret_cast<uint64_t*>(t8 + 256);
  uint64_t* empty_a = full_a + kFAStages;
  uint64_t* full_b = empty_a + kFAStages;
  uint64_t* empty_b = full_b + kFBStages;
  uint64_t* tfull = empty_b + kFBStages;
  uint64_t* tempty = tfull + 1;   // [kFSlices]: one per accumulator
  uint64_t* drain = tempty + kFSlices;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the pair is the cluster (2 x 1 x 1): rank 0 issues the MMAs
  const int rank = static_cast<int>(blockIdx.x & 1);
  const int pair = static_cast<int>(blockIdx.x >> 1), npairs = static_cast<int>(gridDim.x >> 1);
  if (args.sv.code8 != nullptr) build_t8(t8);
  if (threadIdx.x == 0) {
    // Only CTA 0's full_a, full_b and tempty are waited on; every CTA's
    // empty_a, empty_b and tfull receive the pair MMA's multicast commits.
    for (int s = 0; s < kFAStages; ++s) {
      mbar_init(&full_a[s], 1);            // CTA 0's producer, plus both CTAs' bytes
      mbar_init(&empty_a[s], 1);
    }
    for (int s = 0; s < kFBStages; ++s) {
      mbar_init(&full_b[s], 2 * kFDecWarps);   // both CTAs' decoder warps
      mbar_init(&empty_b[s], 1);
    }
    mbar_init(tfull, 1);
    for (int h = 0; h < kFSlices; ++h) mbar_init(&tempty[h], 2 * kFEpiWarps);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  // the peer's barriers are initialised before any arrival reaches them
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int num_tiles = args.m_tiles * args.n_tiles;
  pdl_launch_dependents();   // after this CTA holds its TMEM
  // No wait for the preceding kernel here.  It is always this library's
  // rank-r product (Zc, or dZ), which lets this kernel launch only after all
  // kernels before it have completed: the activations, the weights and the
  // output buffer are final or free, and only the LoRA step's Zc (dZ) comes
  // from the preceding kernel; the producer waits before loading it.

  if (warp == 0) {
    // ------------------------------ TMA producer ---------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tmAct);
      tma_prefetch_desc(&tmLA);
      tma_prefetch_desc(&tmLB);
      uint32_t ia = 0;                          // activation-ring slot counter
      uint32_t last_parity[kFAStages];
#pragma unroll
      for (int s = 0; s < kFAStages; ++s) last_parity[s] = 2;
      bool ok = true;
      // take the next slot; CTA 0 arms its full barrier with both CTAs' bytes
      auto take = [&](uint32_t& s_out, uint32_t bytes) -> bool {
        const uint32_t s = ia % kFAStages, ph = (ia / kFAStages) & 1;
        if (*abort_flag || !mbar_wait(&empty_a[s], ph ^ 1)) return false;
        if (rank == 0) mbar_arrive_expect_tx(&full_a[s], 2 * bytes);
        last_parity[s] = ph;
        s_out = s;
        ++ia;
        return true;
      };
      auto bar0 = [&](uint32_t s) -> uint32_t { return mapa_shared(smem_u32(&full_a[s]), 0); };
      // the activation rows of slice h of this CTA
      auto act_row = [&](int m0, int h) -> int {
        return kBwd ? m0 + 256 * h + 128 * rank : m0 + 256 * rank + 128 * h;
      };
      bool lora_ready = false;
      for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
        const int m0 = (tile % args.m_tiles) * kFPairRows;
        const int n0 = (tile / args.m_tiles) * kFPairCols;
        for (int kk = 0; kk < args.nk && ok; ++kk) {
          uint32_t s;
          if (!take(s, kFA)) { ok = false; break; }
          uint8_t* a = sA + s * kFA;
#pragma unroll
          for (int h = 0; h < kFSlices; ++h)
            tma_load_2d_pair(a + h * 16384, &tmAct, bar0(s), kk * 64, act_row(m0, h));
        }
        if (!ok) break;
        // LoRA step: Zc / dZ into one stage, B / A into the next
        if (!lora_ready) {
          pdl_wait();   // Zc (dZ) is the preceding kernel's output
          lora_ready = true;
        }
        uint32_t s1, s2;
        if (!take(s1, kFA)) { ok = false; break; }
        uint8_t* a = sA + s1 * kFA;
#pragma unroll
        for (int h = 0; h < kFSlices; ++h)
          tma_load_2d_pair(a + h * 16384, &tmLA, bar0(s1), 0, act_row(m0, h));
        if (!take(s2, kFB)) { ok = false; break; }
        uint8_t* b = sA + s2 * kFA;
        if (!kBwd) {
          // B's columns of this CTA's half, two 64-column boxes (MN-major)
#pragma unroll
          for (int nb = 0; nb < kFBN / 64; ++nb)
            tma_load_2d_pair(b + nb * 8192, &tmLB, bar0(s2), n0 + 128 * rank + nb * 64, 0);
        } else {
          // A's rows of this CTA's output columns (K-major)
          tma_load_2d_pair(b, &tmLB, bar0(s2), 0, n0 + 128 * rank);
        }
      }
      if (!ok) *abort_flag = 1;
      // CTA 0: let copies already in flight (its own and the peer's) land
      // before either CTA can exit
      if (rank == 0)
        for (int s = 0; s < kFAStages; ++s)
          if (last_parity[s] < 2) (void)mbar_wait(&full_a[s], last_parity[s]);
    }
  } else if (warp == 1) {
    // ------------------------- MMA issuer (CTA 0 only) ----------------------
    if (lane == 0 && rank == 0) {
      // forward: D[m][n] += act[m][k] * Ŵtile[k][n] (tile MN-major, as B);
      // backward: D[n][m] += Ŵtile[n][k] * dY[m][k] (tile K-major, as A)
      constexpr uint32_t idesc = kBwd ? idesc_bf16_f32(256, kFAccCols, 0, 0)
                                      : idesc_bf16_f32(256, kFAccCols, 0, 1);
      uint32_t ia = 0, ib = 0, tc = 0;
      bool ok = true;
      auto wait_a = [&](uint32_t& s) -> bool {
        s = ia % kFAStages;
        const uint32_t ph = (ia / kFAStages) & 1;
        ++ia;
        return !*abort_flag && mbar_wait(&full_a[s], ph);
      };
      // one 16-wide K slice j of accumulator h: `w0` the weight operand
      // (decoded tile, or B / A in the LoRA step), `a0` the activation stage
      auto mma = [&](int h, uint32_t a0, uint32_t w0, int j, uint32_t accum) {
        const uint64_t adesc = smem_desc(a0 + h * 16384 + j * 32, 16, 1024);
        if (kBwd)
          umma_bf16_pair(tmem + h * kFAccCols, smem_desc(w0 + j * 32, 16, 1024), adesc, idesc, accum);
        else
          umma_bf16_pair(tmem + h * kFAccCols, adesc, smem_desc(w0 + j * 2048, 8192, 1024), idesc,
                         accum);
      };
      for (int tile = pair; tile < num_tiles && ok; tile += npairs, ++tc) {
        const uint32_t tph = (tc & 1) ^ 1;       // parity of the previous tile's release
        for (int kk = 0; kk < args.nk; ++kk) {
          uint32_t sa;
          if (!wait_a(sa)) { ok = false; break; }
          const uint32_t sb = ib % kFBStages, phb = (ib / kFBStages) & 1;
          ++ib;
          if (*abort_flag || !mbar_wait(&full_b[sb], phb)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + sa * kFA), b0 = smem_u32(sB + sb * kFB);
          const uint32_t acc = kk > 0 ? 1u : 0u;
#pragma unroll
          for (int h = 0; h < kFSlices; ++h) {
            if (kk == 0) {   // first K-step of a tile: wait until this accumulator is drained
              if (*abort_flag || !mbar_wait(&tempty[h], tph)) { ok = false; break; }
              tc_fence_after();
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) mma(h, a0, b0, j, (acc || j > 0) ? 1u : 0u);
          }
          if (!ok) break;
          umma_commit_pair_mc(&empty_a[sa], 0x3);
          umma_commit_pair_mc(&empty_b[sb], 0x3);
        }
        if (!ok) break;
        // LoRA step
        uint32_t s1, s2;
        if (!wait_a(s1) || !wait_a(s2)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + s1 * kFA), w0 = smem_u32(sA + s2 * kFA);
        for (int j = 0; j < args.rsteps; ++j)
#pragma unroll
          for (int h = 0; h < kFSlices; ++h) mma(h, a0, w0, j, 1u);
        umma_commit_pair_mc(&empty_a[s1], 0x3);
        umma_commit_pair_mc(&empty_a[s2], 0x3);
        umma_commit_pair_mc(tfull, 0x3);
      }
      if (!ok) *abort_flag = 1;
      umma_commit_pair_mc(drain, 0x1);
      (void)mbar_wait(drain, 0);
    }
  } else if (warp < 2 + kFDecAll) {
    // ------------------------------ decoders -------------------------------
    const int grp = (warp - 2) / kFDecWarps;   // this warp's turn among the groups
    const int R = threadIdx.x - 64 - grp * kFBN;   // row of this CTA's decoded tile
    const int Rg = kFBN * rank + R;                // row of the pair's decoded tile
    const float off = args.sv.code8 != nullptr ? __ldg(args.sv.offset) : 0.0f;
    const int nsteps = args.nk;                // decoded steps per tile
    bool ok = true;
    int tile = pair, kk = 0;                   // the step being decoded
    advance(tile, kk, grp, nsteps, npairs);
    int ptile = tile, pkk = kk;                // the step being prefetched
    uint32_t ib = static_cast<uint32_t>(grp);
    // One K-step: wait for a free weight stage, decode this thread's row.
    auto step = [&](const RowFetch& f) {
      const uint32_t s = ib % kFBStages, ph = (ib / kFBStages) & 1;
      if (*abort_flag || !mbar_wait(&empty_b[s], ph ^ 1)) {
        ok = false;
        return;
      }
      uint8_t* brow = sB + s * kFB + R * 128;
      const uint32_t sw = static_cast<uint32_t>(R & 7);
      if (f.valid) {
        const float a = args.sv.code8 == nullptr
                            ? f.absv
                            : __fadd_rn(__fmul_rn(t8[f.q], f.s2v), off);
        uint32_t H[4], L[4];
        build_lut(kNF4g + 16 * args.sv.codebook, a, H, L);
        const uint32_t pw[8] = {f.p0.x, f.p0.y, f.p0.z, f.p0.w, f.p1.x, f.p1.y, f.p1.z, f.p1.w};
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(brow + ((static_cast<uint32_t>(c) ^ sw) << 4)) =
              decode8(pw[c], H, L);
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(brow + ((static_cast<uint32_t>(c) ^ sw) << 4)) =
              make_uint4(0, 0, 0, 0);
      }
      // the rows are visible to the tensor core (async proxy), then CTA 0's
      // barrier of the stage counts this warp
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&full_b[s]), 0));
      advance(tile, kk, kFDecGroups, nsteps, npairs);
      ib += kFDecGroups;
    };
    // Three prefetch slots consumed and refilled in place (no register moves
    // that would wait on loads still in flight).
    RowFetch q0 = fetch_row<kBwd>(args, ptile, pkk, Rg, num_tiles);
    advance(ptile, pkk, kFDecGroups, nsteps, npairs);
    RowFetch q1 = fetch_row<kBwd>(args, ptile, pkk, Rg, num_tiles);
    advance(ptile, pkk, kFDecGroups, nsteps, npairs);
    RowFetch q2 = fetch_row<kBwd>(args, ptile, pkk, Rg, num_tiles);
    advance(ptile, pkk, kFDecGroups, nsteps, npairs);
    while (ok && tile < num_tiles) {
      step(q0);
      q0 = fetch_row<kBwd>(args, ptile, pkk, Rg, num_tiles);
      advance(ptile, pkk, kFDecGroups, nsteps, npairs);
      if (!ok || tile >= num_tiles) break;
      step(q1);
      q1 = fetch_row<kBwd>(args, ptile, pkk, Rg, num_tiles);
      advance(ptile, pkk, kFDecGroups, nsteps, npairs);
      if (!ok || tile >= num_tiles) break;
      step(q2);
      q2 = fetch_row<kBwd>(args, ptile, pkk, Rg, num_tiles);
      advance(ptile, pkk, kFDecGroups, nsteps, npairs);
    }
    if (!ok) *abort_flag = 1;
  } else {
    // ------------------------------ epilogue -------------------------------
    const int q = warp & 3;
    uint32_t tc = 0;
    bool ok = true;
    const uint32_t tempty0 = mapa_shared(smem_u32(tempty), 0);   // CTA 0's release barriers
    for (int tile = pair; tile < num_tiles && ok; tile += npairs, ++tc) {
      const int m0 = (tile % args.m_tiles) * kFPairRows;
      const int n0 = (tile / args.m_tiles) * kFPairCols;
      if (*abort_flag || !mbar_wait(tfull, tc & 1)) { ok = false; break; }
      tc_fence_after();
      const int64_t ld = args.Nout;
#pragma unroll 1
      for (int h = 0; h < kFSlices; ++h) {
        const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + h * kFAccCols;
#pragma unroll 1
        for (int c = 0; c < kFAccCols / 32; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tbase + c * 32, v);
          tmem_ld_wait();
          if (!kBwd) {
            // lane = output row, 32 consecutive output columns
            const int row = m0 + 256 * rank + h * 128 + q * 32 + lane;
            const int col = n0 + c * 32;
            if (row < args.M && col < args.Nout) {
              uint4* dst = reinterpret_cast<uint4*>(args.out + row * ld + col);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_uint4(
                    pack_bf16x2(__uint_as_float(v[8 * i + 0]), __uint_as_float(v[8 * i + 1])),
                    pack_bf16x2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3])),
                    pack_bf16x2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5])),
                    pack_bf16x2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7])));
            }
          } else {
            // lane = output column, 32 consecutive output rows
            const int col = n0 + 128 * rank + q * 32 + lane;
            const int row0 = m0 + h * kFAccCols + c * 32;
            if (col < args.Nout && row0 < args.M) {
              uint16_t* dst = args.out + row0 * ld + col;
              const int nrows = args.M - row0;   // rows left in the output (>= 1)
#pragma unroll
              for (int i = 0; i < 32; i += 2) {
                const uint32_t pr = pack_bf16x2(__uint_as_float(v[i]), __uint_as_float(v[i + 1]));
                if (i < nrows) dst[i * ld] = static_cast<uint16_t>(pr);
                if (i + 1 < nrows) dst[(i + 1) * ld] = static_cast<uint16_t>(pr >> 16);
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty0 + static_cast<uint32_t>(h) * 8u);
      }
    }
    if (!ok) *abort_flag = 1;
  }

  tc_fence_before();
  __syncthreads();
  // neither CTA leaves while the pair MMA, the peer's copies or the peer's
  // arrivals may still reach it
  cluster_sync_all();
  if (*abort_flag && threadIdx.x == 0) raise_status(args.d_status, QLORA_ERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// Zero-padded copy of a rows x r bf16 matrix into rows x rp (rp = r rounded
// up to a multiple of 8), so that every row starts on a 16-byte boundary as
// the tensor maps need.  Only used when r is not a multiple of 8.
__global__ void __launch_bounds__(256) pad_cols_kernel(const uint16_t* __restrict__ src,
                                                       int64_t rows, int r,
                                                       uint16_t* __restrict__ dst, int rp) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t total = rows * rp;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / rp;
    const int col = static_cast<int>(i - row * rp);
    dst[i] = col < r ? src[row * r + col] : static_cast<uint16_t>(0);
  }
}

// ===========================================================================
// Host side
// ===========================================================================
namespace {

// K splits of a rank-r contraction: one CTA per SM (the kernel's shared
// memory allows no second), so the grid is kept to a single wave.
// The SM count that fixes split counts and the rank-r path, whatever the
// device: results (the fp32 summation order of the rank-r products) depend on
// the shape only.
constexpr int g_ws_sms = 148;

int skinny_splits(int Mp, int nk, int num_sms) {
  const int mt = (Mp + 127) / 128;
  int want = num_sms / mt;
  if (want > kSkMaxSplits) want = kSkMaxSplits;
  if (want < 1) want = 1;
  if (want > nk) want = nk;
  const int per = (nk + want - 1) / want;
  return (nk + per - 1) / per;
}

struct WsCursor {
  char* p;
  size_t left;
  bool ok = true;
  void* take(size_t bytes) {
    bytes = (bytes + 255) & ~static_cast<size_t>(255);
    if (bytes > left) { ok = false; return nullptr; }
    void* r = p;
    p += bytes;
    left -= bytes;
    return r;
  }
};

size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

template <bool A, bool B>
cudaError_t set_skinny_attr() {
  static DeviceOnce once;
  return once.run([](int) {
    return cudaFuncSetAttribute(skinny_gemm_kernel<A, B>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(kSkSmem));
  });
}

// D = scale * A(m',k') B(n',k'): one launch, split-K sums added in-kernel.
// ncols columns of D are summed; the first nout go to `out`, and in mode 0 all
// ncols also go to out2 (a padded copy) when it is not null.
template <bool kAmn, bool kBmn>
cudaError_t run_skinny(const CUtensorMap& ta, const CUtensorMap& tb, int Mp, int Kp, int ncols,
                       float scale, int mode, void* out, int ld, int splits, int32_t* d_status,
                       cudaStream_t st, int nout = -1, uint16_t* out2 = nullptr, int ld2 = 0) {
  cudaError_t e = set_skinny_attr<kAmn, kBmn>();
  if (e != cudaSuccess) return e;
  const int nk = (Kp + 64 * kSkW - 1) / (64 * kSkW);
  SkinnyArgs a;
  a.Mp = Mp;
  a.nk = nk;
  a.kb_per_split = (nk + splits - 1) / splits;
  a.splits = (nk + a.kb_per_split - 1) / a.kb_per_split;
  a.ncols = ncols;
  a.nout = nout < 0 ? ncols : nout;
  a.scale = scale;
  a.mode = mode;
  a.out = out;
  a.ld = ld;
  a.out2 = out2;
  a.ld2 = ld2;
  a.d_status = d_status;
  {
    ProfScope prof(kProfSkinny, st);
    e = launch_pdl(skinny_gemm_kernel<kAmn, kBmn>, dim3((Mp + 127) / 128, a.splits, 1),
                   dim3(kSkThreads, 1, 1), kSkSmem, st, a.splits, ta, tb, a);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <bool A, bool B>
cudaError_t set_rank_rows_attr() {
  static DeviceOnce once;
  return once.run([](int) {
    return cudaFuncSetAttribute(rank_rows_kernel<A, B>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(kSkSmem));
  });
}

// Pairs of the fused GEMM: the fewest that keep its number of waves of tiles
// (so the SMs it leaves free cost it nothing).
int fused_pairs(int tiles, int sms) {
  const int most = sms / 2 > 0 ? sms / 2 : 1;
  const int waves = (tiles + most - 1) / most;
  const int pairs = waves > 0 ? (tiles + waves - 1) / waves : 1;
  return pairs < 1 ? 1 : pairs;
}

// CTAs for rank-r products streaming `bytes` beside the fused GEMM of `tiles`
// pair tiles, or 0 for the split kernel.  Decided for the sizing SM count
// (not the device's), so the forward and the backward's recompute make the
// same choice and form Zc alike: the SMs the fused GEMM leaves free (an even
// number), when there are at least 8 of them and each streams at most
// mb_per_sm MB (done long before the fused GEMM needs the product).
int rank_rows_ctas(double bytes, int tiles, double mb_per_sm) {
  const int free_sms = g_ws_sms - 2 * fused_pairs(tiles, g_ws_sms);
  if (free_sms < 8) return 0;
  if (bytes > mb_per_sm * 1e6 * free_sms) return 0;
  return free_sms;
}

// D = scale * A(m',k') B(n',k') by rank_rows_kernel on `ctas` CTAs; modes as
// for run_skinny (0: bf16 out, and all ncols columns again into out2 when it
// is not null; 1: fp32 out[Mp][ld]; 2: fp32 out[nout][Mp]).
template <bool kAmn, bool kBmn>
cudaError_t run_rank_rows(const CUtensorMap& ta, const CUtensorMap& tb, int Mp, int Kp, int ncols,
                          float scale, int mode, void* out, int ld, int ctas, int32_t* d_status,
                          cudaStream_t st, int nout = -1, uint16_t* out2 = nullptr, int ld2 = 0) {
  cudaError_t e = set_rank_rows_attr<kAmn, kBmn>();
  if (e != cudaSuccess) return e;
  // at most one CTA per tile, in pairs (a 2 x 1 cluster, so that the SMs left
  // to the fused GEMM's pairs stay in pairs)
  const int m_tiles = (Mp + 127) / 128;
  if (ctas > m_tiles) ctas = m_tiles;
  ctas = (ctas + 1) & ~1;
  SkinnyArgs a;
  a.Mp = Mp;
  a.nk = (Kp + 64 * kSkW - 1) / (64 * kSkW);
  a.kb_per_split = a.nk;
  a.splits = 1;
  a.ncols = ncols;
  a.nout = nout < 0 ? ncols : nout;
  a.scale = scale;
  a.mode = mode;
  a.out = out;
  a.ld = ld;
  a.out2 = out2;
  a.ld2 = ld2;
  a.d_status = d_status;
  {
    ProfScope prof(kProfSkinny, st);
    e = launch_pdl_pair(rank_rows_kernel<kAmn, kBmn>, dim3(static_cast<unsigned>(ctas)),
                        dim3(kSkThreads, 1, 1), kSkSmem, st, ta, tb, a);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <bool kBwd>
cudaError_t set_fused_attr() {
  static DeviceOnce once;
  return once.run([](int) {
    return cudaFuncSetAttribute(fused_nf4_gemm_kernel<kBwd>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(kFSmem));
  });
}

constexpr CUtensorMapDataType kBF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
constexpr CUtensorMapSwizzle kSW128 = CU_TENSOR_MAP_SWIZZLE_128B;

int rsteps_of(int r) { return (r + 15) / 16; }

// Rank rounded up to a multiple of 8: the row pitch (rp * 2 bytes) of every
// rank-r operand read by TMA must be a multiple of 16 bytes.
int padded_rank(int r) { return (r + 7) & ~7; }

cudaError_t launch_pad(const uint16_t* src, int64_t rows, int r, uint16_t* dst, int rp,
                       cudaStream_t st) {
  const int64_t want = (rows * rp + 255) / 256;
  const unsigned grid = static_cast<unsigned>(want < 592 ? want : 592);
  cudaError_t e;
  {
    ProfScope prof(kProfOther, st);
    e = launch_pdl(pad_cols_kernel, dim3(grid), dim3(256), 0, st, 1, src, rows, r, dst, rp);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace


// A library-owned stream per device for work that runs beside the caller's
// stream, and the two events of one fork and join.  Created on first use
// (retried after a failure, e.g. inside a stream capture that forbids it);
// g_side_mu is held from a fork to its join, so concurrent callers never
// interleave their records and waits on the shared events.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
static std::mutex g_side_mu;
static SideStream g_side[64];

static SideStream* side_stream(int dev) {
  if (dev < 0 || dev >= 64) return nullptr;
  SideStream& ss = g_side[dev];
  if (ss.s == nullptr) {
    int least = 0, greatest = 0;
    cudaDeviceGetStreamPriorityRange(&least, &greatest);
    cudaStream_t s = nullptr;
    cudaEvent_t f = nullptr, j = nullptr;
    if (cudaStreamCreateWithPriority(&s, cudaStreamNonBlocking, least) != cudaSuccess ||
        cudaEventCreateWithFlags(&f, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&j, cudaEventDisableTiming) != cudaSuccess) {
      if (s != nullptr) cudaStreamDestroy(s);
      if (f != nullptr) cudaEventDestroy(f);
      (void)cudaGetLastError();
      return nullptr;
    }
    ss.fork = f;
    ss.join = j;
    ss.s = s;
  }
  return &ss;
}

size_t linear_fwd_workspace_bytes(int64_t M, int64_t K, int64_t N, int r) {
  const int rp = padded_rank(r);
  // A zero-padded to rp columns when r is not a multiple of 8
  const size_t apad = rp != r ? align256(static_cast<size_t>(K) * rp * 2) : 0;
  if (M > 16) {
    // the rank-r kernel adds its splits in shared memory; a padded copy of Zc
    // for the fused kernel's TMA when r is not a multiple of 8
    return rp != r ? apad + align256(static_cast<size_t>(M) * rp * 2) : 0;
  }
  return apad;   // the GEMV adds its K splits inside a thread-block cluster
}

size_t linear_bwd_workspace_bytes(int64_t M, int64_t K, int64_t N, int r) {
  (void)N;
  const int rp = padded_rank(r);
  // dZ, and Zc when the caller recomputes it instead of saving it (or a padded
  // copy of the caller's Zc), both bf16 M x rp; A padded to rp columns
  return 2 * align256(static_cast<size_t>(M) * rp * 2) +
         (rp != r ? align256(static_cast<size_t>(K) * rp * 2) : 0);
}

cudaError_t launch_linear_fwd(int64_t M, int64_t K, int64_t N, int r, const uint16_t* X,
                              const uint8_t* packed, ScaleView sv, const uint16_t* A,
                              const uint16_t* B, float c, uint16_t* Y, uint16_t* Zc, void* ws,
                              size_t ws_bytes, int32_t* d_status, cudaStream_t st, int num_sms) {
  WsCursor cur{static_cast<char*>(ws), ws_bytes};
  const int rp = padded_rank(r);
  const bool pad = rp != r;
  cudaError_t e = cudaSuccess;
  // A zero-padded to rp columns (16-byte row pitch for TMA) when r % 8 != 0
  const uint16_t* At = A;
  if (pad) {
    uint16_t* Ap = static_cast<uint16_t*>(cur.take(static_cast<size_t>(K) * rp * 2));
    if (!cur.ok) return cudaErrorInvalidValue;
    e = launch_pad(A, K, r, Ap, rp, st);
    if (e != cudaSuccess) return e;
    At = Ap;
  }
  if (!cur.ok) return cudaErrorInvalidValue;
  // Zc = bf16(c * X A): A operand X (K-major), B operand A (MN-major over r)
  CUtensorMap tX, tAl, tZc, tBl;
  if (!make_tmap_2d(&tX, X, kBF16, 2, M, K, K, 64, 128, kSW128)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tAl, At, kBF16, 2, K, rp, rp, 64, 64, kSW128)) return cudaErrorInvalidValue;
  if (M <= 16) {
    // one launch: weights streamed once, X·A and its split sums in the same
    // cluster, Zc and Y written (the GEMV's own SM count fixes its splits)
    return launch_gemv(M, K, N, r, X, packed, sv, At, rp, B, c, Y, Zc, r, false, d_status, st,
                       num_sms);
  }

  // rank-r product for the tensor-core path: Zc = bf16(c * X A), and a copy
  // padded to rp columns for the fused kernel's TMA when r % 8 != 0
  uint16_t* Zp = nullptr;
  if (pad) {
    Zp = static_cast<uint16_t*>(cur.take(static_cast<size_t>(M) * rp * 2));
    if (!cur.ok) return cudaErrorInvalidValue;
  }
  {
    // beside the fused GEMM on the SMs it leaves free, or split-K before it
    const int fwd_tiles = static_cast<int>(((M + kFPairRows - 1) / kFPairRows) *
                                           ((N + kFPairCols - 1) / kFPairCols));
    const int rows_ctas = rank_rows_ctas(2.0 * M * K, fwd_tiles, 2.5);
    if (rows_ctas > 0) {
      e = run_rank_rows<false, true>(tX, tAl, static_cast<int>(M), static_cast<int>(K), rp, c, 0, Zc,
                                     r, rows_ctas, d_status, st, r, Zp, rp);
    } else {
      const int Sz = skinny_splits(static_cast<int>(M), static_cast<int>(K / 64), g_ws_sms);
      e = run_skinny<false, true>(tX, tAl, static_cast<int>(M), static_cast<int>(K), rp, c, 0, Zc, r,
                                  Sz, d_status, st, r, Zp, rp);
    }
    if (e != cudaSuccess) return e;
  }
  e = set_fused_attr<false>();
  if (e != cudaSuccess) return e;
  if (!make_tmap_2d(&tZc, pad ? Zp : Zc, kBF16, 2, M, rp, rp, 64, 128, kSW128)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tBl, B, kBF16, 2, r, N, N, 64, 64, kSW128)) return cudaErrorInvalidValue;
  FusedArgs fa;
  fa.M = static_cast<int>(M);
  fa.Nout = static_cast<int>(N);
  fa.Nw = static_cast<int>(N);
  fa.nk = static_cast<int>(K / 64);
  fa.rsteps = rsteps_of(r);
  fa.m_tiles = static_cast<int>((M + kFPairRows - 1) / kFPairRows);   // pair tiles of 512 rows
  fa.n_tiles = static_cast<int>((N + kFPairCols - 1) / kFPairCols);   // and 256 columns
  fa.sv = sv;
  fa.packed = packed;
  fa.out = Y;
  fa.d_status = d_status;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // persistent pairs of CTAs (a cluster of 2 x 1): the fewest pairs that
  // keep the number of waves of tiles
  const int grid = fused_pairs(fa.m_tiles * fa.n_tiles, sms);
  {
    ProfScope prof(kProfFusedFwd, st);
    e = launch_pdl_pair(fused_nf4_gemm_kernel<false>, dim3(2 * grid), dim3(kFThreads), kFSmem, st, tX,
                        tZc, tBl, fa);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_linear_bwd(int64_t M, int64_t K, int64_t N, int r, const uint16_t* dY,
                              const uint16_t* X, const uint16_t* Zc, const uint8_t* packed,
                              ScaleView sv, const uint16_t* A, const uint16_t* B, float c,
                              uint16_t* dX, float* dA, float* dB, void* ws, size_t ws_bytes,
                              int32_t* d_status, cudaStream_t st, int num_sms) {
  WsCursor cur{static_cast<char*>(ws), ws_bytes};
  const int rp = padded_rank(r);
  const bool pad = rp != r;
  // dZ and the working copy of Zc are bf16 M x rp (row pitch 16-byte aligned)
  uint16_t* dZ = static_cast<uint16_t*>(cur.take(static_cast<size_t>(M) * rp * 2));
  uint16_t* Zc_ws = static_cast<uint16_t*>(cur.take(static_cast<size_t>(M) * rp * 2));
  uint16_t* Ap = pad ? static_cast<uint16_t*>(cur.take(static_cast<size_t>(K) * rp * 2)) : nullptr;
  const int Sz = skinny_splits(static_cast<int>(M), static_cast<int>(N / 64), g_ws_sms);
  const int nkm = static_cast<int>((M + 63) / 64);
  const int Sa = skinny_splits(static_cast<int>(K), nkm, g_ws_sms);
  const int Sb = skinny_splits(static_cast<int>(N), nkm, g_ws_sms);
  if (!cur.ok) return cudaErrorInvalidValue;
  cudaError_t e = cudaSuccess;
  const uint16_t* At = A;
  if (pad) {
    e = launch_pad(A, K, r, Ap, rp, st);
    if (e != cudaSuccess) return e;
    At = Ap;
  }
  if (Zc == nullptr && M <= 16) {
    // saved-activation policy "recompute": Zc = bf16(c X A) exactly as the
    // forward forms it for M <= 16 (the GEMV kernel, its splits and sums)
    e = launch_gemv(M, K, N, r, X, packed, sv, At, rp, B, c, nullptr, Zc_ws, rp, true, d_status, st,
                    num_sms);
    if (e != cudaSuccess) return e;
    Zc = Zc_ws;
  } else if (Zc == nullptr) {
    // saved-activation policy "recompute": Zc = bf16(c X A) exactly as the
    // forward forms it (same kernel, same splits, so the same bits)
    CUtensorMap tXf, tAf;
    if (!make_tmap_2d(&tXf, X, kBF16, 2, M, K, K, 64, 128, kSW128)) return cudaErrorInvalidValue;
    if (!make_tmap_2d(&tAf, At, kBF16, 2, K, rp, rp, 64, 64, kSW128)) return cudaErrorInvalidValue;
    // the forward's choice of kernel and split, so the same bits
    const int fwd_tiles = static_cast<int>(((M + kFPairRows - 1) / kFPairRows) *
                                           ((N + kFPairCols - 1) / kFPairCols));
    const int rows_ctas = rank_rows_ctas(2.0 * M * K, fwd_tiles, 2.5);
    if (rows_ctas > 0) {
      e = run_rank_rows<false, true>(tXf, tAf, static_cast<int>(M), static_cast<int>(K), rp, c, 0,
                                     Zc_ws, rp, rows_ctas, d_status, st);
    } else {
      const int Sf = skinny_splits(static_cast<int>(M), static_cast<int>(K / 64), g_ws_sms);
      e = run_skinny<false, true>(tXf, tAf, static_cast<int>(M), static_cast<int>(K), rp, c, 0, Zc_ws,
                                  rp, Sf, d_status, st);
    }
    if (e != cudaSuccess) return e;
    Zc = Zc_ws;
  } else if (pad) {
    e = launch_pad(Zc, M, r, Zc_ws, rp, st);
    if (e != cudaSuccess) return e;
    Zc = Zc_ws;
  }

  CUtensorMap tG, tBk, tXmn, tdZ, tGmn, tZcmn, tAl;
  // dZ = c * G B^T : A operand G (K-major over N), B operand B (K-major: rows r, cols N);
  // B's rows past r arrive as zero fill, so dZ's padding columns are zero
  if (!make_tmap_2d(&tG, dY, kBF16, 2, M, N, N, 64, 128, kSW128)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tBk, B, kBF16, 2, r, N, N, 64, 64, kSW128)) return cudaErrorInvalidValue;
  {
    const int dx_tiles = static_cast<int>(((M + kFPairRows - 1) / kFPairRows) *
                                          ((K + kFPairCols - 1) / kFPairCols));
    const int rows_ctas = rank_rows_ctas(2.0 * M * N, dx_tiles, 2.5);
    if (rows_ctas > 0)
      e = run_rank_rows<false, false>(tG, tBk, static_cast<int>(M), static_cast<int>(N), rp, c, 0, dZ,
                                      rp, rows_ctas, d_status, st);
    else
      e = run_skinny<false, false>(tG, tBk, static_cast<int>(M), static_cast<int>(N), rp, c, 0, dZ, rp,
                                   Sz, d_status, st);
  }
  if (e != cudaSuccess) return e;
  // dA = X^T dZ : A operand X^T (MN-major over K), B operand dZ (MN-major over r)
  if (!make_tmap_2d(&tXmn, X, kBF16, 2, M, K, K, 64, 64, kSW128)) return cudaErrorInvalidValue;
  // (columns of dZ past rp arrive as TMA zero fill)
  if (!make_tmap_2d(&tdZ, dZ, kBF16, 2, M, rp, rp, 64, 64, kSW128)) return cudaErrorInvalidValue;
  // dB^T = G^T Zc : A operand G^T (MN-major over N), B operand Zc (MN-major over r)
  if (!make_tmap_2d(&tGmn, dY, kBF16, 2, M, N, N, 64, 64, kSW128)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tZcmn, Zc, kBF16, 2, M, rp, rp, 64, 64, kSW128)) return cudaErrorInvalidValue;
  // dX = G W^T + dZ A^T
  e = set_fused_attr<true>();
  if (e != cudaSuccess) return e;
  if (!make_tmap_2d(&tAl, At, kBF16, 2, K, rp, rp, 64, kFBN, kSW128)) return cudaErrorInvalidValue;
  CUtensorMap tdZa;
  if (!make_tmap_2d(&tdZa, dZ, kBF16, 2, M, rp, rp, 64, 128, kSW128)) return cudaErrorInvalidValue;
  FusedArgs fa;
  fa.M = static_cast<int>(M);
  fa.Nout = static_cast<int>(K);
  fa.Nw = static_cast<int>(N);
  fa.nk = static_cast<int>(N / 64);
  fa.rsteps = rsteps_of(r);
  fa.m_tiles = static_cast<int>((M + kFPairRows - 1) / kFPairRows);   // pair tiles of 512 dY rows
  fa.n_tiles = static_cast<int>((K + kFPairCols - 1) / kFPairCols);   // and 256 output columns
  fa.sv = sv;
  fa.packed = packed;
  fa.out = dX;
  fa.d_status = d_status;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // persistent pairs of CTAs (a cluster of 2 x 1): the fewest pairs that
  // keep the number of waves of tiles
  const int grid = fused_pairs(fa.m_tiles * fa.n_tiles, sms);

  // dX on the caller's stream first; dA and dB, which need only dZ, Zc, X and
  // G, on the side stream after dZ, so their CTAs take the SMs that dX's
  // partial last wave of tiles leaves idle.  The caller's stream then waits
  // for them: to the caller the call is ordered as one operation on st.
  std::lock_guard<std::mutex> lock(g_side_mu);
  SideStream* ss = prof_timing(kProfSkinny) ? nullptr : side_stream(dev);
  cudaStream_t s2 = st;
  if (ss != nullptr && cudaEventRecord(ss->fork, st) == cudaSuccess) s2 = ss->s;
  {
    ProfScope prof(kProfFusedBwd, st);
    e = launch_pdl_pair(fused_nf4_gemm_kernel<true>, dim3(2 * grid), dim3(kFThreads), kFSmem, st, tG,
                        tdZa, tAl, fa);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  if (s2 != st) {
    const cudaError_t ew = cudaStreamWaitEvent(s2, ss->fork, 0);
    if (ew != cudaSuccess) {
      // no fork: dA and dB after dX on the caller's stream
      s2 = st;
      if (e == cudaSuccess) e = ew;
    }
  }
  // dA, dB on the SMs dX leaves free when they can stream their 2 x M x
  // (K + N) bytes there well within dX, else split-K
  const int dx_tiles = fa.m_tiles * fa.n_tiles;
  const int dadb_ctas = rank_rows_ctas(2.0 * M * (K + N), dx_tiles, 5.0);
  if (e == cudaSuccess)
    e = dadb_ctas > 0
            ? run_rank_rows<true, true>(tXmn, tdZ, static_cast<int>(K), static_cast<int>(M), r, 1.0f, 1,
                                        dA, r, dadb_ctas, d_status, s2)
            : run_skinny<true, true>(tXmn, tdZ, static_cast<int>(K), static_cast<int>(M), r, 1.0f, 1, dA,
                                     r, Sa, d_status, s2);
  if (e == cudaSuccess)
    e = dadb_ctas > 0
            ? run_rank_rows<true, true>(tGmn, tZcmn, static_cast<int>(N), static_cast<int>(M), r, 1.0f,
                                        2, dB, r, dadb_ctas, d_status, s2)
            : run_skinny<true, true>(tGmn, tZcmn, static_cast<int>(N), static_cast<int>(M), r, 1.0f, 2,
                                     dB, r, Sb, d_status, s2);
  if (s2 != st) {
    // always join, so that nothing on st can run ahead of work already queued
    const cudaError_t ej = cudaEventRecord(ss->join, s2);
    const cudaError_t ew = ej == cudaSuccess ? cudaStreamWaitEvent(st, ss->join, 0) : ej;
    if (e == cudaSuccess) e = ew;
  }
  return e;
}

}  // namespace qnf4
