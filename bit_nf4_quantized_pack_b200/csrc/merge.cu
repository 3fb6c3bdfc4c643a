// Merged dense weight of the trained layer (export).  Page "QLoRA：冻结的 4-bit
// 权重怎样参与一次微调", §Merge 后还是不是训练时的函数: the trained function is
// W_hat together with the adapter; merging delivers W_hat + c·A·B as one
// dense weight, here in bf16:
//   out[k][n] = RN_bf16( ŵ[k][n] + c · Σ_j A[k][j] B[j][n] ),
//   ŵ = RN_bf16(C_j · a'), the same decoded weight as dequantization.
//
// A CTA owns one 64-column NF4 block column and 256 rows; its 64 columns of
// B sit in shared memory, transposed (column n holds B[0..r)[n] contiguous, so
// an mma B fragment is one 32-bit load) with the row stride padded to spread
// the banks.  Each warp computes 32 rows as two 16 x 64 tiles: the rank-r
// product with mma.sync m16n8k16 (bf16 in, fp32 accumulate), then ŵ + c·(A·B)
// in one fp32 fma and one rounding to bf16.  The grid is (N/64) x (K/256).
#include <cfloat>

#include "common.cuh"
#include "kernels.cuh"
#include "profile.cuh"
#include "tmap.cuh"

namespace qnf4 {

__constant__ float kNF4m[32] = {QNF4_TABLE_VALUES, QNF4_INT4_VALUES};   // NF4, INT4

struct MergeArgs {
  int K, N, r;
  float c;
  ScaleView sv;
  const uint8_t* packed;
  const uint16_t* A;   // K x r
  const uint16_t* B;   // r x N
  uint16_t* out;       // K x N
  int32_t* d_status;
};

__device__ __forceinline__ void mma_m16n8k16_bf16(float (&d)[4], const uint32_t (&a)[4],
                                                  uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

constexpr int kMgRows = 256;                 // rows per CTA
constexpr int kMgLd = 64 / 2 + 4;            // 32-bit words per transposed B column (r <= 64)

__global__ void __launch_bounds__(256) nf4_merge_kernel(MergeArgs a) {
  __shared__ float t8[256];
  __shared__ uint32_t bt[64 * kMgLd];        // bt[n][j/2] = (B[j][n], B[j+1][n])
  pdl_launch_dependents();
  if (a.sv.code8 != nullptr) build_t8(t8);
  pdl_wait();   // the table above reads no global memory
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int nb = blockIdx.x, n0 = nb * 64;
  // B[j][n0 .. n0+63] -> bt, rank rows in pairs; rows from r up to the next
  // multiple of 16 (the last mma step) are zero
  const int r16 = (a.r + 15) & ~15;
  for (int i = threadIdx.x; i < (r16 / 2) * 64; i += blockDim.x) {
    const int jp = i >> 6, n = i & 63;
    const uint32_t lo = 2 * jp < a.r ? __ldg(a.B + static_cast<int64_t>(2 * jp) * a.N + n0 + n) : 0u;
    const uint32_t hi =
        2 * jp + 1 < a.r ? __ldg(a.B + static_cast<int64_t>(2 * jp + 1) * a.N + n0 + n) : 0u;
    bt[n * kMgLd + jp] = lo | (hi << 16);
  }
  __syncthreads();
  const int64_t bpr = a.N / 64;
  const float off = a.sv.code8 != nullptr ? __ldg(a.sv.offset) : 0.0f;
  const float* Ctab = kNF4m + 16 * a.sv.codebook;
  bool nonfinite = false;
#pragma unroll 1
  for (int sub = 0; sub < 2; ++sub) {
    const int k0 = blockIdx.y * kMgRows + warp * 32 + sub * 16;
    if (k0 >= a.K) break;   // K is a multiple of 64: rows k0 .. k0+15 all exist
    const int kA = k0 + g, kB = kA + 8;
    float acc[8][4];
#pragma unroll
    for (int s8 = 0; s8 < 8; ++s8)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[s8][i] = 0.0f;
    const int64_t rowA = static_cast<int64_t>(kA) * a.r, rowB = static_cast<int64_t>(kB) * a.r;
    // A[row][j], A[row][j + 1] as one bf16 pair; columns from r on are zero
    // (r may be odd, so the pair is read as two 16-bit values)
    auto a_pair = [&](int64_t row, int j) -> uint32_t {
      const uint32_t lo = j < a.r ? __ldg(a.A + row + j) : 0u;
      const uint32_t hi = j + 1 < a.r ? __ldg(a.A + row + j + 1) : 0u;
      return lo | (hi << 16);
    };
    for (int j0 = 0; j0 < a.r; j0 += 16) {
      uint32_t af[4];
      af[0] = a_pair(rowA, j0 + 2 * t);
      af[1] = a_pair(rowB, j0 + 2 * t);
      af[2] = a_pair(rowA, j0 + 8 + 2 * t);
      af[3] = a_pair(rowB, j0 + 8 + 2 * t);
#pragma unroll
      for (int s8 = 0; s8 < 8; ++s8) {
        const uint32_t* col = bt + (8 * s8 + g) * kMgLd + j0 / 2 + t;
        mma_m16n8k16_bf16(acc[s8], af, col[0], col[4]);
      }
    }
    // decoded weights and the merge, rows kA and kB
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int k = half == 0 ? kA : kB;
      const int64_t blk = static_cast<int64_t>(k) * bpr + nb;
      float sc;
      if (a.sv.code8 == nullptr) {
        sc = __ldg(a.sv.absmax + blk);
      } else {
        sc = __fadd_rn(__fmul_rn(t8[__ldg(a.sv.code8 + blk)], __ldg(a.sv.s2 + (blk >> 8))), off);
      }
      nonfinite |= !(fabsf(sc) <= FLT_MAX);
      const uint4* src =
          reinterpret_cast<const uint4*>(a.packed + (static_cast<int64_t>(k) * a.N + n0) / 2);
      const uint4 q0 = __ldg(src), q1 = __ldg(src + 1);
      const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
      uint16_t* dst = a.out + static_cast<int64_t>(k) * a.N + n0 + 2 * t;
#pragma unroll
      for (int s8 = 0; s8 < 8; ++s8) {
        // byte 4s + t holds columns 8s + 2t (high nibble) and 8s + 2t + 1
        const uint32_t byte = (w[s8] >> (8 * t)) & 0xFFu;
        const float w0 = bf16_bits_to_f32(bf16_of_exact_product(Ctab[byte >> 4], sc));
        const float w1 = bf16_bits_to_f32(bf16_of_exact_product(Ctab[byte & 15u], sc));
        const float m0 = fmaf(a.c, acc[s8][2 * half], w0);
        const float m1 = fmaf(a.c, acc[s8][2 * half + 1], w1);
        *reinterpret_cast<uint32_t*>(dst + 8 * s8) = pack_bf16x2(m0, m1);
      }
    }
  }
  if (nonfinite) raise_status(a.d_status, QLORA_ERR_NONFINITE);
}

// ---------------------------------------------------------------------------
// Tensor-core merge (r a multiple of 8, so that A's rows are 16-byte aligned
// for TMA).  Tiles of 128 rows x 256 columns (four NF4 blocks per row); a CTA
// takes a contiguous range of tiles in row-major order.
//   warp 0      TMA producer: the tile's A rows (128 x 64 rank, K-major,
//               zero beyond r), B columns (64 rank x 256, MN-major, zero
//               beyond r) and packed bytes (128 rows x 128 bytes), 2 stages;
//   warp 1      MMA issuer: the rank-r product A·B (M = 128, N = 256, K = 16
//               per MMA) into one of two TMEM accumulators;
//   warps 2..9  epilogue: the warp of TMEM lane quadrant q and column half h
//               owns rows 32q..32q+31 and columns 128h..128h+127, one row per
//               thread.  Per row and NF4 block it forms the 16-entry table
//               bf16(C_j · a') (single rounding of the exact product), decodes
//               the 64 nibbles through that table (byte permutes), adds
//               c·(A·B) with one fp32 fma, rounds to bf16 into a per-warp
//               staging tile (32 rows x 64 columns, 128-byte swizzle) and
//               stores it with one TMA store.  The scales of the next tile
//               are loaded while the current one is processed.
// ---------------------------------------------------------------------------
constexpr int kMtRows = 128, kMtCols = 256;
constexpr int kMtStages = 2;
constexpr int kMtA = kMtRows * 128;               // 128 rows x 64 rank (bf16)
constexpr int kMtB = 64 * kMtCols * 2;            // 64 rank x 256 columns (bf16), four 64-column boxes
constexpr int kMtP = kMtRows * 128;               // 128 rows x 256 nibbles
constexpr int kMtStage = kMtA + kMtB + kMtP;
constexpr int kMtEpiWarps = 8;
constexpr int kMtOut = 32 * 128;                  // one staging tile: 32 rows x 64 bf16
constexpr int kMtThreads = (2 + kMtEpiWarps) * 32;
constexpr size_t kMtSmem = 1024 + kMtStages * kMtStage + kMtEpiWarps * 2 * kMtOut + 1024 + 256;
static_assert(kMtSmem <= 227 * 1024, "merge tile does not fit in shared memory");

struct MergeTcArgs {
  int K, N, r;
  int tiles_n;            // 256-column tiles per 128-row block
  int tiles;              // all tiles
  float c;
  ScaleView sv;
  int32_t* d_status;
};

__device__ __forceinline__ uint32_t prmt_m(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Eight 4-bit codes (in packing order: the first weight in the high nibble of
// byte 0) -> eight bf16 values, looked up in a 16-entry table whose high and
// low bytes are split into the byte planes H and L (entry e at byte e % 4 of
// word e / 4).  Each 3-bit index picks from the lower and the upper half of a
// plane with one permute each; the code's top bit then selects between them.
__device__ __forceinline__ uint4 decode8_m(uint32_t p, const uint32_t (&H)[4], const uint32_t (&L)[4]) {
  const uint32_t s = p & 0x77777777u;
  const uint32_t b = ((p >> 1) & 0x44444444u) | 0x32103210u;
  uint4 o;
  {
    const uint32_t hF = prmt_m(prmt_m(H[0], H[1], s), prmt_m(H[2], H[3], s), b);
    const uint32_t lF = prmt_m(prmt_m(L[0], L[1], s), prmt_m(L[2], L[3], s), b);
    o.x = prmt_m(lF, hF, 0x4051u);      // weights 0 (low half) and 1
    o.y = prmt_m(lF, hF, 0x6273u);      // weights 2 and 3
  }
  {
    const uint32_t s2 = s >> 16, b2 = b >> 16;
    const uint32_t hF = prmt_m(prmt_m(H[0], H[1], s2), prmt_m(H[2], H[3], s2), b2);
    const uint32_t lF = prmt_m(prmt_m(L[0], L[1], s2), prmt_m(L[2], L[3], s2), b2);
    o.z = prmt_m(lF, hF, 0x4051u);
    o.w = prmt_m(lF, hF, 0x6273u);
  }
  return o;
}

// The raw scale inputs of one row's two NF4 blocks in one column half of a
// tile: with double quantization the 8-bit codes and the second-level scales,
// else the fp32 first-level scales.
struct MergeScales {
  uint32_t code[2];
  float s2[2];
};

__device__ __forceinline__ MergeScales merge_load_scales(const MergeTcArgs& a, int t, int rl, int hc) {
  MergeScales m{{0u, 0u}, {0.0f, 0.0f}};
  if (t < 0) return m;
  const int64_t k = static_cast<int64_t>(t / a.tiles_n) * kMtRows + rl;
  const int nb0 = (t % a.tiles_n) * kMtCols + 128 * hc;
  if (k >= a.K) return m;
  const int64_t bpr = a.N / 64;
#pragma unroll
  for (int bb = 0; bb < 2; ++bb) {
    if (nb0 + 64 * bb >= a.N) break;
    const int64_t blk = k * bpr + (nb0 + 64 * bb) / 64;
    if (a.sv.code8 != nullptr) {
      m.code[bb] = __ldg(a.sv.code8 + blk);
      m.s2[bb] = __ldg(a.sv.s2 + (blk >> 8));
    } else {
      m.s2[bb] = __ldg(a.sv.absmax + blk);
    }
  }
  return m;
}

__global__ void __launch_bounds__(kMtThreads, 1)
    nf4_merge_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmO,
                        MergeTcArgs a) {
  extern __shared__ uint8_t msm_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(msm_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sOut = smem + kMtStages * kMtStage;
  float* t8 = reinterpret_cast<float*>(sOut + kMtEpiWarps * 2 * kMtOut);
  uint64_t* full = reinterpret_cast<uint64_t*>(t8 + 256);
  uint64_t* empty = full + kMtStages;
  uint64_t* afull = empty + kMtStages;     // [2] accumulator ready
  uint64_t* aempty = afull + 2;            // [2] accumulator drained
  uint64_t* drain = aempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (a.sv.code8 != nullptr) build_t8(t8);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kMtStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kMtEpiWarps);   // the MMA's commit and every epilogue warp
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&afull[h], 1);
      mbar_init(&aempty[h], kMtEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  pdl_launch_dependents();
  pdl_wait();
  const int t0 = static_cast<int>((static_cast<int64_t>(blockIdx.x) * a.tiles) / gridDim.x);
  const int t1 = static_cast<int>((static_cast<int64_t>(blockIdx.x + 1) * a.tiles) / gridDim.x);
  const int rsteps = (a.r + 15) >> 4;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      tma_prefetch_desc(&tmP);
      uint32_t last_parity[kMtStages];
      for (int s = 0; s < kMtStages; ++s) last_parity[s] = 2;
      for (int t = t0, i = 0; t < t1; ++t, ++i) {
        const int s = i % kMtStages;
        const uint32_t ph = static_cast<uint32_t>((i / kMtStages) & 1);
        if (*abort_flag || !mbar_wait(&empty[s], ph ^ 1)) { *abort_flag = 1; break; }
        const int k0 = (t / a.tiles_n) * kMtRows, n0 = (t % a.tiles_n) * kMtCols;
        uint8_t* st = smem + s * kMtStage;
        mbar_arrive_expect_tx(&full[s], kMtStage);
        tma_load_2d(st, &tmA, &full[s], 0, k0);
#pragma unroll
        for (int q = 0; q < 4; ++q) tma_load_2d(st + kMtA + q * 8192, &tmB, &full[s], n0 + 64 * q, 0);
        tma_load_2d(st + kMtA + kMtB, &tmP, &full[s], n0 / 2, k0);
        last_parity[s] = ph;
      }
      // no copy may still be landing in this CTA's shared memory when it exits
      for (int s = 0; s < kMtStages; ++s)
        if (last_parity[s] < 2) (void)mbar_wait(&full[s], last_parity[s]);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer -------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kMtRows, kMtCols, 0, 1);
      for (int t = t0, i = 0; t < t1; ++t, ++i) {
        const int s = i % kMtStages, h = i & 1;
        const uint32_t ph = static_cast<uint32_t>((i / kMtStages) & 1);
        const uint32_t hph = static_cast<uint32_t>(((i >> 1) & 1) ^ 1);
        if (*abort_flag || !mbar_wait(&full[s], ph) || !mbar_wait(&aempty[h], hph)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + s * kMtStage), b0 = a0 + kMtA;
        for (int j = 0; j < rsteps; ++j)
          umma_bf16(tmem + h * kMtCols, smem_desc(a0 + j * 32, 16, 1024),
                    smem_desc(b0 + j * 2048, 8192, 1024), idesc, j > 0 ? 1u : 0u);
        umma_commit(&empty[s]);
        umma_commit(&afull[h]);
      }
      umma_commit(drain);
      (void)mbar_wait(drain, 0);
    }
  } else {
    // ------------------------------- epilogue --------------------------------
    const int q = warp & 3, hc = (warp - 2) >> 2;     // TMEM lane quadrant, column half
    const int rl = q * 32 + lane;                      // row within the tile
    const float off = a.sv.code8 != nullptr ? __ldg(a.sv.offset) : 0.0f;
    const float* Ctab = kNF4m + 16 * a.sv.codebook;
    const bool dq = a.sv.code8 != nullptr;
    uint8_t* stage_out = sOut + (warp - 2) * 2 * kMtOut;
    bool nonfinite = false;
    MergeScales nxt = merge_load_scales(a, t0 < t1 ? t0 : -1, rl, hc);
    for (int t = t0, i = 0; t < t1; ++t, ++i) {
      const int h = i & 1, s = i % kMtStages;
      const MergeScales cur = nxt;
      nxt = merge_load_scales(a, t + 1 < t1 ? t + 1 : -1, rl, hc);
      // the accumulator, then the stage's packed bytes (already landed: the
      // MMA waited for them; waited on here so that these threads see them)
      if (*abort_flag || !mbar_wait(&afull[h], static_cast<uint32_t>((i >> 1) & 1)) ||
          !mbar_wait(&full[s], static_cast<uint32_t>((i / kMtStages) & 1))) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int k0 = (t / a.tiles_n) * kMtRows;
      const int n0 = (t % a.tiles_n) * kMtCols + 128 * hc;
      const uint8_t* prow = smem + s * kMtStage + kMtA + kMtB + rl * 128;
#pragma unroll 1
      for (int bb = 0; bb < 2; ++bb) {                 // the two NF4 blocks of this column half
        const uint32_t code = bb ? cur.code[1] : cur.code[0];
        const float s2v = bb ? cur.s2[1] : cur.s2[0];
        const float sc = dq ? __fadd_rn(__fmul_rn(t8[code], s2v), off) : s2v;
        nonfinite |= !(fabsf(sc) <= FLT_MAX);
        // the row's table: entry e = bf16(C_e * sc)
        // (the product of two fp32 values is exact in fp64; one rounding to bf16)
        const double scd = static_cast<double>(sc);
        uint32_t w[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          unsigned short lo, hi;
          asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(lo) : "d"(static_cast<double>(Ctab[2 * j]) * scd));
          asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(hi) : "d"(static_cast<double>(Ctab[2 * j + 1]) * scd));
          w[j] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
        }
        uint32_t H[4], L[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          H[j] = prmt_m(w[2 * j], w[2 * j + 1], 0x7531u);
          L[j] = prmt_m(w[2 * j], w[2 * j + 1], 0x6420u);
        }
        // the 32 packed bytes of this block (16-byte chunks 4hc + 2bb and the
        // next, stored with the 128-byte swizzle: chunk c of row R at c ^ (R & 7))
        const int c0 = 4 * hc + 2 * bb;
        const uint4 pk0 = *reinterpret_cast<const uint4*>(prow + ((c0 ^ (rl & 7)) << 4));
        const uint4 pk1 = *reinterpret_cast<const uint4*>(prow + (((c0 + 1) ^ (rl & 7)) << 4));
        const uint32_t pw[8] = {pk0.x, pk0.y, pk0.z, pk0.w, pk1.x, pk1.y, pk1.z, pk1.w};
        uint8_t* so = stage_out + bb * kMtOut;
        if (lane == 0) bulk_wait_group_read<1>();      // this buffer's previous store has read it
        __syncwarp();
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t v[32];
          const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) +
                                 static_cast<uint32_t>(h * kMtCols + 128 * hc + 64 * bb + 32 * half);
          tmem_ld_32x32b_x32(taddr, v);
          tmem_ld_wait();
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            const uint4 d = decode8_m(pw[4 * half + c8], H, L);   // 8 weights as bf16 pairs
            const uint32_t dw[4] = {d.x, d.y, d.z, d.w};
            uint32_t ow[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float m0 = fmaf(a.c, __uint_as_float(v[8 * c8 + 2 * u]), __uint_as_float(dw[u] << 16));
              const float m1 =
                  fmaf(a.c, __uint_as_float(v[8 * c8 + 2 * u + 1]), __uint_as_float(dw[u] & 0xFFFF0000u));
              ow[u] = pack_bf16x2(m0, m1);
            }
            const int chunk = 4 * half + c8;
            *reinterpret_cast<uint4*>(so + lane * 128 + ((chunk ^ (lane & 7)) << 4)) =
                make_uint4(ow[0], ow[1], ow[2], ow[3]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && n0 + 64 * bb < a.N && k0 + 32 * q < a.K) {   // boxes wholly outside: no store
          tma_store_2d(&tmO, so, n0 + 64 * bb, k0 + 32 * q);
          bulk_commit_group();
        }
      }
      // TMEM accumulator h and the stage's packed bytes are no longer read
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&aempty[h]);
        mbar_arrive(&empty[s]);
      }
    }
    if (lane == 0) bulk_wait_group<0>();
    if (nonfinite) raise_status(a.d_status, QLORA_ERR_NONFINITE);
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) raise_status(a.d_status, QLORA_ERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_merge(int64_t K, int64_t N, int r, float c, ScaleView sv, const uint8_t* packed,
                         const uint16_t* A, const uint16_t* B, uint16_t* out, int32_t* d_status,
                         cudaStream_t st) {
  MergeArgs a;
  a.K = static_cast<int>(K);
  a.N = static_cast<int>(N);
  a.r = r;
  a.c = c;
  a.sv = sv;
  a.packed = packed;
  a.A = A;
  a.B = B;
  a.out = out;
  a.d_status = d_status;
  cudaError_t e;
  if (r % 8 == 0) {
    static DeviceOnce once;
    e = once.run([](int) {
      return cudaFuncSetAttribute(nf4_merge_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kMtSmem));
    });
    if (e != cudaSuccess) return e;
    constexpr CUtensorMapDataType kBF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    constexpr CUtensorMapSwizzle kSW128 = CU_TENSOR_MAP_SWIZZLE_128B;
    CUtensorMap tA, tB, tP, tO;
    if (!make_tmap_2d(&tA, A, kBF16, 2, K, r, r, 64, kMtRows, kSW128) ||
        !make_tmap_2d(&tB, B, kBF16, 2, r, N, N, 64, 64, kSW128) ||
        !make_tmap_2d(&tP, packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, N / 2, N / 2, 128, kMtRows, kSW128) ||
        !make_tmap_2d(&tO, out, kBF16, 2, K, N, N, 64, 32, kSW128))
      return cudaErrorInvalidValue;
    MergeTcArgs m;
    m.K = static_cast<int>(K);
    m.N = static_cast<int>(N);
    m.r = r;
    m.tiles_n = static_cast<int>((N + kMtCols - 1) / kMtCols);
    m.tiles = static_cast<int>((K + kMtRows - 1) / kMtRows) * m.tiles_n;
    m.c = c;
    m.sv = sv;
    m.d_status = d_status;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = m.tiles < sms ? m.tiles : sms;
    {
      ProfScope prof(kProfDequantize, st);
      e = launch_pdl(nf4_merge_tc_kernel, dim3(grid), dim3(kMtThreads), kMtSmem, st, 1, tA, tB, tP, tO, m);
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  const dim3 grid(static_cast<unsigned>(N / 64), static_cast<unsigned>((K + kMgRows - 1) / kMgRows));
  {
    ProfScope prof(kProfDequantize, st);
    e = launch_pdl(nf4_merge_kernel, grid, dim3(256), 0, st, 1, a);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace qnf4
